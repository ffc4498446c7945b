// LSE merge of the partials of units split across warps (device code).
#pragma once

#include "paged_decode_kernel.cuh"

namespace pa {

// --------------------------------------------------------------- merge kernel

// Threads of one merge CTA: enough that every (q-head, 4 columns) item has
// several threads sharing out the contributors.
__host__ __device__ constexpr int merge_threads(int D, int G) { return G * D / 4 >= 256 ? 1024 : 256; }

// One online-softmax fold of a partial (ml, o) into the running (m, l, acc).
__device__ __forceinline__ void fold_partial(float& m, float& l, float4& acc, float2 ml, float4 o) {
  const float mn = fmaxf(m, ml.x);
  const float sa = fast_exp2(m - mn), sb = fast_exp2(ml.x - mn);
  l = l * sa + ml.y * sb;
  acc.x = acc.x * sa + o.x * sb;
  acc.y = acc.y * sa + o.y * sb;
  acc.z = acc.z * sa + o.z * sb;
  acc.w = acc.w * sa + o.w * sb;
  m = mn;
}

// Combines the partials of a unit split across warps w0..w1:
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p
// (m in log2 units).  One CTA per merge job.  The contributors' partial
// slots are resolved once into shared memory; thread (group, item) then folds
// contributors j = group, group + NGRP, ... of one (q-head, 4 columns) item
// into a running (m, l, acc), loading four contributors at a time, and the
// NGRP groups are combined once through shared memory.
template <typename T, int D, int G>
__global__ void __launch_bounds__(merge_threads(D, G)) paged_decode_merge_kernel(const DecodeParams p) {
  using E = Elem<T>;
  constexpr int NT = merge_threads(D, G);
  constexpr int ITEMS = G * D / 4;  // float4 outputs of one job
  constexpr int NGRP = NT / ITEMS;  // contributor groups
  extern __shared__ int mslots[];   // [W]: partial slot of each contributor, -1 if it has none
  __shared__ float4 s_acc[NT];
  __shared__ float2 s_ml[NT];

  griddep_wait();
  griddep_launch_dependents();
  const int W = p.total_warps;
  const int4 job = p.ws_jobs[blockIdx.x];
  if (job.x < 0) return;
  const int64_t NC = p.ws_header[0];
  const int64_t a = job.z, b = a + job.w;
  const int w0 = blockIdx.x;
  const int w1 = static_cast<int>((b * W + NC - 1) / NC - 1);  // warp holding chunk b-1
  const int nw = w1 - w0 + 1;
  const int t = threadIdx.x;
  for (int j = t; j < nw; j += NT) {
    const int64_t w = w0 + j;
    const int64_t s0 = w * NC / W, s1 = (w + 1) * NC / W;  // warps with an empty run wrote nothing
    mslots[j] = s0 < s1 ? static_cast<int>(2 * w + (s0 >= a ? 0 : 1)) : -1;
  }
  __syncthreads();

  const int item = t % ITEMS, grp = t / ITEMS;
  const int g = item / (D / 4), d4 = item % (D / 4);
  auto ml_at = [&](int slot) { return p.ws_ml[(int64_t)slot * G + g]; };
  auto o_at = [&](int slot) { return reinterpret_cast<const float4*>(p.ws_o + ((int64_t)slot * G + g) * D)[d4]; };
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  int j = grp;
  for (; j + 3 * NGRP < nw; j += 4 * NGRP) {
    int sl[4];
    float2 ml[4];
    float4 o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      sl[u] = mslots[j + u * NGRP];
      const int safe = sl[u] < 0 ? 0 : sl[u];  // a valid address; its values are not used
      ml[u] = ml_at(safe);
      o[u] = o_at(safe);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (sl[u] >= 0 && ml[u].x != -INFINITY) fold_partial(m, l, acc, ml[u], o[u]);
  }
  for (; j < nw; j += NGRP) {
    const int slot = mslots[j];
    if (slot < 0) continue;
    const float2 ml = ml_at(slot);
    if (ml.x != -INFINITY) fold_partial(m, l, acc, ml, o_at(slot));
  }
  if (NGRP > 1) {
    s_acc[t] = acc;
    s_ml[t] = make_float2(m, l);
    __syncthreads();
    if (grp != 0) return;
    for (int q = 1; q < NGRP; ++q) {
      const float2 ml = s_ml[q * ITEMS + item];
      if (ml.x != -INFINITY) fold_partial(m, l, acc, ml, s_acc[q * ITEMS + item]);
    }
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  T* dst = static_cast<T*>(p.out) + ((int64_t)job.x * p.num_heads + (int64_t)job.y * G + g) * D + d4 * 4;
  uint2 u;
  u.x = E::pack(acc.x * inv, acc.y * inv);
  u.y = E::pack(acc.z * inv, acc.w * inv);
  *reinterpret_cast<uint2*>(dst) = u;
}

}  // namespace pa
