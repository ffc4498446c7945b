// Log-sum-exp merge of a unit split across warps, run inside the decode
// kernel by the last warp to finish its part of the unit (device code).
//
// A (sequence, kv-head) unit whose chunks span several warps' runs leaves one
// un-normalised partial (m, l, o) per contributing warp, m in log2 units:
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p
// ("【infra之路】10-PagedAttention 与 KV Cache 管理", section 8 Q2: FlashDecoding
// splits a long context and combines the pieces; this is that combination).
#pragma once

#include "pa_device.cuh"

namespace pa {

// The global chunk order is split evenly over W warps: warp w runs chunks
// [floor(w*NC/W), floor((w+1)*NC/W)).
__device__ __forceinline__ int64_t run_begin(int64_t w, int64_t NC, int W) { return w * NC / W; }

// The warp whose run holds global chunk g: the w with
// floor(w*NC/W) <= g < floor((w+1)*NC/W), i.e. ceil((g+1)*W/NC) - 1.
__device__ __forceinline__ int warp_of_chunk(int64_t g, int64_t NC, int W) {
  return static_cast<int>(((g + 1) * W + NC - 1) / NC - 1);
}

// Partial slot of warp w's part of the unit that starts at global chunk a:
// slot 2w holds a warp's first segment, slot 2w+1 its last.  The part is the
// warp's first segment exactly when its run starts at or after a.
__device__ __forceinline__ int64_t partial_slot(int64_t w, int64_t a, int64_t NC, int W) {
  return 2 * w + (run_begin(w, NC, W) >= a ? 0 : 1);
}

// One online-softmax fold of a partial (ml = (m, l), o) into (m, l, acc).
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

// Merge the partials of the unit of `nc` chunks starting at global chunk `a`
// and write its G q-head rows (out_row -> [G][D]).  One warp; lane i owns
// the float4 columns i, i+32, ... of the G*D outputs.  The partials were
// written by other warps of this grid and published by their tickets'
// release (the caller acquired them with the last ticket), so they are read
// through L2 (ld.global.cg), never from a possibly stale L1 line.  A partial
// whose running max is -inf (every token of that part skipped) adds nothing.
template <typename T, int D, int G>
__device__ __forceinline__ void merge_split_unit(const float2* ws_ml, const float* ws_o, T* out_row, int64_t a,
                                                 int nc, int64_t NC, int W, int lane) {
  using E = Elem<T>;
  constexpr int kItems = G * D / 4;                   // float4 outputs
  constexpr int kPerLane = (kItems + 31) / 32;
  // contributors loaded before folding: about eight float4 columns in flight
  // per lane, whatever G (the merge runs inside the streaming loop and its
  // registers add to the loop's)
  constexpr int kBatch = kPerLane >= 8 ? 1 : 8 / kPerLane;
  const int w0 = warp_of_chunk(a, NC, W);
  const int w1 = warp_of_chunk(a + nc - 1, NC, W);
  float m[kPerLane], l[kPerLane];
  float4 acc[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
    acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int w = w0; w <= w1; w += kBatch) {
    float2 ml[kBatch][kPerLane];
    float4 o[kBatch][kPerLane];
    bool use[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int wu = w + u;
      // Warps with an empty run (more warps than chunks) wrote nothing.
      use[u] = wu <= w1 && run_begin(wu, NC, W) < run_begin(wu + 1, NC, W);
      const int64_t slot = use[u] ? partial_slot(wu, a, NC, W) : 0;
#pragma unroll
      for (int i = 0; i < kPerLane; ++i) {
        const int item = lane + 32 * i;
        const int g = item / (D / 4), d4 = item % (D / 4);
        if (use[u] && item < kItems) {
          ml[u][i] = __ldcg(ws_ml + slot * G + g);
          o[u][i] = __ldcg(reinterpret_cast<const float4*>(ws_o + (slot * G + g) * D) + d4);
        } else {
          ml[u][i] = make_float2(-INFINITY, 0.f);
          o[u][i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
#pragma unroll
      for (int i = 0; i < kPerLane; ++i)
        if (ml[u][i].x != -INFINITY) fold_partial(m[i], l[i], acc[i], ml[u][i], o[u][i]);
    }
  }
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int item = lane + 32 * i;
    if (item >= kItems) continue;
    const int g = item / (D / 4), d4 = item % (D / 4);
    const float inv = l[i] > 0.f ? 1.f / l[i] : 0.f;
    uint2 u;
    u.x = E::pack(acc[i].x * inv, acc[i].y * inv);
    u.y = E::pack(acc[i].z * inv, acc[i].w * inv);
    *reinterpret_cast<uint2*>(out_row + g * D + d4 * 4) = u;
  }
}

}  // namespace pa
