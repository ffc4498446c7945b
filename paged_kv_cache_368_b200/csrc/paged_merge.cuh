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
// [floor(w*NC/W), floor((w+1)*NC/W)).  The run bounds are evaluated without
// 64-bit division (a long emulated sequence that every merge and ticket
// used to pay several times): with NC = q*W + r, floor(w*NC/W) =
// w*q + floor(w*r/W), and w*r < W*W fits 32 bits.
struct RunSplit {
  int64_t NC;
  int64_t q;  // NC / W
  uint32_t r;  // NC % W
  int W;

  __device__ __forceinline__ void init(int64_t nc, int w) {
    NC = nc;
    W = w;
    q = nc / w;
    r = static_cast<uint32_t>(nc - q * w);
  }

  __device__ __forceinline__ int64_t begin(int w) const {
    return (int64_t)w * q + (int64_t)((static_cast<uint32_t>(w) * r) / static_cast<uint32_t>(W));
  }

  // The warp whose run holds global chunk g: the w with begin(w) <= g <
  // begin(w+1), which is ceil((g+1)*W/NC) - 1.  That quotient (below 2^11)
  // is estimated in single precision, whose few roundings move it by far
  // less than 1, so the estimate is off by at most one; the run bounds then
  // settle it exactly.
  __device__ __forceinline__ int warp_of(int64_t g) const {
    if (NC <= 0) return 0;
    const float x = static_cast<float>(g + 1) * static_cast<float>(W) / static_cast<float>(NC);
    int w = static_cast<int>(ceilf(x)) - 1;
    w = w < 0 ? 0 : (w > W - 1 ? W - 1 : w);
    if (begin(w) > g) {
      --w;
    } else if (w + 1 < W && begin(w + 1) <= g) {
      ++w;
    }
    return w;
  }

  // Partial slot of warp w's part of the unit that starts at global chunk a:
  // slot 2w holds a warp's first segment, slot 2w+1 its last.  The part is
  // the warp's first segment exactly when its run starts at or after a.
  __device__ __forceinline__ int partial_slot(int w, int64_t a) const { return 2 * w + (begin(w) >= a ? 0 : 1); }
};

// Merge the partials of the unit of `nc` chunks starting at global chunk `a`
// and write its G q-head rows (out_row -> [G][D]).  One warp, two phases per
// block of up to 32 contributors:
//  1. lane j reads contributor j's (m, l) for every q-head; warp reductions
//     give the block's maximum M_g and each contributor's weight
//     2^(m_jg - M_g) (folded into the running maximum of earlier blocks);
//  2. lane i owns the float4 output columns i, i+32, ... and adds up
//     weight * o over the block's contributors.  The weights are known, so
//     the loads of several contributors are independent and in flight
//     together (up to 16 float4 columns per lane), instead of one round trip
//     per contributor.
// The partials were written by other warps of this grid and published by
// their tickets' release (the caller acquired them with the last ticket), so
// they are read through L2 (ld.global.cg), never from a possibly stale L1
// line.  A partial whose running max is -inf (every token of that part
// skipped) has weight 0.
template <typename T, int D, int G>
__device__ __forceinline__ void merge_split_unit(const float2* ws_ml, const float* ws_o, T* out_row, int64_t a,
                                                 int nc, const RunSplit& rs, int lane) {
  using E = Elem<T>;
  constexpr int kItems = G * D / 4;          // float4 outputs
  constexpr int kPerLane = (kItems + 31) / 32;
  constexpr int kBatch = kPerLane >= 8 ? 1 : 4;  // contributors in flight in phase 2
  constexpr int kHeadItems = D / 4;          // float4 columns of one q-head
  const int w0 = rs.warp_of(a);
  const int nw = rs.warp_of(a + nc - 1) - w0 + 1;
  float M[G], L[G];  // running maximum (log2 units) and weighted sum of l, per q-head
  float4 acc[kPerLane];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    M[g] = -INFINITY;
    L[g] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);

  for (int base = 0; base < nw; base += 32) {
    // ---- phase 1: this lane's contributor of the block
    const int wj = w0 + base + lane;
    // Warps with an empty run (more warps than chunks) wrote nothing.
    const bool has = base + lane < nw && rs.begin(wj) < rs.begin(wj + 1);
    const int slot = has ? rs.partial_slot(wj, a) : 0;
    float wgt[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float2 ml = has ? __ldcg(ws_ml + (int64_t)slot * G + g) : make_float2(-INFINITY, 0.f);
      float mb = ml.x;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, off));
      const float mn = fmaxf(M[g], mb);
      // rescale what earlier blocks accumulated for this head to the new maximum
      const float rs = M[g] == -INFINITY ? 0.f : fast_exp2(M[g] - mn);
      if (rs != 1.f) {
        L[g] *= rs;
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
          if ((lane + 32 * i) / kHeadItems == g) {
            acc[i].x *= rs;
            acc[i].y *= rs;
            acc[i].z *= rs;
            acc[i].w *= rs;
          }
        }
      }
      M[g] = mn;
      wgt[g] = ml.x == -INFINITY ? 0.f : fast_exp2(ml.x - mn);
      float ls = wgt[g] * ml.y;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) ls += __shfl_xor_sync(kFull, ls, off);
      L[g] += ls;
    }
    // ---- phase 2: weighted sum of the block's partial outputs
    const int nb = min(32, nw - base);
    for (int j = 0; j < nb; j += kBatch) {
      float4 o[kBatch][kPerLane];
      float wv[kBatch][kPerLane];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int src = min(j + u, 31);
        const bool use = j + u < nb && __shfl_sync(kFull, has, src);
        const int sl = __shfl_sync(kFull, slot, src);
        float wg[G];
#pragma unroll
        for (int g = 0; g < G; ++g) wg[g] = __shfl_sync(kFull, wgt[g], src);
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
          const int item = lane + 32 * i;
          const int g = item / kHeadItems, d4 = item % kHeadItems;
          float w = 0.f;
#pragma unroll
          for (int gg = 0; gg < G; ++gg) w = gg == g ? wg[gg] : w;
          wv[u][i] = use ? w : 0.f;
          o[u][i] = (use && item < kItems && w != 0.f)
                        ? __ldcg(reinterpret_cast<const float4*>(ws_o + ((int64_t)sl * G + g) * D) + d4)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
#pragma unroll
        for (int i = 0; i < kPerLane; ++i) {
          acc[i].x = fmaf(wv[u][i], o[u][i].x, acc[i].x);
          acc[i].y = fmaf(wv[u][i], o[u][i].y, acc[i].y);
          acc[i].z = fmaf(wv[u][i], o[u][i].z, acc[i].z);
          acc[i].w = fmaf(wv[u][i], o[u][i].w, acc[i].w);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int item = lane + 32 * i;
    if (item >= kItems) continue;
    const int g = item / kHeadItems, d4 = item % kHeadItems;
    float lg = 0.f;
#pragma unroll
    for (int gg = 0; gg < G; ++gg) lg = gg == g ? L[gg] : lg;
    const float inv = lg > 0.f ? 1.f / lg : 0.f;
    uint2 u;
    u.x = E::pack(acc[i].x * inv, acc[i].y * inv);
    u.y = E::pack(acc[i].z * inv, acc[i].w * inv);
    *reinterpret_cast<uint2*>(out_row + g * D + d4 * 4) = u;
  }
}

}  // namespace pa
