// Device code of the paged decode kernel (see paged_decode.cu for the design
// notes and the host side).
#pragma once

#include <type_traits>

#include "pa_device.cuh"
#include "paged_merge.cuh"

namespace pa {

constexpr int kChunk = 16;       // tokens per pipeline stage
constexpr int kMaxSeqs = 16384;  // prefix table lives in shared memory (4 bytes a sequence)
#ifndef PA_CORE_WARPS
#define PA_CORE_WARPS 8
#endif
#ifndef PA_CORE_DEPTH
#define PA_CORE_DEPTH 2
#endif
#ifndef PA_MMA_WARPS
#define PA_MMA_WARPS 6
#endif
#ifndef PA_MMA_DEPTH
#define PA_MMA_DEPTH 2
#endif
#ifndef PA_D64_DEPTH
#define PA_D64_DEPTH 4
#endif

// Warps per CTA and pipeline stages per warp for a shape (head_dim D, group G):
// the per-warp ring of DEPTH stages must fit the 227 KB of shared memory.
__host__ __device__ constexpr bool uses_mma(int G) { return G >= 4; }
__host__ __device__ constexpr int warps_for(int D, int G) {
  return D == 64 ? 8 : (uses_mma(G) ? PA_MMA_WARPS : PA_CORE_WARPS);
}
static_assert(PA_CORE_WARPS <= 8 && PA_MMA_WARPS <= 8, "the workspace's ticket region holds 8 warps per SM");
__host__ __device__ constexpr int depth_for(int D, int G) {
  return D == 64 ? PA_D64_DEPTH : (uses_mma(G) ? PA_MMA_DEPTH : PA_CORE_DEPTH);
}
constexpr uint64_t kWaitLimitNs = 1000000000ull;

struct DecodeParams {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_o;       // [2W][G][D] un-normalised partial outputs
  float2* ws_ml;     // [2W][G] (running max in log2 units, running sum)
  int* ws_tickets;   // [W] chunks of a split unit accounted for so far, indexed
                     // by the warp holding the unit's first chunk; every
                     // launch leaves them at zero (callers zero them once)
  int32_t* err_flags;
  int64_t num_blocks;
  int num_seqs;
  int max_blocks_per_seq;
  int ctx_cap;       // min(max_context_len, max_blocks_per_seq * block_size)
  int max_context_len;
  int num_heads;
  int num_kv_heads;
  int block_size;
  int total_warps;
  float scale_log2;  // scale * log2(e)
};

template <int D, int G>
struct Shape {
  static constexpr bool kMma = uses_mma(G);
  static constexpr int kWarps = warps_for(D, G);
  static constexpr int kDepth = depth_for(D, G);
  static constexpr int kTileBytes = kChunk * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQBytes = G * D * 2;
  static constexpr int kStages = kWarps * kDepth;
  static constexpr size_t kFixedSmem =
      1024 + size_t(kStages) * kStageBytes + size_t(kStages) * kQBytes + size_t(kStages) * 8;
  static size_t smem_bytes(int num_seqs) { return kFixedSmem + ((size_t(num_seqs) + 1) * 4 + 15) / 16 * 16; }
};

// --------------------------------------------------------------- chunk lookup

__device__ __forceinline__ int clamp_ctx(int ctx, int cap) { return ctx < 0 ? 0 : (ctx > cap ? cap : ctx); }

// Raw lookup of chunk `g` of the global chunk order: its unit and index from
// the shared-memory prefix table, plus the three global words it needs
// (context length and one or two block-table entries).  Windows of 32 chunks
// are loaded one window ahead of use, so these loads never stall the warp.
struct ChunkRaw {
  int seq;  // -1: no chunk
  int head, c, nc;
  int ctx, p0, p1;
};

// Unit (sequence, kv-head) of global chunk g < KVH * prefix[S], the chunk's
// index c in it and the unit's chunk count nc (shared-memory lookups only).
struct UnitPos {
  int seq, head, c, nc;
};

__device__ __forceinline__ UnitPos unit_pos(const DecodeParams& p, const int* prefix, int64_t g) {
  const int KVH = p.num_kv_heads;
  int lo = 0, hi = p.num_seqs;  // largest s in [0, S) with KVH*prefix[s] <= g
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)KVH * prefix[mid] <= g) lo = mid; else hi = mid;
  }
  UnitPos u;
  u.seq = lo;
  u.nc = prefix[lo + 1] - prefix[lo];
  const int rem = static_cast<int>(g - (int64_t)KVH * prefix[lo]);
  u.head = rem / u.nc;
  u.c = rem - u.head * u.nc;
  return u;
}

__device__ __forceinline__ ChunkRaw chunk_load(const DecodeParams& p, const int* prefix, int64_t g, int64_t end) {
  ChunkRaw r;
  r.seq = -1;
  r.head = r.c = r.nc = r.ctx = r.p0 = 0;
  r.p1 = -1;
  if (g >= end) return r;
  const UnitPos u = unit_pos(p, prefix, g);
  const int s = u.seq, c = u.c;
  const int32_t* row = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
  r.seq = s;
  r.head = u.head;
  r.c = c;
  r.nc = u.nc;
  r.ctx = __ldg(p.context_lens + s);
  if (p.block_size >= kChunk) {
    r.p0 = __ldg(row + c * kChunk / p.block_size);
  } else {  // two blocks of 8 tokens; the second may lie past the context
    r.p0 = __ldg(row + 2 * c);
    if (2 * c + 1 < p.max_blocks_per_seq) r.p1 = __ldg(row + 2 * c + 1);
  }
  return r;
}

// Per-chunk words the warp shuffles around:
//   sh    = seq | kv_head << 16
//   flags = valid tokens (bits 0-4) | first row in the block (bits 5-10)
//           | first chunk of its unit (bit 11) | last chunk of its unit (bit 12)
//           | one of the unit's first kHeadChunks chunks (bit 13)
//   p0/p1 = physical block(s); p1 = -1 when the chunk has one block.
constexpr int kFlagStart = 1 << 11;
constexpr int kFlagEnd = 1 << 12;
constexpr int kFlagHead = 1 << 13;

// L2 residency: blocks shared between sequences (a common prompt prefix,
// beams forked from one request: "【infra之路】10-PagedAttention 与 KV Cache
// 管理", section 4.3) sit at the front of their sequences.  With
// PA_HEAD_CHUNKS > 0 the first PA_HEAD_CHUNKS chunks of every unit are loaded
// with the normal L2 policy and everything after them evict-first, so that a
// shared front block read by one sequence can still be in L2 when its
// sharers read it.  Off by default: at 64 chunks (1024 tokens) it cost ~2 us
// per call on the LLaMA-7B workload, where nothing is shared.
#ifndef PA_HEAD_CHUNKS
#define PA_HEAD_CHUNKS 0
#endif
constexpr int kHeadChunks = PA_HEAD_CHUNKS;


struct ChunkInfo {
  int sh, flags, p0, p1, c, nc;
};

__device__ __forceinline__ ChunkInfo chunk_finalize(const DecodeParams& p, const ChunkRaw& r) {
  ChunkInfo ci;
  ci.sh = ci.flags = ci.p0 = 0;
  ci.p1 = -1;
  ci.c = r.c;
  ci.nc = r.nc;
  if (r.seq < 0) return ci;
  const int ctx = clamp_ctx(r.ctx, p.ctx_cap);
  const int t0 = r.c * kChunk;
  int valid = min(kChunk, ctx - t0);
  int p1 = (p.block_size < kChunk && t0 + 8 < ctx) ? r.p1 : -1;
  const bool ok = r.p0 >= 0 && r.p0 < p.num_blocks && (p1 == -1 || (p1 >= 0 && p1 < p.num_blocks));
  if (!ok) {
    set_err(p.err_flags, PA_ERRF_BLOCK_RANGE);
    valid = 0;
    p1 = -1;
  }
  const int row0 = p.block_size >= kChunk ? t0 % p.block_size : 0;
  ci.sh = r.seq | (r.head << 16);
  ci.flags = valid | (row0 << 5) | (r.c == 0 ? kFlagStart : 0) | (r.c == r.nc - 1 ? kFlagEnd : 0) |
             (r.c < kHeadChunks ? kFlagHead : 0);
  ci.p0 = r.p0;
  ci.p1 = p1;
  return ci;
}

// --------------------------------------------------------------- CUDA-core path

template <typename T, int D, int G>
struct CoreWarp {
  using E = Elem<T>;
  static constexpr int LPT = D / 8;         // lanes per 16-byte-vectorised row
  static constexpr int TPW = 32 / LPT;      // token rows per warp instruction
  static constexpr int IT = kChunk / TPW;   // instructions per chunk

  float qf[G][8];
  float o[G][8];
  float m[G], l[G];

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY;
      l[g] = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) o[g][e] = 0.f;
    }
  }

  __device__ __forceinline__ void load_q(uint32_t qslot, float scale_log2, int lane) {
    const int j = lane % LPT;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint4 u = lds128(qslot + g * D * 2 + j * 16);
      const float2 a = E::to_f2(u.x), b = E::to_f2(u.y), c = E::to_f2(u.z), d = E::to_f2(u.w);
      qf[g][0] = a.x * scale_log2; qf[g][1] = a.y * scale_log2;
      qf[g][2] = b.x * scale_log2; qf[g][3] = b.y * scale_log2;
      qf[g][4] = c.x * scale_log2; qf[g][5] = c.y * scale_log2;
      qf[g][6] = d.x * scale_log2; qf[g][7] = d.y * scale_log2;
    }
  }

  template <bool kMasked>
  __device__ __forceinline__ void chunk(uint32_t ktile, uint32_t vtile, int valid, int lane) {
    const int grp = lane / LPT, j = lane % LPT;
    float acc[G][IT];
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const int tok = it * TPW + grp;
      const uint4 u = lds128(ktile + tile_off(tok, j));
      const float2 a = E::to_f2(u.x), b = E::to_f2(u.y), c = E::to_f2(u.z), d = E::to_f2(u.w);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float s = qf[g][0] * a.x;
        s = fmaf(qf[g][1], a.y, s);
        s = fmaf(qf[g][2], b.x, s);
        s = fmaf(qf[g][3], b.y, s);
        s = fmaf(qf[g][4], c.x, s);
        s = fmaf(qf[g][5], c.y, s);
        s = fmaf(qf[g][6], d.x, s);
        s = fmaf(qf[g][7], d.y, s);
        acc[g][it] = s;
      }
    }
    // Transposing reduction over the LPT lanes of a row group: each step
    // halves the values a lane keeps; afterwards lane j holds the full dot
    // product of token (j >> 1) * TPW + grp (lanes j and j^1 agree).
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int step = IT / 2, mask = LPT / 2; step >= 1; step >>= 1, mask >>= 1) {
        const bool upper = (j & mask) != 0;
#pragma unroll
        for (int i = 0; i < step; ++i) {
          const float send = upper ? acc[g][i] : acc[g][i + step];
          const float keep = upper ? acc[g][i + step] : acc[g][i];
          acc[g][i] = keep + __shfl_xor_sync(kFull, send, mask);
        }
      }
      acc[g][0] += __shfl_xor_sync(kFull, acc[g][0], 1);
    }
    const int my_tok = (j >> 1) * TPW + grp;
    float pg[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float s = (!kMasked || my_tok < valid) ? acc[g][0] : -INFINITY;
      float cm = s;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, off));
      const float mn = fmaxf(m[g], cm);
      const float alpha = fast_exp2(m[g] - mn);
      const float pv = fast_exp2(s - mn);
      l[g] = l[g] * alpha + ((j & 1) ? 0.f : pv);
#pragma unroll
      for (int e = 0; e < 8; ++e) o[g][e] *= alpha;
      m[g] = mn;
      pg[g] = pv;
    }
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const int tok = it * TPW + grp;
      float pt[G];
#pragma unroll
      for (int g = 0; g < G; ++g) pt[g] = __shfl_sync(kFull, pg[g], grp * LPT + 2 * it);
      if (!kMasked || tok < valid) {
        const uint4 u = lds128(vtile + tile_off(tok, j));
        const float2 a = E::to_f2(u.x), b = E::to_f2(u.y), c = E::to_f2(u.z), d = E::to_f2(u.w);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          o[g][0] = fmaf(pt[g], a.x, o[g][0]);
          o[g][1] = fmaf(pt[g], a.y, o[g][1]);
          o[g][2] = fmaf(pt[g], b.x, o[g][2]);
          o[g][3] = fmaf(pt[g], b.y, o[g][3]);
          o[g][4] = fmaf(pt[g], c.x, o[g][4]);
          o[g][5] = fmaf(pt[g], c.y, o[g][5]);
          o[g][6] = fmaf(pt[g], d.x, o[g][6]);
          o[g][7] = fmaf(pt[g], d.y, o[g][7]);
        }
      }
    }
  }

  // Sum the row groups and the lanes' running sums.
  __device__ __forceinline__ void finish() {
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int off = LPT; off < 32; off <<= 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) o[g][e] += __shfl_xor_sync(kFull, o[g][e], off);
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) l[g] += __shfl_xor_sync(kFull, l[g], off);
    }
  }

  __device__ __forceinline__ void write_out(T* out_row, int lane) const {  // out_row -> [G][D]
    const int j = lane % LPT;
    if (lane >= LPT) return;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float inv = l[g] > 0.f ? 1.f / l[g] : 0.f;
      uint4 u;
      u.x = E::pack(o[g][0] * inv, o[g][1] * inv);
      u.y = E::pack(o[g][2] * inv, o[g][3] * inv);
      u.z = E::pack(o[g][4] * inv, o[g][5] * inv);
      u.w = E::pack(o[g][6] * inv, o[g][7] * inv);
      *reinterpret_cast<uint4*>(out_row + g * D + j * 8) = u;
    }
  }

  __device__ __forceinline__ void write_partial(float* po, float2* pml, int lane) const {  // po -> [G][D]
    const int j = lane % LPT;
    if (lane < LPT) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float4* dst = reinterpret_cast<float4*>(po + g * D + j * 8);
        dst[0] = make_float4(o[g][0], o[g][1], o[g][2], o[g][3]);
        dst[1] = make_float4(o[g][4], o[g][5], o[g][6], o[g][7]);
      }
    }
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < G; ++g) pml[g] = make_float2(m[g], l[g]);
    }
  }
};

// --------------------------------------------------------------- tensor-core path

template <typename T, int D, int G>
struct MmaWarp {
  using E = Elem<T>;
  static constexpr int NT = D / 8;   // 8-wide output column tiles
  static constexpr int KS = D / 16;  // k-steps of the QK product

  uint32_t qa[KS][2];  // A fragments of Q (rows = q-heads 0..7; rows 8..15 are zero)
  float o[NT][2];      // O rows gid, columns 8*n + 2*tq + {0,1}
  float m, l;

  // D[0..1] += A * B for the upper 8 rows of a 16x8 tile; the lower rows of A
  // are zero, so the lower rows of D are discarded.
  __device__ static __forceinline__ void mma_top(float& d0, float& d1, uint32_t a0, uint32_t a2, uint32_t b0,
                                                 uint32_t b1) {
    float d[4] = {d0, d1, 0.f, 0.f};
    E::mma(d, a0, 0u, a2, 0u, b0, b1);
    d0 = d[0];
    d1 = d[1];
  }

  __device__ __forceinline__ void reset() {
    m = -INFINITY;
    l = 0.f;
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = 0.f;
  }

  __device__ __forceinline__ void load_q(uint32_t qslot, float /*scale_log2*/, int lane) {
    const int gid = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t a0 = 0u, a2 = 0u;
      if (gid < G) {
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a0) : "r"(qslot + (gid * D + ks * 16 + 2 * tq) * 2));
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a2) : "r"(qslot + (gid * D + ks * 16 + 8 + 2 * tq) * 2));
      }
      qa[ks][0] = a0;
      qa[ks][1] = a2;
    }
  }

  template <bool kMasked>
  __device__ __forceinline__ void chunk(uint32_t ktile, uint32_t vtile, int valid, int lane, float scale_log2) {
    const int gid = lane >> 2, tq = lane & 3;
    // S = Q K^T for tokens 0-7 (n-tile 0) and 8-15 (n-tile 1); two
    // accumulators per tile (even/odd k-step pairs) shorten the mma chains.
    float s[2][2][2] = {};
#pragma unroll
    for (int kp = 0; kp < D / 32; ++kp) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(ktile + tile_off(nt * 8 + (lane & 7), kp * 4 + (lane >> 3)), b0, b1, b2, b3);
        mma_top(s[nt][kp & 1][0], s[nt][kp & 1][1], qa[2 * kp][0], qa[2 * kp][1], b0, b1);
        mma_top(s[nt][kp & 1][0], s[nt][kp & 1][1], qa[2 * kp + 1][0], qa[2 * kp + 1][1], b2, b3);
      }
    }
    float sc[4];
    sc[0] = (s[0][0][0] + s[0][1][0]) * scale_log2;
    sc[1] = (s[0][0][1] + s[0][1][1]) * scale_log2;
    sc[2] = (s[1][0][0] + s[1][1][0]) * scale_log2;
    sc[3] = (s[1][0][1] + s[1][1][1]) * scale_log2;
    if (kMasked) {
      const int t0 = 2 * tq;
      if (t0 >= valid) sc[0] = -INFINITY;
      if (t0 + 1 >= valid) sc[1] = -INFINITY;
      if (t0 + 8 >= valid) sc[2] = -INFINITY;
      if (t0 + 9 >= valid) sc[3] = -INFINITY;
    }
    float cm = fmaxf(fmaxf(sc[0], sc[1]), fmaxf(sc[2], sc[3]));
    cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 1));
    cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 2));
    const float mn = fmaxf(m, cm);
    const float alpha = fast_exp2(m - mn);
    float pr[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) pr[i] = fast_exp2(sc[i] - mn);
    l = l * alpha + ((pr[0] + pr[1]) + (pr[2] + pr[3]));
    m = mn;
    if (!__all_sync(kFull, alpha == 1.f)) {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        o[n][0] *= alpha;
        o[n][1] *= alpha;
      }
    }
    uint32_t a0 = E::pack(pr[0], pr[1]);
    uint32_t a2 = E::pack(pr[2], pr[3]);
    if (gid >= G) a0 = a2 = 0u;
    // O += P V: B fragments of V (k = tokens, n = 8 output columns) by ldmatrix.trans.
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4_trans(vtile + tile_off(((lane >> 3) & 1) * 8 + (lane & 7), 2 * np + (lane >> 4)), b0, b1, b2,
                        b3);
      mma_top(o[2 * np][0], o[2 * np][1], a0, a2, b0, b1);
      mma_top(o[2 * np + 1][0], o[2 * np + 1][1], a0, a2, b2, b3);
    }
  }

  __device__ __forceinline__ void finish() {
    l += __shfl_xor_sync(kFull, l, 1);
    l += __shfl_xor_sync(kFull, l, 2);
  }

  __device__ __forceinline__ void write_out(T* out_row, int lane) const {  // out_row -> [G][D]
    const int gid = lane >> 2, tq = lane & 3;
    if (gid >= G) return;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int n = 0; n < NT; ++n)
      *reinterpret_cast<uint32_t*>(out_row + gid * D + n * 8 + 2 * tq) = E::pack(o[n][0] * inv, o[n][1] * inv);
  }

  __device__ __forceinline__ void write_partial(float* po, float2* pml, int lane) const {
    const int gid = lane >> 2, tq = lane & 3;
    if (gid >= G) return;
#pragma unroll
    for (int n = 0; n < NT; ++n)
      *reinterpret_cast<float2*>(po + gid * D + n * 8 + 2 * tq) = make_float2(o[n][0], o[n][1]);
    if (tq == 0) pml[gid] = make_float2(m, l);
  }
};

// Zero V rows [valid, 16) of a chunk tile: the P V product multiplies them
// by an exact zero weight, and 0 * NaN would poison the output.
template <int D>
__device__ __forceinline__ void zero_tail_rows(uint32_t vtile, int valid, int lane) {
  const int n = (kChunk - valid) * (D / 8);
  for (int i = lane; i < n; i += 32) {
    const int r = valid + i / (D / 8);
    const int c16 = i % (D / 8);
    sts128(vtile + tile_off(r, c16), make_uint4(0u, 0u, 0u, 0u));
  }
  fence_proxy_async_smem();
  __syncwarp();
}

// --------------------------------------------------------------- prefix of chunk counts

template <int NT>
__device__ __forceinline__ void build_prefix(const DecodeParams& p, int* prefix) {
  __shared__ int warp_tot[NT / 32];
  const int S = p.num_seqs;
  const int t = threadIdx.x;
  const int per = (S + NT - 1) / NT;
  const int s0 = min(S, t * per), s1 = min(S, s0 + per);
  int local = 0;
  bool bad = false;
  for (int s = s0; s < s1; ++s) {
    const int ctx = p.context_lens[s];
    bad |= ctx < 0 || ctx > p.ctx_cap;
    local += (clamp_ctx(ctx, p.ctx_cap) + kChunk - 1) / kChunk;
  }
  if (bad && blockIdx.x == 0) set_err(p.err_flags, PA_ERRF_CONTEXT);
  const int lane = t & 31, warp = t >> 5;
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(kFull, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_tot[w];
  int run = base + incl - local;
  for (int s = s0; s < s1; ++s) {
    prefix[s] = run;
    run += (clamp_ctx(p.context_lens[s], p.ctx_cap) + kChunk - 1) / kChunk;
  }
  if (t == NT - 1) prefix[S] = base + incl;
}

// --------------------------------------------------------------- main kernel

template <typename T, int D, int G>
__global__ void __launch_bounds__(Shape<D, G>::kWarps * 32, 1)
    paged_decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                        const DecodeParams p) {
  using SH = Shape<D, G>;
  using Warp = typename std::conditional<SH::kMma, MmaWarp<T, D, G>, CoreWarp<T, D, G>>::type;
  constexpr int DEPTH = SH::kDepth;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  const uint32_t tiles = base;
  const uint32_t qslots = tiles + SH::kStages * SH::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SH::kStages * (SH::kStageBytes + SH::kQBytes));
  int* prefix = reinterpret_cast<int*>(bars + SH::kStages);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * SH::kWarps + warp;
  const int W = p.total_warps;

  // Work that reads no global memory overlaps the previous kernel's tail
  // (programmatic dependent launch); everything after griddep_wait sees all
  // of its writes.
  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  if (lane == 0) {
    for (int i = 0; i < DEPTH; ++i) mbar_init(&bars[warp * DEPTH + i], 1);
    fence_barrier_init();
  }
  griddep_wait();
  griddep_launch_dependents();
  build_prefix<SH::kWarps * 32>(p, prefix);
  __syncthreads();

  const int S = p.num_seqs, H = p.num_heads;
  const int64_t NC = (int64_t)p.num_kv_heads * prefix[S];
  RunSplit rs;
  rs.init(NC, W);
  const int64_t c0 = rs.begin(gw), c1 = rs.begin(gw + 1);
  const int n = static_cast<int>(c1 - c0);

  // The run's split parts.  Its first segment (containing the run's first
  // chunk) and its last segment (containing the last chunk) may each cover
  // only part of a unit; every other segment is a whole unit.
  UnitPos uf{0, 0, 0, 1}, ul{0, 0, 0, 1};
  int64_t af = 0, al = 0;  // global first chunks of those two units
  bool part_f = false, part_l = false;
  int mine_f = 0, mine_l = 0;  // chunks of those units in this run
  if (n > 0) {
    uf = unit_pos(p, prefix, c0);
    ul = unit_pos(p, prefix, c1 - 1);
    af = c0 - uf.c;
    al = c1 - 1 - ul.c;
    if (af == al) {  // the whole run lies in one unit
      part_f = !(uf.c == 0 && ul.c == ul.nc - 1);
      mine_f = n;
    } else {
      part_f = uf.c != 0;
      mine_f = uf.nc - uf.c;
      part_l = ul.c != ul.nc - 1;
      mine_l = ul.c + 1;
    }
  }
  // Processing order (CUDA-core path): the last segment first, when it is a
  // split part, then the run from its start, which begins with the first
  // segment.  Both split parts are thus done early and their merges (below)
  // overlap the other warps' streaming instead of lengthening the kernel's
  // tail.  Measured on one box: 1 us faster per LLaMA-7B call, but ~5 us
  // slower on the tensor-core (GQA) path, which keeps the plain order.
  // Virtual index k in [0, n) is physical chunk c0 + phys(k).
  const int shift = (!SH::kMma && part_l) ? n - mine_l : 0;
  auto phys = [&](int k) { return k + shift < n ? k + shift : k + shift - n; };
  auto gchunk = [&](int k) { return k < n ? c0 + phys(k) : c1; };  // c1: past the run

  // Chunk windows: `cur` holds chunks [kb, kb+32), `nxt` [kb+32, kb+64), and
  // the raw loads of [kb+64, kb+96) are in flight (processing order).
  const ChunkRaw r0 = chunk_load(p, prefix, gchunk(lane), c1);
  const ChunkRaw r1 = chunk_load(p, prefix, gchunk(32 + lane), c1);
  ChunkRaw rnext = chunk_load(p, prefix, gchunk(64 + lane), c1);
  ChunkInfo cur = chunk_finalize(p, r0);
  ChunkInfo nxt = chunk_finalize(p, r1);
  int kb = 0;

  // Sequences with an empty context produce zeros.
  for (int s = gw; s < S; s += W) {
    if (clamp_ctx(p.context_lens[s], p.ctx_cap) == 0) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<T*>(p.out) + (int64_t)s * H * D);
      for (int i = lane; i < H * D / 8; i += 32) dst[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }

  const uint64_t policy_stream = l2_evict_first_policy();
  const uint64_t policy_head = l2_evict_normal_policy();
  const int rows_per_block = p.block_size < kChunk ? p.block_size : kChunk;
  const uint32_t box_bytes = rows_per_block * 128;
  const T* qbase = static_cast<const T*>(p.q);
  // A segment starts at the first chunk processed, at a unit's first chunk,
  // and where the processing order wraps to the run's first chunk.
  auto seg_starts = [&](int k, int flags) { return k == 0 || (flags & kFlagStart) || phys(k) == 0; };
  auto seg_ends = [&](int k, int flags) { return k == n - 1 || (flags & kFlagEnd) || phys(k) == n - 1; };

  // Issue the loads of chunk k into its stage (lane 0; all lanes shuffle).
  auto issue = [&](int k) {
    const int d = k - kb;
    const bool in_cur = d < 32;
    const int src = d & 31;
    const int flags = __shfl_sync(kFull, in_cur ? cur.flags : nxt.flags, src);
    const int sh = __shfl_sync(kFull, in_cur ? cur.sh : nxt.sh, src);
    const int p0 = __shfl_sync(kFull, in_cur ? cur.p0 : nxt.p0, src);
    const int p1 = __shfl_sync(kFull, in_cur ? cur.p1 : nxt.p1, src);
    if (lane != 0) return;
    const int stage = warp * DEPTH + (k % DEPTH);
    uint64_t* bar = &bars[stage];
    const bool seg_start = seg_starts(k, flags);
    const int valid = flags & 31;
    const int row0 = (flags >> 5) & 63;
    const int head = sh >> 16, seq = sh & 0xffff;
    const int nblk = valid > 0 ? (p1 >= 0 ? 2 : 1) : 0;
    const uint64_t policy = (flags & kFlagHead) ? policy_head : policy_stream;
    const uint32_t bytes = nblk * (D / 64) * box_bytes * 2 + (seg_start ? SH::kQBytes : 0);
    mbar_arrive_expect_tx(bar, bytes);
    const uint32_t kt = tiles + stage * SH::kStageBytes;
    const uint32_t vt = kt + SH::kTileBytes;
    for (int b = 0; b < nblk; ++b) {
      const int phys_blk = b == 0 ? p0 : p1;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const uint32_t off = c * 2048 + b * 1024;
        tma_load_4d(kt + off, &kmap, bar, 64 * c, row0, head, phys_blk, policy);
        tma_load_4d(vt + off, &vmap, bar, 64 * c, row0, head, phys_blk, policy);
      }
    }
    if (seg_start) {
      const T* q_src = qbase + ((int64_t)seq * H + (int64_t)head * G) * D;
      bulk_load(qslots + stage * SH::kQBytes, q_src, SH::kQBytes, bar);
    }
  };

  // Split units: for each split part the warp adds its chunk count to the
  // unit's ticket counter, right after writing the part's partial; the warp
  // whose addition completes the unit's count merges every part and writes
  // the output, so no warp ever waits for another.
  bool ticket_f = false, ticket_l = false;
  auto take_ticket = [&](bool first) {
    const int64_t a = first ? af : al;
    const UnitPos& u = first ? uf : ul;
    const int mine = first ? mine_f : mine_l;
    // Ordering without fences: the warp barrier orders every lane's partial
    // stores before lane 0's ticket, whose release semantics publish them at
    // GPU scope; the acquire half makes the other parts' partials (published
    // the same way before their tickets) visible to lane 0, and the second
    // barrier extends that to the lanes that read them.  (A __threadfence()
    // on either side stalled each warp on its own loads in flight: ~3.5 us
    // per launch on the LLaMA-7B workload.)
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      int* t = p.ws_tickets + rs.warp_of(a);
      int before;
      asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(before) : "l"(t), "r"(mine) : "memory");
      last = before + mine == u.nc;
      if (last) *t = 0;  // all parts counted; nobody else touches it in this launch
    }
    last = __shfl_sync(kFull, last, 0);
    __syncwarp();
    if (last) {
      merge_split_unit<T, D, G>(p.ws_ml, p.ws_o,
                                static_cast<T*>(p.out) + ((int64_t)u.seq * H + (int64_t)u.head * G) * D, a,
                                u.nc, rs, lane);
    }
    (first ? ticket_f : ticket_l) = true;
  };

  for (int i = 0; i < DEPTH && i < n; ++i) issue(i);

  Warp st;
  st.reset();
  bool seg_from_unit_start = false;
  bool seg_has_run_start = false;  // the segment holds the run's first chunk: partial slot 0, else 1
  bool timed_out = false;
  int k = 0;
  for (; k < n; ++k) {
    if (k - kb >= 32) {
      cur = nxt;
      nxt = chunk_finalize(p, rnext);
      kb += 32;
      rnext = chunk_load(p, prefix, gchunk(kb + 64 + lane), c1);
    }
    const int d = k - kb;
    const int flags = __shfl_sync(kFull, cur.flags, d);
    const int sh = __shfl_sync(kFull, cur.sh, d);
    const int stage = warp * DEPTH + (k % DEPTH);
    const uint32_t parity = (k / DEPTH) & 1;
    // Every lane waits (acquiring the TMA writes); the give-up decision is
    // made warp-wide so that the lanes never diverge around the shuffles.
    const bool arrived = mbar_wait_bounded(&bars[stage], parity, kWaitLimitNs);
    if (!__all_sync(kFull, arrived)) {
      timed_out = true;
      break;
    }
    const bool seg_start = seg_starts(k, flags);
    const bool seg_end = seg_ends(k, flags);
    if (seg_start) {
      st.reset();
      st.load_q(qslots + stage * SH::kQBytes, p.scale_log2, lane);
      seg_from_unit_start = (flags & kFlagStart) != 0;
      seg_has_run_start = phys(k) == 0;
    }
    const int valid = flags & 31;
    const uint32_t kt = tiles + stage * SH::kStageBytes;
    const uint32_t vt = kt + SH::kTileBytes;
    if (valid == kChunk) {
      if constexpr (SH::kMma) st.template chunk<false>(kt, vt, kChunk, lane, p.scale_log2);
      else st.template chunk<false>(kt, vt, kChunk, lane);
    } else if (valid > 0) {
      if constexpr (SH::kMma) {
        zero_tail_rows<D>(vt, valid, lane);
        st.template chunk<true>(kt, vt, valid, lane, p.scale_log2);
      } else {
        st.template chunk<true>(kt, vt, valid, lane);
      }
    }
    __syncwarp();
    if (k + DEPTH < n) issue(k + DEPTH);
    if (seg_end) {
      st.finish();
      const int seq = sh & 0xffff, kvh = sh >> 16;
      const bool unit_end = (flags & kFlagEnd) != 0;
      if (seg_from_unit_start && unit_end) {
        st.write_out(static_cast<T*>(p.out) + ((int64_t)seq * H + (int64_t)kvh * G) * D, lane);
      } else {
        const int slot = 2 * gw + (seg_has_run_start ? 0 : 1);
        st.write_partial(p.ws_o + (int64_t)slot * G * D, p.ws_ml + (int64_t)slot * G, lane);
        take_ticket(seg_has_run_start);
      }
    }
  }
  if (timed_out) {
    set_err(p.err_flags, PA_ERRF_TIMEOUT);
    // Let this warp's copies in flight land before the CTA can exit.
    for (int kk = k; kk < n && kk < k + DEPTH; ++kk)
      mbar_wait_bounded(&bars[warp * DEPTH + (kk % DEPTH)], (kk / DEPTH) & 1, kWaitLimitNs);
    // The split parts not reached still count their chunks, so the counters
    // return to zero (their outputs are flagged as not written).
    if (part_f && !ticket_f) take_ticket(true);
    if (part_l && !ticket_l) take_ticket(false);
  }
}

}  // namespace pa
