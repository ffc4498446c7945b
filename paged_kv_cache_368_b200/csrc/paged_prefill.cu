// Multi-token paged attention: a chunk of new tokens per sequence (a prompt,
// a chunked prefill, or several speculative tokens) attends causally over the
// paged KV cache.
//
// What is computed: the ops-transformer page's PagedAttention call takes a
// query of [batch, heads, seq_len, head_dim] against the paged cache; each
// query row is the decode formula of "【infra之路】10-PagedAttention 与 KV Cache
// 管理" (section 1.1) restricted to the positions up to its own.  Sequence s
// owns query rows cu_q[s] .. cu_q[s+1]-1; its n new tokens are the last n of
// its context_lens[s] cached positions (appended before this call), so row i
// sits at position ctx - n + i and attends to positions 0..ctx-n+i.
//
// Design: one CTA per (64-row query tile, q-head, sequence), tiles of a
// sequence launched longest-first.  Four consumer warps own 16 query rows
// each; a fifth warp streams the K/V rows of 16-token key chunks with TMA
// (128-byte swizzle, block-table lookups prefetched 32 chunks at a time) into
// a CTA-shared ring with full/empty mbarriers.  Per chunk, S = Q K^T and
// O += P V run on the tensor cores (mma.sync m16n8k16, query rows on M, the
// FlashAttention-2 register reuse of S as P), with an online softmax and the
// causal mask applied only on diagonal chunks.
#include <algorithm>
#include <atomic>
#include <cmath>

#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {
namespace pf {

constexpr int kRows = 16;               // query rows per consumer warp (mma M)
constexpr int kConsumers = 4;           // consumer warps per CTA
constexpr int kTileQ = kRows * kConsumers;
constexpr int kChunk = 16;              // keys per stage
constexpr int kDepth = 4;               // stages in the ring
constexpr uint64_t kWaitLimitNs = 1000000000ull;

struct Params {
  void* out;
  const void* q;
  const int32_t* cu_q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  int32_t* err_flags;
  int64_t num_blocks;
  int num_seqs;
  int max_blocks_per_seq;
  int ctx_cap;
  int num_heads;
  int num_kv_heads;
  int block_size;
  int q_tiles;
  int total_q;
  float scale_log2;
};

template <int D>
struct Layout {
  static constexpr int kTileBytes = kChunk * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr size_t kSmem = 1024 + size_t(kDepth) * kStageBytes + 2 * kDepth * 8 + kDepth * 4;
};

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// 4-D tiled TMA load without an L2 policy: prefill re-reads a sequence's
// K/V from every query tile and q-head of its group, so they should stay in L2.
__device__ __forceinline__ void tma_load_4d_keep(uint32_t dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                                 int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_addr(bar))
      : "memory");
}

// D[0..3] += A(16x16) * B(16x8), all four accumulator rows live.
template <typename T>
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  Elem<T>::mma(d, a[0], a[1], a[2], a[3], b0, b1);
}

template <typename T, int D>
__global__ void __launch_bounds__((kConsumers + 1) * 32, 2)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                         const Params p) {
  using E = Elem<T>;
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kDepth * L::kStageBytes);
  uint64_t* empty = full + kDepth;
  int* stage_ok = reinterpret_cast<int*>(empty + kDepth);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = p.q_tiles - 1 - static_cast<int>(blockIdx.x);  // longest rows first
  const int h = blockIdx.y, s = blockIdx.z;
  const int G = p.num_heads / p.num_kv_heads;
  const int kvh = h / G;

  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
    for (int i = 0; i < kDepth; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumers);
    }
    fence_barrier_init();
  }
  griddep_wait();
  griddep_launch_dependents();
  __syncthreads();

  // Geometry of this sequence and tile.
  const int qa = __ldg(p.cu_q + s), qb = __ldg(p.cu_q + s + 1);
  const int ctx_raw = __ldg(p.context_lens + s);
  const int ctx = ctx_raw < 0 ? 0 : (ctx_raw > p.ctx_cap ? p.ctx_cap : ctx_raw);
  int n = qb - qa;
  if (qa < 0 || qb > p.total_q) n = 0;  // malformed offsets: touch no row of q or out
  if (ctx != ctx_raw || n != qb - qa || n > ctx) {
    if (threadIdx.x == 0 && tile == 0 && h == 0) set_err(p.err_flags, PA_ERRF_CONTEXT);
    n = n < 0 ? 0 : (n > ctx ? ctx : n);
  }
  const int r0 = tile * kTileQ;
  if (r0 >= n) return;  // uniform over the CTA
  const int rows = min(kTileQ, n - r0);
  const int pos0 = ctx - n + r0;  // position of the tile's first row
  const int kend = pos0 + rows;   // keys 0..kend-1 are visible to some row
  const int nchunks = (kend + kChunk - 1) / kChunk;

  if (warp == kConsumers) {
    // ---------------------------------------------------------------- producer
    const int bs = p.block_size;
    const int32_t* row = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
    const uint32_t box_bytes = (bs < kChunk ? bs : kChunk) * 128;
    bool abort = false;
    for (int c_base = 0; c_base < nchunks && !abort; c_base += 32) {
      const int c = c_base + lane;
      int b0 = -1, b1 = -1, row0 = 0;
      if (c < nchunks) {
        const int t0 = c * kChunk;
        if (bs >= kChunk) {
          b0 = __ldg(row + t0 / bs);
          row0 = t0 % bs;
        } else {
          b0 = __ldg(row + 2 * c);
          if (t0 + 8 < kend) b1 = __ldg(row + 2 * c + 1);
        }
        const bool ok = b0 >= 0 && b0 < p.num_blocks && (b1 == -1 || (b1 >= 0 && b1 < p.num_blocks));
        if (!ok) {
          set_err(p.err_flags, PA_ERRF_BLOCK_RANGE);
          b0 = -1;
          b1 = -1;
        }
      }
      for (int j = 0; j < 32 && c_base + j < nchunks; ++j) {
        const int cc = c_base + j;
        const int pb0 = __shfl_sync(kFull, b0, j), pb1 = __shfl_sync(kFull, b1, j);
        const int prow0 = __shfl_sync(kFull, row0, j);
        int bad = 0;
        if (lane == 0) {
          const int st = cc % kDepth;
          if (cc >= kDepth && !mbar_wait_bounded(&empty[st], ((cc / kDepth) - 1) & 1, kWaitLimitNs)) {
            set_err(p.err_flags, PA_ERRF_TIMEOUT);
            bad = 1;
          } else {
            const int nb = pb0 < 0 ? 0 : (pb1 >= 0 ? 2 : 1);
            stage_ok[st] = nb > 0;
            mbar_arrive_expect_tx(&full[st], nb * (D / 64) * box_bytes * 2);
            const uint32_t kt = base + st * L::kStageBytes;
            const uint32_t vt = kt + L::kTileBytes;
            for (int b = 0; b < nb; ++b) {
              const int phys = b == 0 ? pb0 : pb1;
#pragma unroll
              for (int cq = 0; cq < D / 64; ++cq) {
                const uint32_t off = cq * 2048 + b * 1024;
                tma_load_4d_keep(kt + off, &kmap, &full[st], 64 * cq, prow0, kvh, phys);
                tma_load_4d_keep(vt + off, &vmap, &full[st], 64 * cq, prow0, kvh, phys);
              }
            }
          }
        }
        if (__shfl_sync(kFull, bad, 0)) {
          abort = true;
          break;
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int gid = lane >> 2, tq = lane & 3;
  const int wr0 = warp * kRows;  // first row of this warp within the tile
  const int wrows = rows - wr0;  // rows of this warp (may be <= 0)
  const int wpos0 = pos0 + wr0;
  const int wlast = wpos0 + min(kRows, wrows) - 1;
  const T* qbase = static_cast<const T*>(p.q);
  const int H = p.num_heads;

  constexpr int KS = D / 16, NT = D / 8;
  uint32_t qa_frag[KS][4];
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int rr = gid + 8 * r;
      uint32_t lo = 0u, hi = 0u;
      if (rr < wrows) {
        const T* src = qbase + ((int64_t)(qa + r0 + wr0 + rr) * H + h) * D + ks * 16 + 2 * tq;
        lo = *reinterpret_cast<const uint32_t*>(src);
        hi = *reinterpret_cast<const uint32_t*>(src + 8);
      }
      qa_frag[ks][r] = lo;      // a0 (row gid) / a1 (row gid+8): k = 2tq, 2tq+1
      qa_frag[ks][2 + r] = hi;  // a2 / a3: k = 2tq+8, 2tq+9
    }
  }

  float o[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};

  bool failed = false;
  for (int c = 0; c < nchunks; ++c) {
    const int st = c % kDepth;
    const bool arrived = mbar_wait_bounded(&full[st], (c / kDepth) & 1, kWaitLimitNs);
    if (!__all_sync(kFull, arrived)) {
      set_err(p.err_flags, PA_ERRF_TIMEOUT);
      failed = true;
      if (warp == 0) {  // let copies still in flight land before the CTA exits
        for (int cc = c + 1; cc < nchunks && cc < c + kDepth; ++cc)
          mbar_wait_bounded(&full[cc % kDepth], (cc / kDepth) & 1, kWaitLimitNs);
      }
      break;
    }
    const int key0 = c * kChunk;
    if (wrows > 0 && key0 <= wlast && stage_ok[st]) {
      const uint32_t kt = base + st * L::kStageBytes;
      const uint32_t vt = kt + L::kTileBytes;
      // S = Q K^T for keys key0..key0+15 (two 8-key n-tiles)
      float sacc[2][4] = {};
#pragma unroll
      for (int kp = 0; kp < D / 32; ++kp) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          uint32_t b0, b1, b2, b3;
          ldmatrix_x4(kt + tile_off(nt * 8 + (lane & 7), kp * 4 + (lane >> 3)), b0, b1, b2, b3);
          mma16816<T>(sacc[nt], qa_frag[2 * kp], b0, b1);
          mma16816<T>(sacc[nt], qa_frag[2 * kp + 1], b2, b3);
        }
      }
      // scores in log2 units; causal mask (and keys past the context) only
      // where the chunk reaches past the first row's position
      float sc[2][4];
      const bool diag = key0 + kChunk - 1 > wpos0;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float v = sacc[nt][e] * p.scale_log2;
          if (diag) {
            const int kpos = key0 + nt * 8 + 2 * tq + (e & 1);
            const int rpos = wpos0 + gid + 8 * (e >> 1);
            if (kpos > rpos) v = -INFINITY;
          }
          sc[nt][e] = v;
        }
      float alpha[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        float cm = fmaxf(fmaxf(sc[0][2 * r], sc[0][2 * r + 1]), fmaxf(sc[1][2 * r], sc[1][2 * r + 1]));
        cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 1));
        cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 2));
        const float mn = fmaxf(m[r], cm);
        // a row whose every key so far is masked keeps m = -inf and weight 0
        const float mref = mn == -INFINITY ? 0.f : mn;
        alpha[r] = fast_exp2(m[r] - mref);
        float rs = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float pv = fast_exp2(sc[nt][2 * r + e] - mref);
            sc[nt][2 * r + e] = pv;
            rs += pv;
          }
        l[r] = l[r] * alpha[r] + rs;
        m[r] = mn;
      }
      if (!__all_sync(kFull, alpha[0] == 1.f && alpha[1] == 1.f)) {
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          o[j][0] *= alpha[0];
          o[j][1] *= alpha[0];
          o[j][2] *= alpha[1];
          o[j][3] *= alpha[1];
        }
      }
      uint32_t pa_frag[4];
      pa_frag[0] = E::pack(sc[0][0], sc[0][1]);  // row gid,   keys 2tq..
      pa_frag[1] = E::pack(sc[0][2], sc[0][3]);  // row gid+8, keys 2tq..
      pa_frag[2] = E::pack(sc[1][0], sc[1][1]);  // row gid,   keys 8+2tq..
      pa_frag[3] = E::pack(sc[1][2], sc[1][3]);  // row gid+8, keys 8+2tq..
      // V rows at keys >= kend carry zero weight for every row of the tile and
      // may hold no data (unwritten slots, possibly NaN, or a second block of
      // 8 that was not loaded): zero them in the fragments so 0 * V stays 0.
      const int vlim = kend - key0;  // V rows of this chunk that may carry weight
      const bool vmask = vlim < kChunk;
#pragma unroll
      for (int np = 0; np < NT / 2; ++np) {
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4_trans(vt + tile_off(((lane >> 3) & 1) * 8 + (lane & 7), 2 * np + (lane >> 4)), b0, b1, b2, b3);
        if (vmask) {
          const int t = 2 * tq;
          const uint32_t m_lo = (t < vlim ? 0x0000ffffu : 0u) | (t + 1 < vlim ? 0xffff0000u : 0u);
          const uint32_t m_hi = (t + 8 < vlim ? 0x0000ffffu : 0u) | (t + 9 < vlim ? 0xffff0000u : 0u);
          b0 &= m_lo;
          b2 &= m_lo;
          b1 &= m_hi;
          b3 &= m_hi;
        }
        mma16816<T>(o[2 * np], pa_frag, b0, b1);
        mma16816<T>(o[2 * np + 1], pa_frag, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
  }
  if (failed || wrows <= 0) return;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(kFull, l[r], 1);
    l[r] += __shfl_xor_sync(kFull, l[r], 2);
  }
  T* obase = static_cast<T*>(p.out);
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int rr = gid + 8 * r;
    if (rr >= wrows) continue;
    const float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
    T* dst = obase + ((int64_t)(qa + r0 + wr0 + rr) * H + h) * D + 2 * tq;
#pragma unroll
    for (int j = 0; j < NT; ++j)
      *reinterpret_cast<uint32_t*>(dst + j * 8) = E::pack(o[j][2 * r] * inv, o[j][2 * r + 1] * inv);
  }
}

}  // namespace pf
}  // namespace pa

namespace {

inline bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

template <typename T, int D>
pa_status launch_prefill(const CUtensorMap& km, const CUtensorMap& vm, const pa::pf::Params& p, int dev,
                         cudaStream_t stream) {
  auto kern = pa::pf::paged_prefill_kernel<T, D>;
  const size_t smem = pa::pf::Layout<D>::kSmem;
  static std::atomic<int> smem_set[pa::kMaxDevices];
  if (dev >= 0 && dev < pa::kMaxDevices && !smem_set[dev].load(std::memory_order_relaxed)) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "cudaFuncSetAttribute(prefill)", e);
    smem_set[dev].store(1, std::memory_order_relaxed);
  }
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.q_tiles, p.num_heads, p.num_seqs);
  cfg.blockDim = dim3((pa::pf::kConsumers + 1) * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, km, vm, p);
  return e == cudaSuccess ? PA_OK : pa::fail(PA_ERR_CUDA, "launching paged_prefill_kernel", e);
}

}  // namespace

extern "C" pa_status pa_prefill_mma(void* out, const void* q, const int32_t* cu_q_lens, int total_q, int max_q_len,
                                const void* k_cache, const void* v_cache, const int32_t* block_tables,
                                int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                                int max_context_len, float scale, int num_heads, int num_kv_heads, int head_dim,
                                int block_size, int64_t num_blocks, pa_dtype dtype, int32_t* err_flags,
                                pa_stream_t stream) {
  if (num_seqs < 0 || total_q < 0 || max_q_len < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
      num_heads % num_kv_heads)
    return PA_ERR_INVALID;
  if (max_blocks_per_seq <= 0 || max_context_len < 0 || num_blocks <= 0) return PA_ERR_INVALID;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID;
  if (!std::isfinite(scale)) return PA_ERR_INVALID;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != 8 && block_size != 16 && block_size != 32 && block_size != 64) return PA_ERR_UNSUPPORTED;
  if (num_seqs > 65535 || num_heads > 65535) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || total_q == 0 || max_q_len == 0) return PA_OK;
  if (!out || !q || !cu_q_lens || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_INVALID;
  if (!aligned_to(out, 16) || !aligned_to(q, 16) || !aligned_to(k_cache, 16) || !aligned_to(v_cache, 16) ||
      !aligned_to(cu_q_lens, 4) || !aligned_to(block_tables, 4) || !aligned_to(context_lens, 4))
    return PA_ERR_INVALID;
  if (num_blocks > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return pa::fail(PA_ERR_CUDA, "cudaGetDevice", ce);
  if (!pa::have_tensor_map_encoder())
    return pa::fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found", cudaSuccess);
  CUtensorMap km, vm;
  if (!pa::make_cache_map(&km, k_cache, num_blocks, num_kv_heads, block_size, head_dim) ||
      !pa::make_cache_map(&vm, v_cache, num_blocks, num_kv_heads, block_size, head_dim))
    return pa::fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled rejected the cache layout", cudaSuccess);
  pa::pf::Params p;
  p.out = out;
  p.q = q;
  p.cu_q = cu_q_lens;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.err_flags = err_flags;
  p.num_blocks = num_blocks;
  p.num_seqs = num_seqs;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.ctx_cap = static_cast<int>(std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * block_size));
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.block_size = block_size;
  p.total_q = total_q;
  p.q_tiles = (max_q_len + pa::pf::kTileQ - 1) / pa::pf::kTileQ;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == PA_F16)
    return head_dim == 128 ? launch_prefill<__half, 128>(km, vm, p, dev, s) : launch_prefill<__half, 64>(km, vm, p, dev, s);
  return head_dim == 128 ? launch_prefill<__nv_bfloat16, 128>(km, vm, p, dev, s)
                         : launch_prefill<__nv_bfloat16, 64>(km, vm, p, dev, s);
}
