// Multi-token paged attention on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory).  Same contract as the mma.sync kernel in
// paged_prefill.cu: the last n cached tokens of each sequence attend causally
// over its paged K/V (the ops-transformer page's [batch, heads, seq_len,
// head_dim] call; each row the section 1.1 formula of "【infra之路】10-
// PagedAttention 与 KV Cache 管理", restricted to positions up to its own).
//
// One CTA per (128-row query tile, q-head, sequence), 8 warps:
//   warp 0      TMA producer: the Q tile once (3-D map over [token][head][d]),
//               then K and V of 64-key tiles, 16 rows per box read through
//               the block table, into a 3-stage ring;
//   warp 1      allocates tensor memory and issues the MMAs (one thread):
//               S_j = Q K_j^T (M 128, N 64) into one of two TMEM buffers, and
//               O += P_j V_j (M 128, N head_dim) into a TMEM accumulator;
//               S_{j+1} is issued before waiting for P_j, so it overlaps the
//               softmax of tile j;
//   warps 4-7   softmax: thread t owns query row t (TMEM lane t).  It reads
//               S_j, applies the causal mask, keeps a running max that is
//               only moved when it grows by more than 2^8 (so the O rescale in
//               tensor memory is rare), writes P_j (bf16/fp16) into a swizzled
//               shared tile, and at the end reads O and divides by the sum.
// All operand tiles are 128-byte-swizzled, the layout TMA writes and the MMA
// descriptors name directly.
#include <algorithm>
#include <atomic>
#include <cmath>

#include "pa_host.h"
#include "tcgen05.cuh"

namespace pa {
namespace ptc {

constexpr int BM = 128;     // query rows per CTA (MMA M)
constexpr int BN = 64;      // keys per tile
constexpr int STAGES = 3;   // K/V ring
constexpr int kThreads = 256;
constexpr uint64_t kWaitNs = 1000000000ull;
constexpr uint32_t kTmemCols = 256;  // S0 [0,64), S1 [64,128), O [128, 128+D)

struct Params {
  void* out;
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
struct Lay {
  static constexpr int kQ = BM * D * 2;    // [D/64][BM rows][128 B]
  static constexpr int kKV = BN * D * 2;   // [D/64][BN rows][128 B]
  static constexpr int kP = BM * BN * 2;   // [BM rows][128 B]
  static constexpr int kOffK = kQ;
  static constexpr int kOffV = kOffK + STAGES * kKV;
  static constexpr int kOffP = kOffV + STAGES * kKV;
  static constexpr int kOffBar = kOffP + kP;
  // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], s_free[2], p_full, pv_done, mma_done
  static constexpr int kBars = 1 + 2 * STAGES + 2 + 2 + 3;
  static constexpr size_t kSmem = 1024 + kOffBar + kBars * 8 + 16;
};

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                            const __grid_constant__ CUtensorMap qmap, const Params p) {
  using E = Elem<T>;
  using L = Lay<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + STAGES;
  uint64_t* s_full = kv_empty + STAGES;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* mma_done = pv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = p.q_tiles - 1 - static_cast<int>(blockIdx.x);  // longest rows first
  const int h = blockIdx.y, s = blockIdx.z;
  const int kvh = h / (p.num_heads / p.num_kv_heads);

  if (threadIdx.x == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
    prefetch_tensormap(&qmap);
    mbar_init(q_full, 1);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) tc5::tmem_alloc(tmem_slot, kTmemCols);
  griddep_wait();
  griddep_launch_dependents();
  tc5::fence_before();
  __syncthreads();
  tc5::fence_after();
  const uint32_t tmem = *tmem_slot;

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
  const int r0 = tile * BM;
  const bool active = r0 < n;
  const int rows = active ? min(BM, n - r0) : 0;
  const int pos0 = ctx - n + r0;
  const int kend = pos0 + rows;
  const int ntiles = active ? (kend + BN - 1) / BN : 0;
  const uint32_t q_s = base, k_s = base + L::kOffK, v_s = base + L::kOffV, p_s = base + L::kOffP;

  if (active && warp == 0) {
    // ------------------------------------------------------------- producer
    const int bs = p.block_size;
    const int32_t* row = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
    const uint32_t box_bytes = (bs < 16 ? bs : 16) * 128;
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, L::kQ);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tc5::tma_load_3d(q_s + c * (BM * 128), &qmap, q_full, 64 * c, h, qa + r0);
    }
    const int nchunks = ntiles * (BN / 16);
    bool abort = false;
    for (int c_base = 0; c_base < nchunks && !abort; c_base += 32) {
      // table entries of the next 32 16-key chunks, one per lane
      const int c = c_base + lane;
      int b0 = -1, b1 = -1, row0 = 0;
      if (c < nchunks && c * 16 < kend) {
        const int t0 = c * 16;
        if (bs >= 16) {
          b0 = __ldg(row + t0 / bs);
          row0 = t0 % bs;
        } else {
          b0 = __ldg(row + 2 * c);
          if (t0 + 8 < kend) b1 = __ldg(row + 2 * c + 1);
        }
        if (!(b0 >= 0 && b0 < p.num_blocks && (b1 == -1 || (b1 >= 0 && b1 < p.num_blocks)))) {
          set_err(p.err_flags, PA_ERRF_BLOCK_RANGE);
          b0 = b1 = -1;
        }
      }
      // one 64-key tile = 4 chunks
      for (int jt = 0; jt < 32 / (BN / 16) && c_base + jt * (BN / 16) < nchunks; ++jt) {
        const int j = c_base / (BN / 16) + jt;
        int bb0[BN / 16], bb1[BN / 16], rr0[BN / 16];
#pragma unroll
        for (int q = 0; q < BN / 16; ++q) {
          bb0[q] = __shfl_sync(kFull, b0, jt * (BN / 16) + q);
          bb1[q] = __shfl_sync(kFull, b1, jt * (BN / 16) + q);
          rr0[q] = __shfl_sync(kFull, row0, jt * (BN / 16) + q);
        }
        int bad = 0;
        if (lane == 0) {
          const int st = j % STAGES;
          if (j >= STAGES && !mbar_wait_bounded(&kv_empty[st], ((j / STAGES) - 1) & 1, kWaitNs)) {
            set_err(p.err_flags, PA_ERRF_TIMEOUT);
            bad = 1;
          } else {
            uint32_t bytes = 0;
#pragma unroll
            for (int q = 0; q < BN / 16; ++q)
              bytes += (bb0[q] < 0 ? 0 : (bb1[q] >= 0 ? 2 : 1)) * (D / 64) * box_bytes * 2;
            mbar_arrive_expect_tx(&kv_full[st], bytes);
            const uint32_t kt = k_s + st * L::kKV, vt = v_s + st * L::kKV;
#pragma unroll
            for (int q = 0; q < BN / 16; ++q) {
              const int nb = bb0[q] < 0 ? 0 : (bb1[q] >= 0 ? 2 : 1);
              for (int b = 0; b < nb; ++b) {
                const int phys = b == 0 ? bb0[q] : bb1[q];
#pragma unroll
                for (int cq = 0; cq < D / 64; ++cq) {
                  const uint32_t off = cq * (BN * 128) + q * 2048 + b * 1024;
                  tc5::tma_load_4d(kt + off, &kmap, &kv_full[st], 64 * cq, rr0[q], kvh, phys);
                  tc5::tma_load_4d(vt + off, &vmap, &kv_full[st], 64 * cq, rr0[q], kvh, phys);
                }
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
    // The last tiles' copies have landed (always, on the normal path) before
    // the CTA may exit.
    if (lane == 0) {
      for (int j = max(0, ntiles - STAGES); j < ntiles; ++j)
        mbar_wait_bounded(&kv_full[j % STAGES], (j / STAGES) & 1, kWaitNs);
    }
  } else if (active && warp == 1) {
    // ------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr int fmt = Elem<T>::kind == PA_BF16 ? 1 : 0;
      constexpr uint32_t id_qk = tc5::f16_idesc(fmt, BM, BN, 0, 0);
      constexpr uint32_t id_pv = tc5::f16_idesc(fmt, BM, D, 0, 1);
      bool ok = mbar_wait_bounded(q_full, 0, kWaitNs);
      auto issue_qk = [&](int j) -> bool {
        const int st = j % STAGES, sb = j & 1;
        if (!mbar_wait_bounded(&kv_full[st], (j / STAGES) & 1, kWaitNs)) return false;
        if (j >= 2 && !mbar_wait_bounded(&s_free[sb], ((j >> 1) - 1) & 1, kWaitNs)) return false;
        tc5::fence_after();
        const uint32_t kt = k_s + st * L::kKV;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t da = tc5::sw128_desc(q_s + (ks >> 2) * (BM * 128) + (ks & 3) * 32, 16, 1024);
          const uint64_t db = tc5::sw128_desc(kt + (ks >> 2) * (BN * 128) + (ks & 3) * 32, 16, 1024);
          tc5::mma_ss(tmem + sb * BN, da, db, id_qk, ks > 0);
        }
        tc5::commit(&s_full[sb]);
        return true;
      };
      if (ok) {
        tc5::fence_after();
        ok = issue_qk(0);
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        if (j + 1 < ntiles && !issue_qk(j + 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait_bounded(p_full, j & 1, kWaitNs)) {
          ok = false;
          break;
        }
        tc5::fence_after();
        const uint32_t vt = v_s + (j % STAGES) * L::kKV;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          const uint64_t da = tc5::sw128_desc(p_s + ks * 32, 16, 1024);
          const uint64_t db = tc5::sw128_desc(vt + ks * (16 * 128), BN * 128, 1024);
          tc5::mma_ss(tmem + 2 * BN, da, db, id_pv, (j > 0 || ks > 0) ? 1u : 0u);
        }
        tc5::commit(pv_done);
        tc5::commit(&kv_empty[j % STAGES]);
      }
      if (!ok) set_err(p.err_flags, PA_ERRF_TIMEOUT);
      tc5::commit(mma_done);  // lets the CTA free tensor memory once every MMA has finished
    }
  } else if (active && warp >= 4) {
    // ------------------------------------------------------------- softmax
    const int w = warp - 4;
    const int r = w * 32 + lane;  // query row of this thread (TMEM lane)
    const uint32_t lane_off = uint32_t(w * 32) << 16;
    const int rp = pos0 + r;      // its position
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1;
      const bool got = mbar_wait_bounded(&s_full[sb], (j >> 1) & 1, kWaitNs);
      if (!__all_sync(kFull, got)) {
        ok = false;
        break;
      }
      tc5::fence_after();
      uint32_t sr0[32], sr1[32];
      tc5::ld32(tmem + lane_off + sb * BN, sr0);
      tc5::ld32(tmem + lane_off + sb * BN + 32, sr1);
      tc5::wait_ld();
      tc5::fence_before();
      __syncwarp();
      if (lane == 0) tc5::arrive(&s_free[sb]);

      const int key0 = j * BN;
      const bool diag = key0 + BN - 1 > pos0;
      float sv[BN];
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < BN; ++i) {
        float v = __uint_as_float(i < 32 ? sr0[i] : sr1[i - 32]) * p.scale_log2;
        if (diag && (key0 + i > rp || key0 + i >= kend)) v = -INFINITY;
        sv[i] = v;
        mt = fmaxf(mt, v);
      }
      const float m_new = fmaxf(m_ref, mt);
      const bool resc = m_new > m_ref + 8.f;  // also true the first time (m_ref = -inf)
      if (j > 0) {
        const bool done = mbar_wait_bounded(pv_done, (j - 1) & 1, kWaitNs);
        if (!__all_sync(kFull, done)) {
          ok = false;
          break;
        }
        tc5::fence_after();
        if (__any_sync(kFull, resc)) {  // rescale O rows whose reference max moves
          const float alpha = resc ? fast_exp2(m_ref - m_new) : 1.f;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tc5::ld32(tmem + lane_off + 2 * BN + cc * 32, o);
            tc5::wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tc5::st32(tmem + lane_off + 2 * BN + cc * 32, o);
          }
          tc5::wait_st();
        }
      }
      if (resc) {
        l *= (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - m_new);
        m_ref = m_new;
      }
      const float mref = m_ref == -INFINITY ? 0.f : m_ref;
      // P row: keys 8c..8c+7 go to 16-byte chunk c, stored at chunk c ^ (r % 8)
      const uint32_t prow = p_s + r * 128;
#pragma unroll
      for (int c8 = 0; c8 < BN / 8; ++c8) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pv[e] = fast_exp2(sv[c8 * 8 + e] - mref);
          l += pv[e];
        }
        uint4 u;
        u.x = E::pack(pv[0], pv[1]);
        u.y = E::pack(pv[2], pv[3]);
        u.z = E::pack(pv[4], pv[5]);
        u.w = E::pack(pv[6], pv[7]);
        sts128(prow + ((c8 ^ (r & 7)) << 4), u);
      }
      // V rows at keys >= kend carry zero weight but may hold no data: zero them.
      if (key0 + BN > kend) {
        const int vfirst = max(0, kend - key0);
        const uint32_t vt = v_s + (j % STAGES) * L::kKV;
        const int nvec = (BN - vfirst) * (D / 8);
        for (int i = r; i < nvec; i += BM) {
          const int vr = vfirst + i / (D / 8), c16 = i % (D / 8);
          sts128(vt + (c16 >> 3) * (BN * 128) + vr * 128 + (((c16 & 7) ^ (vr & 7)) << 4), make_uint4(0, 0, 0, 0));
        }
      }
      fence_proxy_async_smem();
      tc5::fence_before();
      __syncwarp();
      if (lane == 0) tc5::arrive(p_full);
    }
    if (ok) {
      const bool done = mbar_wait_bounded(pv_done, (ntiles - 1) & 1, kWaitNs);
      ok = __all_sync(kFull, done);
    }
    if (!ok) {
      set_err(p.err_flags, PA_ERRF_TIMEOUT);
    } else {
      tc5::fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      T* dst = static_cast<T*>(p.out) + ((int64_t)(qa + r0 + r) * p.num_heads + h) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tc5::ld32(tmem + lane_off + 2 * BN + cc * 32, o);
        tc5::wait_ld();
        if (r < rows) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            uint4 u;
            u.x = E::pack(__uint_as_float(o[v4 * 8 + 0]) * inv, __uint_as_float(o[v4 * 8 + 1]) * inv);
            u.y = E::pack(__uint_as_float(o[v4 * 8 + 2]) * inv, __uint_as_float(o[v4 * 8 + 3]) * inv);
            u.z = E::pack(__uint_as_float(o[v4 * 8 + 4]) * inv, __uint_as_float(o[v4 * 8 + 5]) * inv);
            u.w = E::pack(__uint_as_float(o[v4 * 8 + 6]) * inv, __uint_as_float(o[v4 * 8 + 7]) * inv);
            *reinterpret_cast<uint4*>(dst + cc * 32 + v4 * 8) = u;
          }
        }
      }
    }
  }
  // Free tensor memory once every MMA of this CTA has completed.
  tc5::fence_before();
  __syncthreads();
  if (warp == 1) {
    if (active) mbar_wait_bounded(mma_done, 0, kWaitNs);
    __syncwarp();
    tc5::fence_after();
    tc5::tmem_free(tmem, kTmemCols);
  }
}

}  // namespace ptc
}  // namespace pa

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// Q as a 3-D tensor [total_q][num_heads][head_dim]: box {64, 1, 128 rows}, 128-byte swizzle.
bool make_q_map(CUtensorMap* map, const void* q, int total_q, int heads, int d) {
  void* fn_ptr = nullptr;
  cudaDriverEntryPointQueryResult qr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn_ptr, cudaEnableDefault, &qr) != cudaSuccess ||
      qr != cudaDriverEntryPointSuccess)
    return false;
  auto fn = reinterpret_cast<EncodeTiledFn>(fn_ptr);
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)heads, (cuuint64_t)total_q};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)heads * d * 2};
  const cuuint32_t box[3] = {64, 1, (cuuint32_t)pa::ptc::BM};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int D>
pa_status launch_tc(const CUtensorMap& km, const CUtensorMap& vm, const CUtensorMap& qm, const pa::ptc::Params& p,
                    int dev, cudaStream_t stream) {
  auto kern = pa::ptc::paged_prefill_tc_kernel<T, D>;
  const size_t smem = pa::ptc::Lay<D>::kSmem;
  static std::atomic<int> smem_set[pa::kMaxDevices];
  if (dev >= 0 && dev < pa::kMaxDevices && !smem_set[dev].load(std::memory_order_relaxed)) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "cudaFuncSetAttribute(prefill tcgen05)", e);
    smem_set[dev].store(1, std::memory_order_relaxed);
  }
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.q_tiles, p.num_heads, p.num_seqs);
  cfg.blockDim = dim3(pa::ptc::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, km, vm, qm, p);
  return e == cudaSuccess ? PA_OK : pa::fail(PA_ERR_CUDA, "launching paged_prefill_tc_kernel", e);
}

inline bool al(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" pa_status pa_prefill(void* out, const void* q, const int32_t* cu_q_lens, int total_q, int max_q_len,
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
  if (!al(out, 16) || !al(q, 16) || !al(k_cache, 16) || !al(v_cache, 16) || !al(cu_q_lens, 4) ||
      !al(block_tables, 4) || !al(context_lens, 4))
    return PA_ERR_INVALID;
  if (num_blocks > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return pa::fail(PA_ERR_CUDA, "cudaGetDevice", ce);
  CUtensorMap km, vm, qm;
  if (!pa::make_cache_map(&km, k_cache, num_blocks, num_kv_heads, block_size, head_dim) ||
      !pa::make_cache_map(&vm, v_cache, num_blocks, num_kv_heads, block_size, head_dim) ||
      !make_q_map(&qm, q, total_q, num_heads, head_dim))
    return pa::fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled rejected a layout", cudaSuccess);
  pa::ptc::Params p;
  p.out = out;
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
  p.q_tiles = (max_q_len + pa::ptc::BM - 1) / pa::ptc::BM;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == PA_F16)
    return head_dim == 128 ? launch_tc<__half, 128>(km, vm, qm, p, dev, s) : launch_tc<__half, 64>(km, vm, qm, p, dev, s);
  return head_dim == 128 ? launch_tc<__nv_bfloat16, 128>(km, vm, qm, p, dev, s)
                         : launch_tc<__nv_bfloat16, 64>(km, vm, qm, p, dev, s);
}
