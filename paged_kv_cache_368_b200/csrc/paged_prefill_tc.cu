// Multi-token paged attention on the 5th-generation tensor cores (tcgen05,
// accumulators in tensor memory).  Same contract as the mma.sync kernel in
// paged_prefill.cu: the last n cached tokens of each sequence attend causally
// over its paged K/V (the ops-transformer page's [batch, heads, seq_len,
// head_dim] call; each row the section 1.1 formula of "【infra之路】10-
// PagedAttention 与 KV Cache 管理", restricted to positions up to its own).
//
// One CTA per (256 query rows, q-head, sequence), 12 warps:
//   warp 0      TMA: both 128-row Q tiles once (3-D map over [token][head][d]),
//               then the K tiles of 64 keys, one 16-row box per block and
//               head_dim half, read through the block table;
//   warp 2      TMA: the V tiles, one 5-D box per block covering both
//               head_dim halves (chunk-major layout);
//               K and V go into a ring 5 tiles deep (8 at head_dim 64);
//   warp 1      allocates tensor memory and runs the MMA schedule as a whole
//               warp, one elected lane issuing: S = Q K^T (M 128, N 64, both
//               operands in shared memory) into one of two TMEM buffers per
//               query tile, and O += P V (M 128, N head_dim) with P read from
//               tensor memory; per query tile, P.V of tile j comes before the
//               scores of tile j+2, which reuse P's columns;
//   warps 4-7,  softmax of query tiles 0 and 1: thread t owns query row t
//   8-11        (TMEM lane t).  It reads S_j, masks on tiles that reach its
//               first row, keeps a reference max that moves only when it grows
//               by more than 2^8 (so the O rescale in tensor memory is rare),
//               writes P_j as 16-bit pairs over S_j, and at the end reads O and
//               divides by the row sum;
//   warp 3      idle.
// Shared-memory operand tiles are 128-byte-swizzled, the layout TMA writes
// and the MMA descriptors name directly.
#include <algorithm>
#include <atomic>
#include <cmath>

#include "exp2_poly.cuh"
#include "pa_host.h"
#include "tcgen05.cuh"

namespace pa {
namespace ptc {

constexpr int BM = 128;  // query rows per softmax group (MMA M)
constexpr int BN = 64;   // keys per tile (MMA N of S, K of P.V)
constexpr int kGroups = 2;  // query tiles (softmax warpgroups) per CTA sharing each K/V tile
constexpr uint64_t kWaitNs = 1000000000ull;

// Which exponentials of the softmax run as the FMA-pipe polynomial of
// exp2_poly.cuh (two at a time) instead of on the special-function unit:
// bit b of the mask set -> the key pairs 8m+b.
#ifndef PA_PREFILL_POLY_MASK_D128
#define PA_PREFILL_POLY_MASK_D128 0x00  // none: measured 908 vs 917 TFLOP/s with 1/8
#endif
#ifndef PA_PREFILL_POLY_MASK_D64
#define PA_PREFILL_POLY_MASK_D64 0x88   // pairs 3 and 7 of 8: 1/4 (547 vs 513 TFLOP/s)
#endif


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
  static constexpr int NWG = kGroups;
  static constexpr int STAGES = D == 128 ? 5 : 8;  // K/V ring depth (tiles in flight)
  static constexpr int kQ = BM * D * 2;   // per group: [D/64][BM rows][128 B]
  // one K or V tile; K: [D/64][BN rows][128 B], V: [BN/16 chunks][block][D/64][rows][128 B]
  static constexpr int kKV = BN * D * 2;
  static constexpr int kOffK = NWG * kQ;
  static constexpr int kOffV = kOffK + STAGES * kKV;
  static constexpr int kOffBar = kOffV + STAGES * kKV;
  // barriers: q_full, kv_full[S] (one arrival per producer warp), kv_empty[S];
  // per group s_full[2], p_full[2], pv_done[2]; mma_done
  static constexpr int kBars = 1 + 2 * STAGES + NWG * 6 + 1;
  static constexpr size_t kSmem = 1024 + kOffBar + kBars * 8 + 16;
  static constexpr int kThreads = (4 + 4 * NWG) * 32;  // warps 0-3: TMA (Q, K), MMA, TMA (V), idle
  // key pairs 8m+b with bit b set take the FMA-pipe polynomial for their exponentials
  static constexpr unsigned kPolyMask = D == 128 ? PA_PREFILL_POLY_MASK_D128 : PA_PREFILL_POLY_MASK_D64;
  // Tensor memory per group: S0 | S1 | O.  P of tile j (16-bit, two per
  // column) overwrites the front of S(j & 1) once the softmax has read it.
  static constexpr uint32_t kColsPerGroup = 2 * BN + D;
  static constexpr uint32_t kTmemCols = NWG * kColsPerGroup <= 256 ? 256u : 512u;
  static_assert(NWG * kColsPerGroup <= 512, "tensor memory");
  static_assert(kSmem <= 232448, "shared memory per CTA");
};

template <typename T, int D>
__global__ void __launch_bounds__(Lay<D>::kThreads, 1)
    paged_prefill_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                            const __grid_constant__ CUtensorMap qmap, const Params p) {
  using E = Elem<T>;
  using L = Lay<D>;
  constexpr int NWG = L::NWG, STAGES = L::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;  // K and V of a tile: the score MMA waits for both
  uint64_t* kv_empty = kv_full + STAGES;
  // Group g owns bars [6g, 6g+6); double-buffered barriers are indexed by the
  // tile's parity, so no waiter can fall two phases behind.
  uint64_t* grp_bars = kv_empty + STAGES;
  auto s_full = [&](int g, int b) { return grp_bars + 6 * g + b; };
  auto p_full = [&](int g, int b) { return grp_bars + 6 * g + 2 + b; };
  auto pv_done = [&](int g, int b) { return grp_bars + 6 * g + 4 + b; };
  uint64_t* mma_done = grp_bars + 6 * NWG;
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
      mbar_init(&kv_full[i], 2);
      mbar_init(&kv_empty[i], 1);
    }
    for (int g = 0; g < NWG; ++g) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(s_full(g, b), 1);
        mbar_init(p_full(g, b), 4);
        mbar_init(pv_done(g, b), 1);
      }
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 1) tc5::tmem_alloc(tmem_slot, L::kTmemCols);
  griddep_wait();
  griddep_launch_dependents();
  tc5::fence_before();
  __syncthreads();
  tc5::fence_after();
  const uint32_t tmem = *tmem_slot;

  // Geometry: the CTA covers query rows r0 .. r0 + NWG*BM - 1 of the sequence;
  // group g the BM rows starting at r0 + g*BM.
  const int qa = __ldg(p.cu_q + s), qb = __ldg(p.cu_q + s + 1);
  const int ctx_raw = __ldg(p.context_lens + s);
  const int ctx = ctx_raw < 0 ? 0 : (ctx_raw > p.ctx_cap ? p.ctx_cap : ctx_raw);
  int n = qb - qa;
  if (qa < 0 || qb > p.total_q) n = 0;  // malformed offsets: touch no row of q or out
  if (ctx != ctx_raw || n != qb - qa || n > ctx) {
    if (threadIdx.x == 0 && tile == 0 && h == 0) set_err(p.err_flags, PA_ERRF_CONTEXT);
    n = n < 0 ? 0 : (n > ctx ? ctx : n);
  }
  const int r0 = tile * (NWG * BM);
  auto g_rows = [&](int g) { return max(0, min(BM, n - r0 - g * BM)); };
  auto g_pos0 = [&](int g) { return ctx - n + r0 + g * BM; };
  auto g_tiles = [&](int g) { return g_rows(g) > 0 ? (g_pos0(g) + g_rows(g) + BN - 1) / BN : 0; };
  int ntiles = 0, kend = 0, lastg = 0;
#pragma unroll
  for (int g = 0; g < NWG; ++g)
    if (g_rows(g) > 0) {
      ntiles = g_tiles(g);
      kend = g_pos0(g) + g_rows(g);
      lastg = g;
    }
  const bool active = ntiles > 0;
  const uint32_t q_s = base, k_s = base + L::kOffK, v_s = base + L::kOffV;

  if (active && (warp == 0 || warp == 2)) {
    // ------------------------------------------------------------- producers
    // Warp 0 copies Q and every K tile, warp 2 every V tile: one thread
    // issues a TMA box only every 100-200 cycles, so the two streams go out
    // in parallel.  Both walk the same block-table entries.
    const bool kprod = warp == 0;
    const int bs = p.block_size;
    const int32_t* row = p.block_tables + (int64_t)s * p.max_blocks_per_seq;
    const uint32_t box_bytes = (bs < 16 ? bs : 16) * 128;
    if (kprod && lane == 0) {
      uint32_t qbytes = 0;
      for (int g = 0; g < NWG; ++g)
        if (g_rows(g) > 0) qbytes += L::kQ;
      mbar_arrive_expect_tx(q_full, qbytes);
      for (int g = 0; g < NWG; ++g) {
        if (g_rows(g) == 0) continue;
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tc5::tma_load_3d(q_s + g * L::kQ + c * (BM * 128), &qmap, q_full, 64 * c, h, qa + r0 + g * BM);
      }
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
          if (kprod) set_err(p.err_flags, PA_ERRF_BLOCK_RANGE);
          b0 = b1 = -1;
        }
      }
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
          if (j >= STAGES && !tc5::wait(&kv_empty[st], ((j / STAGES) - 1) & 1, kWaitNs)) {
            set_err(p.err_flags, PA_ERRF_TIMEOUT);
            bad = 1;
          } else {
            uint32_t bytes = 0;  // per pool
#pragma unroll
            for (int q = 0; q < BN / 16; ++q)
              bytes += (bb0[q] < 0 ? 0 : (bb1[q] >= 0 ? 2 : 1)) * (D / 64) * box_bytes;
            if (kprod) {
              // K: one box per head_dim half and block, into [half][BN rows][128 B].
              const uint32_t kdst = k_s + st * L::kKV;
              mbar_arrive_expect_tx(&kv_full[st], bytes);
#pragma unroll
              for (int q = 0; q < BN / 16; ++q) {
                const int nb = bb0[q] < 0 ? 0 : (bb1[q] >= 0 ? 2 : 1);
                for (int b = 0; b < nb; ++b) {
                  const int phys = b == 0 ? bb0[q] : bb1[q];
#pragma unroll
                  for (int cq = 0; cq < D / 64; ++cq)
                    tc5::tma_load_4d(kdst + cq * (BN * 128) + q * 2048 + b * 1024, &kmap, &kv_full[st], 64 * cq,
                                     rr0[q], kvh, phys);
                }
              }
            } else {
              // V: one box per block covering both head_dim halves, chunk-major
              // ([16-key chunk][block][half][rows][128 B]).
              const uint32_t vdst = v_s + st * L::kKV;
              mbar_arrive_expect_tx(&kv_full[st], bytes);
#pragma unroll
              for (int q = 0; q < BN / 16; ++q) {
                const int nb = bb0[q] < 0 ? 0 : (bb1[q] >= 0 ? 2 : 1);
                for (int b = 0; b < nb; ++b)
                  tc5::tma_load_5d(vdst + q * (32 * D) + b * (D / 64) * box_bytes, &vmap, &kv_full[st], 0, rr0[q], 0,
                                   kvh, b == 0 ? bb0[q] : bb1[q]);
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
        tc5::wait(&kv_full[j % STAGES], (j / STAGES) & 1, kWaitNs);
    }
  } else if (active && warp == 1) {
    // ------------------------------------------------------------- MMA issue
    // The whole warp follows the schedule, converged, and one elected lane
    // issues every MMA and commit under a predicate (issuing from a lane
    // that has diverged from its warp measured ~4x slower per MMA).  The
    // warp shares its scheduler with two softmax warps and paces the tensor
    // pipe, so its instruction count per tile matters: descriptors and tile
    // counts are computed once, and each MMA only adds a constant offset.
    // Per tile j, per query tile g: P.V of tile j, then the scores of tile
    // j+2 into the S buffer that P occupied (tensor-core operations of one
    // thread run in issue order).
    constexpr int fmt = Elem<T>::kind == PA_BF16 ? 1 : 0;
    constexpr uint32_t id_qk = tc5::f16_idesc(fmt, BM, BN, 0, 0);
    constexpr uint32_t id_pv = tc5::f16_idesc(fmt, BM, D, 0, 1);
    const uint32_t leader = tc5::elect_one();
    // V tile, chunk-major: the head_dim halves of a chunk are box_rows * 128 B
    // apart (LBO) and its two 8-key row groups 1 KB apart, or one block's box
    // apart when a chunk spans two 8-row blocks (SBO).
    const int box_rows = p.block_size < 16 ? p.block_size : 16;
    const uint32_t v_lbo = box_rows * 128;
    const uint32_t v_sbo = p.block_size >= 16 ? 1024u : uint32_t(D / 64) * 1024u;
    // Descriptors of the first operand tiles; the offsets added below are in
    // the descriptor's 16-byte units (the start-address field never carries:
    // shared memory ends below 2^18 bytes).
    const uint64_t dq = tc5::sw128_desc(q_s, 16, 1024);
    const uint64_t dk = tc5::sw128_desc(k_s, 16, 1024);
    const uint64_t dv = tc5::sw128_desc(v_s, v_lbo, v_sbo);
    static_assert(NWG == 2, "two query tiles per CTA");
    const int gt0 = g_tiles(0), gt1 = g_tiles(1);
    auto gt = [&](int g) { return g == 0 ? gt0 : gt1; };
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      // one plain probe first: most of these waits are already satisfied,
      // and the suspending form costs the pacing warp ~100 cycles even then
      const bool got = tc5::wait_fast(bar, parity, kWaitNs);
      return __all_sync(kFull, got);
    };
    int kv_seen = -1;  // highest tile whose copies this warp has already waited for
    auto issue_qk = [&](int g, int j) -> bool {  // S(g, j&1) = Q_g K_j^T
      const int st = j % STAGES;
      // Tiles are waited for in increasing order; the second query tile's
      // scores of the same tile skip the (already satisfied) wait.
      if (j > kv_seen) {
        if (!wait_all(&kv_full[st], (j / STAGES) & 1)) return false;
        kv_seen = j;
      }
      tc5::fence_after();
      const uint64_t a = dq + uint64_t(g * (L::kQ >> 4));
      const uint64_t b = dk + uint64_t(st * (L::kKV >> 4));
      const uint32_t sd = tmem + g * L::kColsPerGroup + (j & 1) * BN;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks)
        tc5::mma_ss_if(leader, sd, a + uint64_t(((ks >> 2) * (BM * 128) + (ks & 3) * 32) >> 4),
                       b + uint64_t(((ks >> 2) * (BN * 128) + (ks & 3) * 32) >> 4), id_qk, ks > 0);
      tc5::commit_if(leader, s_full(g, j & 1));
      __syncwarp();
      return true;
    };
    auto issue_pv = [&](int g, int j) -> bool {  // O_g += P(g, j) V_j, P from tensor memory
      // V landed with K: the scores of tile j, issued earlier, waited for both.
      if (!wait_all(p_full(g, j & 1), (j >> 1) & 1)) return false;
      tc5::fence_after();
      const uint64_t b = dv + uint64_t((j % STAGES) * (L::kKV >> 4));
      const uint32_t pa = tmem + g * L::kColsPerGroup + (j & 1) * BN;
      const uint32_t od = tmem + g * L::kColsPerGroup + 2 * BN;
      const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
      for (int ks = 0; ks < BN / 16; ++ks)
        tc5::mma_ts_if(leader, od, pa + ks * 8, b + uint64_t((ks * (32 * D)) >> 4), id_pv, ks > 0 ? 1u : acc0);
      tc5::commit_if(leader, pv_done(g, j & 1));
      __syncwarp();
      return true;
    };
    bool ok = wait_all(q_full, 0);
    if (ok) tc5::fence_after();
    for (int j = 0; j < 2 && ok; ++j)
      for (int g = 0; g < NWG && ok; ++g)
        if (j < gt(g)) ok = issue_qk(g, j);
    for (int j = 0; ok && j < ntiles; ++j) {
      // On the CTA's last tile the query tile that zeroes the unused V rows goes first.
      const bool last = j == ntiles - 1;
#pragma unroll
      for (int gi = 0; gi < NWG; ++gi) {
        const int g = last ? NWG - 1 - gi : gi;
        if (ok && j < gt(g)) ok = issue_pv(g, j);
        if (ok && gi == NWG - 1) tc5::commit_if(leader, &kv_empty[j % STAGES]);  // every P.V of tile j issued
        if (ok && j + 2 < gt(g)) ok = issue_qk(g, j + 2);
      }
    }
    if (!ok && leader) set_err(p.err_flags, PA_ERRF_TIMEOUT);
    tc5::commit_if(leader, mma_done);  // lets the CTA free tensor memory once every MMA has finished
  } else if (active && warp >= 4) {
    // ------------------------------------------------------------- softmax
    const int g = (warp - 4) >> 2;  // query tile (warpgroup) of this warp
    const int w = warp & 3;         // tensor-memory lanes 32w..32w+31
    const int r = w * 32 + lane;    // query row within the group's tile
    const int rows = g_rows(g), pos0 = g_pos0(g), gtiles = g_tiles(g);
    const int gkend = pos0 + rows;
    const uint32_t lane_off = uint32_t(w * 32) << 16;
    const uint32_t s_col = tmem + g * L::kColsPerGroup + lane_off, o_col = s_col + 2 * BN;
    const int rp = pos0 + r;  // this row's position
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < gtiles; ++j) {
      const uint32_t sj = s_col + (j & 1) * BN;
      const bool got = tc5::wait(s_full(g, j & 1), (j >> 1) & 1, kWaitNs);
      if (!__all_sync(kFull, got)) {
        ok = false;
        break;
      }
      tc5::fence_after();
      uint32_t sr[BN / 32][32];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) tc5::ld32(sj + c * 32, sr[c]);
      tc5::wait_ld();

      const int key0 = j * BN;
      // Only tiles that reach past the group's first row need the causal
      // mask (warp-uniform); keys [0, lim) of the tile are visible to this row.
      const bool diag = key0 + BN - 1 > pos0;
      const int lim = diag ? min(rp + 1, gkend) - key0 : BN;
      float sv[BN];  // raw scores q.k
#pragma unroll
      for (int i = 0; i < BN; ++i) sv[i] = __uint_as_float(sr[i >> 5][i & 31]);
      if (diag) {
#pragma unroll
        for (int i = 0; i < BN; ++i) sv[i] = i < lim ? sv[i] : -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
      for (int i = 0; i < BN; i += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = tc5::max3(mx[k], sv[i + k], sv[i + 8 + k]);
      const float rmax = tc5::max3(tc5::max3(mx[0], mx[1], mx[2]), tc5::max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
      // the scale is positive (checked on the host), so it commutes with the max
      const float mt = rmax == -INFINITY ? -INFINITY : rmax * p.scale_log2;
      const float m_new = fmaxf(m_ref, mt);
      const bool resc = m_new > m_ref + 8.f;  // also true the first time (m_ref = -inf)
      // O may be rescaled only after the P.V of tile j-1 has landed in it.
      if (j > 0 && __any_sync(kFull, resc)) {
        const bool done = tc5::wait(pv_done(g, (j - 1) & 1), ((j - 1) >> 1) & 1, kWaitNs);
        if (!__all_sync(kFull, done)) {
          ok = false;
          break;
        }
        tc5::fence_after();
        const float alpha = resc ? fast_exp2(m_ref - m_new) : 1.f;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tc5::ld32(o_col + cc * 32, o);
          tc5::wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tc5::st32(o_col + cc * 32, o);
        }
      }
      if (resc) {
        l *= (m_ref == -INFINITY) ? 0.f : fast_exp2(m_ref - m_new);
        m_ref = m_new;
      }
      const float mref = m_ref == -INFINITY ? 0.f : m_ref;
      // P row, 16-bit, two keys per tensor-memory column, into the front of
      // this tile's S buffer (already read).
      // Scale-and-shift and the row sum run as packed fp32x2 operations (one
      // instruction for two keys); the exponentials on the special-function unit.
      uint32_t pk[BN / 2];
      float ls[4][2] = {};
#pragma unroll
      for (int i = 0; i < BN / 2; ++i) {
        float x0, x1, p0, p1;
        tc5::fma2(x0, x1, sv[2 * i], sv[2 * i + 1], p.scale_log2, -mref);
        if ((L::kPolyMask >> (i & 7)) & 1u) {
          exp2_poly2(p0, p1, x0, x1);
        } else {
          p0 = fast_exp2(x0);
          p1 = fast_exp2(x1);
        }
        tc5::add2(ls[i & 3][0], ls[i & 3][1], p0, p1);
        pk[i] = E::pack(p0, p1);
      }
      l += ((ls[0][0] + ls[0][1]) + (ls[1][0] + ls[1][1])) + ((ls[2][0] + ls[2][1]) + (ls[3][0] + ls[3][1]));
      tc5::st32(sj, pk);
      // V rows at keys >= the CTA's last visible key carry zero weight for
      // every row but may hold no data: the last group with rows zeroes them
      // in the CTA's last tile (once its copy has landed), and its P.V is
      // issued before the others'.
      if (g == lastg && key0 + BN > kend) {
        const bool vin = tc5::wait(&kv_full[j % STAGES], (j / STAGES) & 1, kWaitNs);
        if (!__all_sync(kFull, vin)) {
          ok = false;
          break;
        }
        const int vfirst = max(0, kend - key0);
        const uint32_t vt = v_s + (j % STAGES) * L::kKV;
        const int nvec = (BN - vfirst) * (D / 8);
        const int box_rows = p.block_size < 16 ? p.block_size : 16;
        for (int i = r; i < nvec; i += BM) {
          const int vr = vfirst + i / (D / 8), c16 = i % (D / 8);
          const int kk = vr & 15, vb = kk / box_rows, rr = kk % box_rows;
          sts128(vt + (vr >> 4) * (32 * D) + (vb * (D / 64) + (c16 >> 3)) * box_rows * 128 + rr * 128 +
                     (((c16 & 7) ^ (rr & 7)) << 4),
                 make_uint4(0, 0, 0, 0));
        }
        fence_proxy_async_smem();
      }
      tc5::wait_st();
      tc5::fence_before();
      __syncwarp();
      if (lane == 0) tc5::arrive(p_full(g, j & 1));
    }
    if (ok && gtiles > 0) {
      const int jl = gtiles - 1;
      const bool done = tc5::wait(pv_done(g, jl & 1), (jl >> 1) & 1, kWaitNs);
      ok = __all_sync(kFull, done);
    }
    if (!ok) {
      set_err(p.err_flags, PA_ERRF_TIMEOUT);
    } else if (gtiles > 0) {
      tc5::fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      T* dst = static_cast<T*>(p.out) + ((int64_t)(qa + r0 + g * BM + r) * p.num_heads + h) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tc5::ld32(o_col + cc * 32, o);
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
    if (active) tc5::wait(mma_done, 0, kWaitNs);
    __syncwarp();
    tc5::fence_after();
    tc5::tmem_free(tmem, L::kTmemCols);
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

// V pool [NB][KVH][BS][D] as a 5-D tensor {64 dims, rows, D/64 halves, kv
// head, block} so that one box brings a block's rows for every head_dim half
// ([half][rows][128 B], 128-byte swizzle).
bool make_v_map(CUtensorMap* map, const void* v, int64_t nb, int kvh, int bs, int d) {
  void* fn_ptr = nullptr;
  cudaDriverEntryPointQueryResult qr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn_ptr, cudaEnableDefault, &qr) != cudaSuccess ||
      qr != cudaDriverEntryPointSuccess)
    return false;
  auto fn = reinterpret_cast<EncodeTiledFn>(fn_ptr);
  const cuuint64_t dims[5] = {64, (cuuint64_t)bs, (cuuint64_t)(d / 64), (cuuint64_t)kvh, (cuuint64_t)nb};
  const cuuint64_t strides[4] = {(cuuint64_t)d * 2, 128, (cuuint64_t)bs * d * 2, (cuuint64_t)kvh * bs * d * 2};
  const cuuint32_t box[5] = {64, (cuuint32_t)(bs < 16 ? bs : 16), (cuuint32_t)(d / 64), 1, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 5, const_cast<void*>(v), dims, strides, box, estr,
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
  cfg.blockDim = dim3(pa::ptc::Lay<D>::kThreads);
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
  if (!(scale > 0.f)) return PA_ERR_UNSUPPORTED;
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
      !make_v_map(&vm, v_cache, num_blocks, num_kv_heads, block_size, head_dim) ||
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
  const int rows_per_cta = pa::ptc::BM * pa::ptc::kGroups;
  p.q_tiles = (max_q_len + rows_per_cta - 1) / rows_per_cta;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == PA_F16)
    return head_dim == 128 ? launch_tc<__half, 128>(km, vm, qm, p, dev, s) : launch_tc<__half, 64>(km, vm, qm, p, dev, s);
  return head_dim == 128 ? launch_tc<__nv_bfloat16, 128>(km, vm, qm, p, dev, s)
                         : launch_tc<__nv_bfloat16, 64>(km, vm, qm, p, dev, s);
}
