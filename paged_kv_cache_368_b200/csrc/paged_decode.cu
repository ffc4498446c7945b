// Paged decode attention for B200 (sm_100a).
//
// What is computed ("【infra之路】10-PagedAttention 与 KV Cache 管理"):
//   section 1.1 -- one new query per sequence attends over every cached token,
//                  out = softmax(q K^T * scale) V;
//   sections 3.2-3.4 -- K/V live in fixed-size physical blocks reached through a
//                  per-sequence block table; attention itself is unchanged;
//   section 8 (Q2, Q3) -- long contexts are split FlashDecoding-style and the
//                  pieces are combined; the kernel tiles like FlashAttention
//                  (running max / running sum, "online softmax").
//
// Design (B200-first; the pages' own Ascend kernel copies scattered pages into
// a contiguous buffer first, which this design does not do):
//  * Work unit = (sequence, kv-head).  Its context is cut into chunks of 16
//    tokens.  All chunks of all units are laid end to end (sequence-major,
//    then kv-head, then chunk) and split evenly over every warp of a
//    persistent grid (one CTA per SM, 6-8 warps each): each warp owns one
//    contiguous run of chunks, so mixed context lengths balance to within a
//    chunk and no partition-size heuristic is needed.
//  * A warp's run is cut at unit boundaries into segments.  A segment that
//    covers a whole unit writes the normalised output directly; a unit split
//    across warps leaves un-normalised partials (m, l, o), and each
//    contributing warp then adds its chunk count to the unit's ticket
//    counter.  The warp that completes the count merges the partials by
//    log-sum-exp and writes the output, in the same launch: no warp waits
//    for another and there is no second kernel.
//  * Each warp is its own producer: lane 0 issues TMA tile loads (128-byte
//    swizzle, L2 evict-first) of the K and V rows of chunk k+DEPTH into a
//    per-warp ring of shared-memory stages, completion counted on an
//    mbarrier, while the warp computes on chunk k.  Block-table entries for
//    the next 32 chunks are fetched with one coalesced load (one per lane)
//    and kept in registers.
//  * Groups of 1-2 q-heads per kv-head (MHA) use CUDA cores: 16 lanes cover
//    one 256-byte K row (one 16-byte vector each), partial dot products of
//    8 tokens are reduced with a transposing shuffle tree.  Groups of 4-8
//    q-heads (GQA) form a real contraction: S = Q K^T and O += P V run on
//    the tensor cores (mma.sync m16n8k16, q-heads on M), fed by ldmatrix
//    from the swizzled tiles.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <mutex>

#include "paged_decode_kernel.cuh"
#include "pa_host.h"

// =============================================================== host side

namespace {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

namespace pa {
thread_local char g_last_error[256] = "no error";

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}


int device_sms(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

// The (cache-pool) tensor map: dims {head_dim, block_size, kv_heads, blocks},
// box {64 elements = 128 B, min(block_size, 16) rows, 1, 1}, 128-byte swizzle.
bool make_cache_map(CUtensorMap* map, const void* base, int64_t nb, int kvh, int bs, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)bs, (cuuint64_t)kvh, (cuuint64_t)nb};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)bs * d * 2, (cuuint64_t)kvh * bs * d * 2};
  const cuuint32_t box[4] = {64, (cuuint32_t)(bs < 16 ? bs : 16), 1, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}




bool have_tensor_map_encoder() { return encode_fn() != nullptr; }

pa_status fail(pa_status st, const char* what, cudaError_t e) {
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, e == cudaSuccess ? "" : cudaGetErrorString(e));
  return st;
}
}  // namespace pa

namespace {

template <typename T, int D, int G>
pa_status launch_decode(const CUtensorMap& km, const CUtensorMap& vm, const pa::DecodeParams& p, int ctas,
                        cudaStream_t stream, int dev) {
  using SH = pa::Shape<D, G>;
  auto kern = pa::paged_decode_kernel<T, D, G>;
  static std::atomic<int> smem_set[pa::kMaxDevices];
  const size_t smem = SH::smem_bytes(p.num_seqs);
  if (dev >= 0 && dev < pa::kMaxDevices && smem_set[dev].load(std::memory_order_relaxed) < (int)smem) {
    // Opt in to the largest dynamic size this kernel can use: the per-block
    // limit minus the kernel's static shared memory.
    int optin = 0;
    cudaFuncAttributes fa;
    cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "querying shared-memory limits", e);
    const int dyn_max = optin - static_cast<int>(fa.sharedSizeBytes);
    if (dyn_max < (int)smem) return pa::fail(PA_ERR_UNSUPPORTED, "num_seqs too large for shared memory", cudaSuccess);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max);
    if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "cudaFuncSetAttribute(decode)", e);
    smem_set[dev].store(dyn_max, std::memory_order_relaxed);
  }
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(SH::kWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, km, vm, p);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "launching paged_decode_kernel", e);
  return PA_OK;
}

template <typename T, int D>
pa_status dispatch_g(int G, const CUtensorMap& km, const CUtensorMap& vm, const pa::DecodeParams& p, int ctas,
                     cudaStream_t s, int dev) {
  switch (G) {
    case 1: return launch_decode<T, D, 1>(km, vm, p, ctas, s, dev);
    case 2: return launch_decode<T, D, 2>(km, vm, p, ctas, s, dev);
    case 4: return launch_decode<T, D, 4>(km, vm, p, ctas, s, dev);
    case 8: return launch_decode<T, D, 8>(km, vm, p, ctas, s, dev);
    default: return PA_ERR_UNSUPPORTED;
  }
}

bool valid_block_size(int bs) { return bs == 8 || bs == 16 || bs == 32 || bs == 64; }

}  // namespace

namespace pa {

// Host checks of a decode call's sizes (no CUDA call).  Returns PA_OK and
// fills the shape part of `plan`, or the status to return without launching.
pa_status plan_decode(int num_seqs, int max_blocks_per_seq, int max_context_len, float scale, int num_heads,
                      int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                      int max_ctas, DecodePlan* plan) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads) return PA_ERR_INVALID;
  if (max_blocks_per_seq <= 0 || max_context_len < 0 || num_blocks <= 0 || max_ctas < 0) return PA_ERR_INVALID;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_INVALID;
  if (!std::isfinite(scale)) return PA_ERR_INVALID;
  const int G = num_heads / num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (!valid_block_size(block_size)) return PA_ERR_UNSUPPORTED;
  if (num_kv_heads >= (1 << 15)) return PA_ERR_UNSUPPORTED;
  // One launch takes at most kMaxSeqs sequences (its per-sequence prefix
  // table lives in shared memory); pa_decode runs a larger batch as several
  // launches, so the limits below are those of one launch.
  const int64_t batch = std::min(num_seqs, kMaxSeqs);
  const int64_t cap64 = std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * block_size);
  const int64_t upper = batch * num_kv_heads * ((cap64 + kChunk - 1) / kChunk);
  if (upper >= (int64_t(1) << 31)) return PA_ERR_UNSUPPORTED;
  if (num_blocks > 0x7fffffffLL) return PA_ERR_UNSUPPORTED;
  plan->G = G;
  plan->head_dim = head_dim;
  plan->ctx_cap = static_cast<int>(cap64);
  plan->warps = warps_for(head_dim, G);
  plan->ctas = 0;
  plan->layout = ws_layout(0, 0, G, head_dim);
  plan->upper_chunks = upper;
  return PA_OK;
}

// The grid for the current device (its SM count) and its workspace layout.
pa_status plan_decode_grid(int max_ctas, DecodePlan* plan) {
  const int64_t upper = plan->upper_chunks;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return fail(PA_ERR_CUDA, "cudaGetDevice", ce);
  const int sms = device_sms(dev);
  if (sms <= 0) return fail(PA_ERR_CUDA, "querying the SM count", cudaSuccess);
  // A persistent grid: at most one CTA per SM, and no more CTAs than give
  // each warp about four chunks.
  int ctas = static_cast<int>(std::min<int64_t>(sms, std::max<int64_t>(1, (upper + plan->warps * 4 - 1) /
                                                                            (plan->warps * 4))));
  if (max_ctas > 0) ctas = std::min(ctas, max_ctas);
  plan->ctas = ctas;
  plan->layout = ws_layout(ctas * plan->warps, sms * kMaxWarpsPerCta, plan->G, plan->head_dim);
  return PA_OK;
}

}  // namespace pa

extern "C" size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                           int max_context_len) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads) return 0;
  if (head_dim != 64 && head_dim != 128) return 0;
  if (max_context_len < 0) return 0;
  const int G = num_heads / num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const int sms = pa::device_sms(dev);
  if (sms <= 0) return 0;
  // The largest grid this shape can launch on this device (one CTA per SM).
  return pa::ws_layout(sms * pa::warps_for(head_dim, G), sms * pa::kMaxWarpsPerCta, G, head_dim).total;
}

extern "C" pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                               int num_seqs, int max_context_len, float scale, int num_heads, int num_kv_heads,
                               int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype, void* workspace,
                               size_t workspace_bytes, int max_ctas, int32_t* err_flags, pa_stream_t stream) {
  pa::DecodePlan plan;
  const pa_status st = pa::plan_decode(num_seqs, max_blocks_per_seq, max_context_len, scale, num_heads,
                                       num_kv_heads, head_dim, block_size, num_blocks, dtype, max_ctas, &plan);
  if (st != PA_OK) return st;
  if (num_seqs == 0) return PA_OK;
  if (!pa::decode_pointers_ok(out, q, k_cache, v_cache, block_tables, context_lens)) return PA_ERR_INVALID;
  const pa_status gst = pa::plan_decode_grid(max_ctas, &plan);
  if (gst != PA_OK) return gst;
  const pa::WsLayout& L = plan.layout;
  if (!workspace || workspace_bytes < L.total || !aligned(workspace, 16)) return PA_ERR_WORKSPACE;
  const int G = plan.G, ctas = plan.ctas, warps = plan.warps;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return pa::fail(PA_ERR_CUDA, "cudaGetDevice", ce);

  CUtensorMap km, vm;
  if (!pa::have_tensor_map_encoder())
    return pa::fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not found", cudaSuccess);
  if (!pa::make_cache_map(&km, k_cache, num_blocks, num_kv_heads, block_size, head_dim) ||
      !pa::make_cache_map(&vm, v_cache, num_blocks, num_kv_heads, block_size, head_dim))
    return pa::fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled rejected the cache layout", cudaSuccess);

  pa::DecodeParams p;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.err_flags = err_flags;
  p.num_blocks = num_blocks;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.ctx_cap = plan.ctx_cap;
  p.max_context_len = max_context_len;
  p.num_heads = num_heads;
  p.num_kv_heads = num_kv_heads;
  p.block_size = block_size;
  p.scale_log2 = scale * 1.4426950408889634f;

  // Batches of at most kMaxSeqs sequences, one launch each, in order on
  // `stream`.  They share the workspace: a launch touches it only after its
  // programmatic wait for the previous one, and leaves the ticket counters at
  // zero.  The first batch is the largest, so its grid and layout (checked
  // above) bound every later one's.
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t row_bytes = (size_t)num_heads * head_dim * 2;  // one sequence of q or out
  for (int s0 = 0; s0 < num_seqs; s0 += pa::kMaxSeqs) {
    const int nb = std::min(pa::kMaxSeqs, num_seqs - s0);
    int bctas = ctas;
    pa::WsLayout BL = L;
    if (s0 > 0) {  // the last batch may be smaller: its own grid
      pa::DecodePlan bp;
      const pa_status bst = pa::plan_decode(nb, max_blocks_per_seq, max_context_len, scale, num_heads, num_kv_heads,
                                            head_dim, block_size, num_blocks, dtype, max_ctas, &bp);
      if (bst != PA_OK) return bst;
      const pa_status bgst = pa::plan_decode_grid(max_ctas, &bp);
      if (bgst != PA_OK) return bgst;
      bctas = bp.ctas;
      BL = bp.layout;
    }
    p.out = static_cast<uint8_t*>(out) + (size_t)s0 * row_bytes;
    p.q = static_cast<const uint8_t*>(q) + (size_t)s0 * row_bytes;
    p.block_tables = block_tables + (size_t)s0 * max_blocks_per_seq;
    p.context_lens = context_lens + s0;
    p.num_seqs = nb;
    p.ws_tickets = reinterpret_cast<int*>(ws + BL.tickets);
    p.ws_ml = reinterpret_cast<float2*>(ws + BL.ml);
    p.ws_o = reinterpret_cast<float*>(ws + BL.o);
    p.total_warps = bctas * warps;
    pa_status lst;
    if (dtype == PA_F16) {
      lst = head_dim == 128 ? dispatch_g<__half, 128>(G, km, vm, p, bctas, s, dev)
                            : dispatch_g<__half, 64>(G, km, vm, p, bctas, s, dev);
    } else {
      lst = head_dim == 128 ? dispatch_g<__nv_bfloat16, 128>(G, km, vm, p, bctas, s, dev)
                            : dispatch_g<__nv_bfloat16, 64>(G, km, vm, p, bctas, s, dev);
    }
    if (lst != PA_OK) return lst;
  }
  return PA_OK;
}

extern "C" const char* pa_status_string(pa_status status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID: return "PA_ERR_INVALID: invalid argument";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED: shape or size outside the compiled set";
    case PA_ERR_CUDA: return "PA_ERR_CUDA: CUDA call or kernel launch failed";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE: workspace missing or too small";
    case PA_ERR_OUT_OF_BLOCKS: return "PA_ERR_OUT_OF_BLOCKS: not enough free blocks";
  }
  return "unknown pa_status";
}

extern "C" int pa_version(void) { return 100; }

extern "C" const char* pa_last_error(void) { return pa::g_last_error; }
