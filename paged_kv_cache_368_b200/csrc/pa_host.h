// Host-side helpers shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "paged.h"

namespace pa {

constexpr int kMaxDevices = 64;

// Decode workspace for a grid of W warps on a device whose largest grid has
// Wmax warps (SM count x kMaxWarpsPerCta), group size G, head_dim D:
//   tickets [Wmax] int32  per split unit (indexed by the warp holding its
//                         first chunk): chunks accounted for so far; zero
//                         between calls
//   ml      [2W][G]       float2 (running max in log2 units, running sum)
//   o       [2W][G][D]    float  un-normalised partial outputs
// Two partial slots per warp: a warp's run has at most two segments that
// cover only part of a unit (its first and its last).  The ticket region has
// the same size for every call on a device, so the partials of one call
// never land on the counters of another that reuses the workspace with a
// larger grid.
constexpr int kMaxWarpsPerCta = 8;

struct WsLayout {
  size_t tickets, ml, o, total;
};

constexpr size_t round256(size_t x) { return (x + 255) / 256 * 256; }

constexpr WsLayout ws_layout(int W, int Wmax, int G, int D) {
  return WsLayout{0, round256(size_t(Wmax) * 4), round256(size_t(Wmax) * 4) + round256(size_t(2) * W * G * 8),
                  round256(size_t(Wmax) * 4) + round256(size_t(2) * W * G * 8) + size_t(2) * W * G * D * 4};
}

struct DecodePlan {
  int G, head_dim, ctx_cap, warps, ctas;
  int64_t upper_chunks;  // num_seqs * num_kv_heads * ceil(context bound / 16)
  WsLayout layout;       // for the grid that will be launched (after plan_decode_grid)
};

// Argument checks of a decode call (no CUDA call): PA_OK, or the status to
// return before anything is launched.
pa_status plan_decode(int num_seqs, int max_blocks_per_seq, int max_context_len, float scale, int num_heads,
                      int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, pa_dtype dtype,
                      int max_ctas, DecodePlan* plan);

// The launch grid on the current device and its workspace layout.
pa_status plan_decode_grid(int max_ctas, DecodePlan* plan);

// Non-null and aligned data pointers of a decode call (16 bytes for the
// fp16/bf16 arrays, 4 for the int32 ones).
inline bool decode_pointers_ok(const void* out, const void* q, const void* k_cache, const void* v_cache,
                               const void* block_tables, const void* context_lens) {
  auto al = [](const void* p, uintptr_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
  return al(out, 16) && al(q, 16) && al(k_cache, 16) && al(v_cache, 16) && al(block_tables, 4) &&
         al(context_lens, 4);
}

// SM count of device `dev` (cached), 0 on error.
int device_sms(int dev);

// Tensor map of a cache pool [nb][kvh][bs][d] of 16-bit elements: box
// {64 elements = 128 B, min(bs, 16) rows, 1, 1}, 128-byte swizzle.
bool make_cache_map(CUtensorMap* map, const void* base, int64_t nb, int kvh, int bs, int d);

// Whether the cuTensorMapEncodeTiled driver entry point was found.
bool have_tensor_map_encoder();

}  // namespace pa
