// Host-side helpers shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace pa {

constexpr int kMaxDevices = 64;

// SM count of device `dev` (cached), 0 on error.
int device_sms(int dev);

// Tensor map of a cache pool [nb][kvh][bs][d] of 16-bit elements: box
// {64 elements = 128 B, min(bs, 16) rows, 1, 1}, 128-byte swizzle.
bool make_cache_map(CUtensorMap* map, const void* base, int64_t nb, int kvh, int bs, int d);

// Whether the cuTensorMapEncodeTiled driver entry point was found.
bool have_tensor_map_encoder();

}  // namespace pa
