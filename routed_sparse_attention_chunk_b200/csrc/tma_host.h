// Host helpers for TMA tensor maps (cuTensorMapEncodeTiled, reached through the
// runtime's driver entry point so the library does not link libcuda directly),
// and a per-device SM count cache.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace msa {

// 2D bf16 tensor map over a row-major [outer, inner] matrix whose rows are
// `row_bytes` apart, box = [box_outer rows, box_inner elements], 128-byte
// swizzle, out-of-bounds elements read as zero.  False if the driver rejects it.
bool make_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                       uint32_t box_inner, uint32_t box_outer);

// Streaming multiprocessors of the current device (cached).
int sm_count();

}  // namespace msa
