// TMA tensor maps of the tensor-core forward kernels: q, k, alpha, v (and o)
// seen as [rows, H * 128] bf16 matrices, 64 x 64 boxes, 128-byte swizzle.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace kda {

struct TcMaps {
    CUtensorMap q, k, a, v, o;
};

// out may be null (segment summaries write no output): its map then reuses v's.
// False if the driver entry point is missing or a map is rejected.
bool make_tc_maps(TcMaps* m, const void* q, const void* k, const void* v, const void* alpha,
                  const void* out, int64_t rows, int H);

}  // namespace kda
