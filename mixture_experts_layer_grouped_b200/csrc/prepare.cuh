// Weight preparation: row-major bf16 matrices -> tile-major layout.
//
// A matrix of R rows (R % 128 == 0) and K columns (K % 64 == 0) is stored as
// tiles of 128 rows x 64 columns (16 KB), tile (rs, kt) at index
// rs * (K/64) + kt, each tile row-major inside.  One K-step of one 128-row
// weight slab is then a single contiguous 16 KB read, which keeps the HBM
// stream of the grouped GEMM sequential instead of 128 strided 128-byte pieces.
#pragma once

#include "common.cuh"

namespace moe {

// One block per tile; 256 threads move 1024 16-byte pieces.
__global__ void __launch_bounds__(256) tile_rows_kernel(const uint4* __restrict__ src,
                                                        uint4* __restrict__ dst, int64_t rows,
                                                        int K) {
  pdl_wait();
  pdl_trigger();
  const int kt_n = K / 64;
  const int64_t tile = blockIdx.x;
  const int64_t rs = tile / kt_n;
  const int kt = static_cast<int>(tile - rs * kt_n);
  const int64_t row_vecs = K / 8;  // 16-byte pieces per source row
  for (int i = threadIdx.x; i < 1024; i += 256) {
    const int r = i >> 3, c = i & 7;
    const int64_t grow = rs * 128 + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (grow < rows) v = src[grow * row_vecs + kt * 8 + c];
    dst[tile * 1024 + i] = v;
  }
}

}  // namespace moe
