// Block-scaled quantization kernels.
//
// MXFP8 (TransformerEngine PR "DeepSeekV3Layer", Performance section, MXFP8
// rows): e4m3 elements with one e8m0 scale per 32 consecutive K elements.  The
// scale of a block with absolute maximum amax is 2^(floor(log2 amax) - 8)
// (biased exponent clamped to [0, 254], 127 for an all-zero block), and each
// element is v / scale rounded to nearest-even e4m3, saturating at 448.
//
// Codes are row-major (one byte per element); scales use the MMA scale layout
// (sf_offset): 128-row x 4-block chunks of 512 bytes.
#pragma once

#include "common.cuh"

namespace moe {

// One thread per 32-element block of a row-major bf16 [rows, cols] matrix.
// Codes go to codes[r * cols + k]; scales to scales[sf_offset(r, k/32, cols/32)].
__global__ void __launch_bounds__(256) quantize_mxfp8_rows_kernel(
    const __nv_bfloat16* __restrict__ in, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, int64_t rows, int cols) {
  const int KB = cols / 32;
  const int64_t blk = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (blk >= rows * KB) return;
  const int64_t r = blk / KB;
  const int kb = static_cast<int>(blk - r * KB);
  const uint4* src = reinterpret_cast<const uint4*>(in + r * cols + kb * 32);
  float v[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 raw = src[q];
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p2[i]);
      v[q * 8 + 2 * i] = f.x;
      v[q * 8 + 2 * i + 1] = f.y;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t code = mx_scale_code(amax);
  const float inv = mx_inv_scale(code);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = static_cast<uint32_t>(to_e4m3(v[4 * i] * inv)) |
           (static_cast<uint32_t>(to_e4m3(v[4 * i + 1] * inv)) << 8) |
           (static_cast<uint32_t>(to_e4m3(v[4 * i + 2] * inv)) << 16) |
           (static_cast<uint32_t>(to_e4m3(v[4 * i + 3] * inv)) << 24);
  uint4* dst = reinterpret_cast<uint4*>(codes + r * cols + kb * 32);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  scales[sf_offset(r, kb, KB)] = static_cast<uint8_t>(code);
}

// Weights: the same quantization, with codes written tile-major (128 rows x
// 128 bytes per tile, tile (r/128, k/128) at index (r/128)*(cols/128) + k/128).
__global__ void __launch_bounds__(256) quantize_mxfp8_tiles_kernel(
    const __nv_bfloat16* __restrict__ in, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, int64_t rows, int cols) {
  const int KB = cols / 32;
  const int64_t blk = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (blk >= rows * KB) return;
  const int64_t r = blk / KB;
  const int kb = static_cast<int>(blk - r * KB);
  const uint4* src = reinterpret_cast<const uint4*>(in + r * cols + kb * 32);
  float v[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 raw = src[q];
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p2[i]);
      v[q * 8 + 2 * i] = f.x;
      v[q * 8 + 2 * i + 1] = f.y;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t code = mx_scale_code(amax);
  const float inv = mx_inv_scale(code);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = static_cast<uint32_t>(to_e4m3(v[4 * i] * inv)) |
           (static_cast<uint32_t>(to_e4m3(v[4 * i + 1] * inv)) << 8) |
           (static_cast<uint32_t>(to_e4m3(v[4 * i + 2] * inv)) << 16) |
           (static_cast<uint32_t>(to_e4m3(v[4 * i + 3] * inv)) << 24);
  const int64_t tile = (r >> 7) * (cols >> 7) + (kb >> 2);
  uint4* dst = reinterpret_cast<uint4*>(codes + tile * 16384 + (r & 127) * 128 + (kb & 3) * 32);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  scales[sf_offset(r, kb, KB)] = static_cast<uint8_t>(code);
}

// Expert-major gather of MXFP8 rows: codes (one warp per destination row,
// 16-byte vectors) and the scale words of the row (4 consecutive k-blocks share
// one 32-bit word of the MMA layout).  Pad rows get zero codes and zero words.
struct GatherMxArgs {
  const uint8_t* src_codes;   // [T, H]
  const uint8_t* src_scales;  // MMA layout, T rows
  uint8_t* dst_codes;         // [r_cap, H]
  uint8_t* dst_scales;        // MMA layout, r_cap rows
  const int32_t* row_token;
  const int32_t* offsets;
  int E, H;
};

__global__ void __launch_bounds__(256) permute_gather_mx_kernel(GatherMxArgs a) {
  const int rows = a.offsets[a.E];
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  const int vecs = a.H >> 4;
  const int KB = a.H / 32, W = KB / 4;
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int t = a.row_token[r];
    uint4* d = reinterpret_cast<uint4*>(a.dst_codes + static_cast<int64_t>(r) * a.H);
    if (t >= 0) {
      const uint4* s = reinterpret_cast<const uint4*>(a.src_codes + static_cast<int64_t>(t) * a.H);
      for (int v = lane; v < vecs; v += 32) d[v] = __ldg(s + v);
      for (int w = lane; w < W; w += 32)
        *reinterpret_cast<uint32_t*>(a.dst_scales + sf_offset(r, 4 * w, KB)) =
            *reinterpret_cast<const uint32_t*>(a.src_scales + sf_offset(t, 4 * w, KB));
    } else {
      for (int v = lane; v < vecs; v += 32) d[v] = make_uint4(0, 0, 0, 0);
      for (int w = lane; w < W; w += 32)
        *reinterpret_cast<uint32_t*>(a.dst_scales + sf_offset(r, 4 * w, KB)) = 0u;
    }
  }
}

}  // namespace moe
