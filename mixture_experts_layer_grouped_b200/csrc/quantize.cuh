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
  pdl_wait();
  pdl_trigger();
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
  pdl_wait();
  pdl_trigger();
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
  pdl_wait();
  pdl_trigger();
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
      if (a.dst_codes) warp_copy_row(d, s, vecs, lane);
      for (int w = lane; w < W; w += 32)
        *reinterpret_cast<uint32_t*>(a.dst_scales + sf_offset(r, 4 * w, KB)) =
            *reinterpret_cast<const uint32_t*>(a.src_scales + sf_offset(t, 4 * w, KB));
    } else {
      if (a.dst_codes) warp_copy_row(d, nullptr, vecs, lane);
      for (int w = lane; w < W; w += 32)
        *reinterpret_cast<uint32_t*>(a.dst_scales + sf_offset(r, 4 * w, KB)) = 0u;
    }
  }
}

}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------
// NVFP4 (sglang PR "Mistral Large 3 NVFP4 TRTLLM MoE support", Modifications:
// W4A4 NVFP4): e2m1 elements, a ue4m3 scale per 16 K elements and an fp32
// global encode scale g = 2688 / amax of the tensor.  Codes are packed two per
// byte (element 2i in the low nibble); scales use the MMA scale layout with
// KB = cols / 16 blocks per row.
// ---------------------------------------------------------------------------

// amax per group: out[blockIdx.y] = max |in[blockIdx.y * group_elems + i]|
// over a group of group_elems bf16 values (group_elems % 8 == 0; out must start
// at zero).  Each block reduces a strided slice and issues one atomic.
__global__ void __launch_bounds__(256) amax_groups_kernel(const __nv_bfloat16* __restrict__ in,
                                                          int64_t group_elems, float* out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[8];
  const int64_t vecs = group_elems / 8;
  const uint4* base = reinterpret_cast<const uint4*>(in + blockIdx.y * group_elems);
  float m = 0.f;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < vecs;
       v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 raw = base[v];
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p2[i]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
    if (m > 0.f) atomic_max_nonneg(out + blockIdx.y, m);
  }
}

// In place: amax -> global encode scale.
__global__ void amax_to_global_kernel(float* v, int n) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) v[i] = nv_global_scale(v[i]);
}

__device__ __forceinline__ void load_bf16x16(const __nv_bfloat16* src, float (&v)[16]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint4 raw = s[q];
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p2[i]);
      v[q * 8 + 2 * i] = f.x;
      v[q * 8 + 2 * i + 1] = f.y;
    }
  }
}

// One thread per 16-element block of a row-major bf16 [rows, cols] matrix,
// global scale g[r / rows_per_group] (rows_per_group 0: g[0]).  tiled != 0
// writes codes tile-major (128 rows x 128 bytes = 256 elements per tile).
__global__ void __launch_bounds__(256) quantize_nvfp4_kernel(
    const __nv_bfloat16* __restrict__ in, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, int64_t rows, int cols, const float* __restrict__ g,
    int64_t rows_per_group, int tiled) {
  pdl_wait();
  pdl_trigger();
  const int KB = cols / 16;
  const int64_t blk = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (blk >= rows * KB) return;
  const int64_t r = blk / KB;
  const int kb = static_cast<int>(blk - r * KB);
  float v[16];
  load_bf16x16(in + r * cols + kb * 16, v);
  const float gs = g[rows_per_group > 0 ? r / rows_per_group : 0];
  uint32_t packed[2];
  const uint32_t sb = nv_quantize_block16(v, gs, packed);
  uint8_t* dst;
  if (tiled) {
    const int64_t tile = (r >> 7) * (cols >> 8) + (kb >> 4);
    dst = codes + tile * 16384 + (r & 127) * 128 + (kb & 15) * 8;
  } else {
    dst = codes + r * (cols / 2) + kb * 8;
  }
  *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
  scales[sf_offset(r, kb, KB)] = static_cast<uint8_t>(sb);
}

// NVFP4 quantization of the fc2 input h (bf16, expert-major rows), over the
// rows that hold a token: valid row v (in expert order) is row
// offsets[e] + v - cnt_prefix[e] of expert e, whose global scale is g_h[e].
// Pad rows are left as they are (their outputs are masked).  One warp per
// row.  `dense` > 0 quantizes `dense` token-order rows with g_h[0] instead.
__global__ void __launch_bounds__(256) quantize_h_nvfp4_kernel(
    const __nv_bfloat16* __restrict__ h, uint8_t* __restrict__ codes,
    uint8_t* __restrict__ scales, int cols, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ counts, int E, const float* __restrict__ g_h, int dense) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t s_cpre[1025];
  const int KB = cols / 16;
  int64_t n_rows = dense;
  if (!dense) {
    block_scan_padded(counts, E, 1, s_cpre);
    n_rows = s_cpre[E];
  }
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t vr = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       vr < n_rows; vr += warps) {
    int64_t r = vr;
    int e = 0;
    if (!dense) {
      int lo = 0, hi = E;  // s_cpre[lo] <= vr < s_cpre[lo + 1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_cpre[mid] <= vr) lo = mid; else hi = mid;
      }
      e = lo;
      r = __ldg(offsets + e) + (vr - s_cpre[e]);
    }
    const float g = __ldg(g_h + e);
    for (int kb = lane; kb < KB; kb += 32) {
      float v[16];
      load_bf16x16(h + r * cols + kb * 16, v);
      uint32_t packed[2];
      const uint32_t sb = nv_quantize_block16(v, g, packed);
      *reinterpret_cast<uint2*>(codes + r * (cols / 2) + kb * 8) =
          make_uint2(packed[0], packed[1]);
      scales[sf_offset(r, kb, KB)] = static_cast<uint8_t>(sb);
    }
  }
}

// One-round form of the block-scaled gathers (MXFP8: row_bytes = H, KB = H/32;
// NVFP4: row_bytes = H/2, KB = H/16) for rows of at most 32 * MAXV vectors and
// 256 scale words: all loads of a row, codes and scale words, are issued before
// its first store, and the next row's token index is read one row ahead, so a
// warp waits about one memory latency per row instead of one per 8 vectors
// and one per 32 scale words.  (Plain loads: the compiler may not move them
// past the stores, which could alias, so all of them stay in flight at once;
// read-only loads let it sink each load to its store and serialize the row.)
template <int MAXV>
__global__ void __launch_bounds__(256) permute_gather_bs_kernel(GatherMxArgs a, int row_bytes,
                                                                int KB) {
  constexpr int MAXW = 8;
  pdl_wait();
  pdl_trigger();
  const int rows = a.offsets[a.E];
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  const int vecs = row_bytes >> 4, W = KB / 4;
  int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  int t = r < rows ? a.row_token[r] : -1;
  for (; r < rows; r += warps) {
    const int t_next = r + warps < rows ? a.row_token[r + warps] : -1;
    const uint4* src = (t >= 0 && a.dst_codes)
                           ? reinterpret_cast<const uint4*>(a.src_codes + static_cast<int64_t>(t) * row_bytes)
                           : nullptr;
    uint4 buf[MAXV];
    uint32_t sw[MAXW];
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = i * 32 + lane;
      buf[i] = (src && v < vecs) ? src[v] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < MAXW; ++i) {
      const int w = i * 32 + lane;
      sw[i] = (t >= 0 && w < W)
                  ? *reinterpret_cast<const uint32_t*>(a.src_scales + sf_offset(t, 4 * w, KB))
                  : 0u;
    }
    if (a.dst_codes) {
      uint4* d = reinterpret_cast<uint4*>(a.dst_codes + static_cast<int64_t>(r) * row_bytes);
#pragma unroll
      for (int i = 0; i < MAXV; ++i)
        if (i * 32 + lane < vecs) d[i * 32 + lane] = buf[i];
    }
#pragma unroll
    for (int i = 0; i < MAXW; ++i) {
      const int w = i * 32 + lane;
      if (w < W) *reinterpret_cast<uint32_t*>(a.dst_scales + sf_offset(r, 4 * w, KB)) = sw[i];
    }
    t = t_next;
  }
}

// Expert-major gather of NVFP4 rows (packed codes, H/2 bytes per row) and
// their scale words (4 blocks of 16 per 32-bit word).
__global__ void __launch_bounds__(256) permute_gather_nv_kernel(GatherMxArgs a) {
  pdl_wait();
  pdl_trigger();
  const int rows = a.offsets[a.E];
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  const int row_bytes = a.H / 2;
  const int vecs = row_bytes >> 4;
  const int KB = a.H / 16, W = KB / 4;
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int t = a.row_token[r];
    uint4* d = reinterpret_cast<uint4*>(a.dst_codes + static_cast<int64_t>(r) * row_bytes);
    if (t >= 0) {
      const uint4* s =
          reinterpret_cast<const uint4*>(a.src_codes + static_cast<int64_t>(t) * row_bytes);
      if (a.dst_codes) warp_copy_row(d, s, vecs, lane);
      for (int w = lane; w < W; w += 32)
        *reinterpret_cast<uint32_t*>(a.dst_scales + sf_offset(r, 4 * w, KB)) =
            *reinterpret_cast<const uint32_t*>(a.src_scales + sf_offset(t, 4 * w, KB));
    } else {
      if (a.dst_codes) warp_copy_row(d, nullptr, vecs, lane);
      for (int w = lane; w < W; w += 32)
        *reinterpret_cast<uint32_t*>(a.dst_scales + sf_offset(r, 4 * w, KB)) = 0u;
    }
  }
}

}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------
// NVFP4 quantize and permute in one pass (the one-call forward's path): each
// token's row of x is read once, quantized once (the per-block arithmetic of
// quantize_nvfp4_kernel), and its codes and scales are written to every
// expert-major row the token feeds (token_row), and to token order when the
// shared expert needs them.  Expert-major rows without a token (segment pads)
// get zero codes and scales, as the separate permute gives them.
// ---------------------------------------------------------------------------
struct QScatterArgs {
  const __nv_bfloat16* x;     // [T, H]
  const int32_t* token_row;   // [T * k]
  const int32_t* row_token;   // [r_cap]
  const int32_t* offsets;     // [E + 1]: offsets[E] = expert-major rows in use
  uint8_t* rows;              // [r_cap, H / 2] packed e2m1 codes
  uint8_t* rows_sf;           // MMA scale layout over r_cap rows
  uint8_t* xq;                // [T, H / 2] codes in token order, or null
  uint8_t* xq_sf;             // their scales, or null
  const float* g;             // global encode scale of x
  int T, H, k, E;
};

// Work items of one token and 64 consecutive 16-element blocks of its row, two
// blocks per lane (16 code bytes, one vector store per destination row), so
// that short batches still spread over every SM; then a warp per expert-major
// row zeroes the pads.  H % 256 == 0, so the block count KB is a multiple of
// 16 and the two lanes of a 4-block scale word are both in range or both past it.
__global__ void __launch_bounds__(256) quantize_scatter_nvfp4_kernel(QScatterArgs a) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int KB = a.H / 16, row_bytes = a.H / 2, nch = (KB + 63) / 64;
  const int64_t warp0 = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const float g = __ldg(a.g);
  const int64_t items = static_cast<int64_t>(a.T) * nch;
  for (int64_t it = warp0; it < items; it += warps) {
    const int64_t t = it / nch;
    const int kb = static_cast<int>(it - t * nch) * 64 + 2 * lane;  // this lane's first block
    const bool valid = kb < KB;
    int dst = -1;  // lane j < k: row of (t, j)
    if (lane < a.k) dst = __ldg(a.token_row + t * a.k + lane);
    uint4 code = make_uint4(0, 0, 0, 0);
    uint32_t sc2 = 0;  // the two blocks' scale bytes
    if (valid) {
      const __nv_bfloat16* src = a.x + t * a.H + static_cast<int64_t>(kb) * 16;
      float v0[16], v1[16];
      load_bf16x16(src, v0);
      load_bf16x16(src + 16, v1);
      uint32_t p0[2], p1[2];
      const uint32_t s0 = nv_quantize_block16(v0, g, p0);
      const uint32_t s1 = nv_quantize_block16(v1, g, p1);
      code = make_uint4(p0[0], p0[1], p1[0], p1[1]);
      sc2 = (s0 & 0xFFu) | ((s1 & 0xFFu) << 8);
    }
    // even lanes hold blocks kb .. kb + 3 of a scale word (kb % 4 == 0)
    const uint32_t word = sc2 | (__shfl_down_sync(0xffffffffu, sc2, 1) << 16);
    for (int j = 0; j <= a.k; ++j) {
      int64_t r;
      uint8_t *codes, *scales;
      if (j < a.k) {
        r = __shfl_sync(0xffffffffu, dst, j);
        if (r < 0) continue;          // an entry the permute dropped (bad expert index)
        codes = a.rows;
        scales = a.rows_sf;
      } else {
        if (a.xq == nullptr) break;   // token order only for the shared expert
        r = t;
        codes = a.xq;
        scales = a.xq_sf;
      }
      if (!valid) continue;
      *reinterpret_cast<uint4*>(codes + r * row_bytes + static_cast<int64_t>(kb) * 8) = code;
      if ((lane & 1) == 0)
        *reinterpret_cast<uint32_t*>(scales + sf_offset(r, kb, KB)) = word;
    }
  }
  // pad rows of the expert-major layout: zero codes and scale words
  const int rows_used = __ldg(a.offsets + a.E);
  const int W = KB / 4;
  for (int64_t r = warp0; r < rows_used; r += warps) {
    if (__ldg(a.row_token + r) >= 0) continue;
    uint4* cd = reinterpret_cast<uint4*>(a.rows + r * row_bytes);
    for (int v = lane; v < row_bytes / 16; v += 32) cd[v] = make_uint4(0, 0, 0, 0);
    for (int w = lane; w < W; w += 32)
      *reinterpret_cast<uint32_t*>(a.rows_sf + sf_offset(r, 4 * w, KB)) = 0u;
  }
}

}  // namespace moe
