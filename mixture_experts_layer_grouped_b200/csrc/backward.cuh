// Backward of the bf16 layer: the combine and gate backward, the SwiGLU
// backward, and the weight copies the dgrad contractions read.  The
// contractions run on the grouped GEMM (grouped_gemm.cuh: fc2 mode with
// transposed weight copies, and fc1's backward form, which recomputes a and u
// and stores both); the weight gradients in wgrad.cuh; the host steps in
// backward_api.cuh.
//
//   combine backward:  dO[row(t, j)] = bf16(w[t, j] * dy[t]),
//                      g[t, j] = <dy[t], O[row(t, j)]>  (fp32),
//   gate backward:     w_j = rsf * s_j / S over the selected experts, so
//                      ds_j = rsf * (g_j / S - sum_i g_i s_i / S^2),
//                      dlogit_j = ds_j * s_j * (1 - s_j), zero elsewhere;
//   SwiGLU backward:   h = silu(a) * u:  da = dh * u * silu'(a),
//                      du = dh * silu(a), silu'(a) = s (1 + a (1 - s)), s = sigmoid(a).
// (TransformerEngine PR "DeepSeekV3Layer", Performance, "fused grouped MLP"
//  row: dGLU backward and the grouped GEMMs of the backward pass.)
#pragma once

#include "common.cuh"

namespace moe {

struct CombineBwdArgs {
  const __nv_bfloat16* dy;        // [T, H]
  const __nv_bfloat16* out_rows;  // [r_cap, H]: the forward's fc2 rows (O)
  const int32_t* token_row;       // [T * k]
  const int32_t* topk_idx;        // [T * k]
  const float* topk_w;            // [T * k]
  const float* logits;            // [T, E]: the forward's router logits
  __nv_bfloat16* dO;              // [r_cap, H]
  float* dgate;                   // [T * k]
  float* dlogits;                 // [T, E] or null
  __nv_bfloat16* dense_b;         // [T, ld_b]: dlogits as bf16 at column col_b, zeros to ld_b
  int T, H, k, E, col_b, ld_b;
  float rsf;
};

// A warp per token, eight tokens per 256-thread block: each lane takes every
// 32nd 16-byte vector of the row (8 bf16 columns), issuing the vector's k + 1
// loads (dy and the k fc2 rows) before its arithmetic, and the k dot products
// are reduced across the warp with shuffles (every lane ends with all of them).
template <int K>
__global__ void __launch_bounds__(256) combine_backward_kernel(CombineBwdArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int KM = K > 0 ? K : 32;
  const int lane = threadIdx.x & 31;
  const int t = static_cast<int>((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5);
  if (t >= a.T) return;
  const int kk = K > 0 ? K : a.k;
  int rows[KM];
  float ws[KM], part[KM];
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    rows[j] = j < kk ? __ldg(a.token_row + static_cast<int64_t>(t) * kk + j) : -1;
    ws[j] = j < kk ? __ldg(a.topk_w + static_cast<int64_t>(t) * kk + j) : 0.f;
    part[j] = 0.f;
  }
  const int vecs = a.H >> 3;
  const uint4* dy4 = reinterpret_cast<const uint4*>(a.dy + static_cast<int64_t>(t) * a.H);
  auto body = [&](int v, const uint4& draw, const uint4 (&o)[KM]) {
    const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&draw);
    float d[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(d2[q]);
      d[2 * q] = f.x;
      d[2 * q + 1] = f.y;
    }
#pragma unroll
    for (int j = 0; j < KM; ++j) {
      if (j >= kk || rows[j] < 0) continue;
      const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o[j]);
      float sdot = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(o2[q]);
        sdot = fmaf(d[2 * q], f.x, sdot);
        sdot = fmaf(d[2 * q + 1], f.y, sdot);
      }
      part[j] += sdot;
      uint4 w;
      __nv_bfloat162* w2 = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        w2[q] = __floats2bfloat162_rn(ws[j] * d[2 * q], ws[j] * d[2 * q + 1]);
      reinterpret_cast<uint4*>(a.dO + static_cast<int64_t>(rows[j]) * a.H)[v] = w;
    }
  };
  for (int v = lane; v < vecs; v += 32) {
    const uint4 draw = __ldg(dy4 + v);
    uint4 o[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j)
      if (j < kk && rows[j] >= 0)
        o[j] = __ldg(reinterpret_cast<const uint4*>(a.out_rows + static_cast<int64_t>(rows[j]) * a.H) + v);
    body(v, draw, o);
  }
  // g[t, j]: every lane ends with the warp's sums
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    if (j >= kk) break;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], off);
  }
#pragma unroll
  for (int j = 0; j < KM; ++j)
    if (j < kk && lane == j) a.dgate[static_cast<int64_t>(t) * kk + j] = part[j];
  // gate backward: the token's dlogits (fp32, optional) and their bf16 copy in
  // the dense GEMM's operand row, zeros elsewhere
  const float* lg = a.logits + static_cast<int64_t>(t) * a.E;
  const int32_t* ti = a.topk_idx + static_cast<int64_t>(t) * kk;
  float S = 0.f, gs = 0.f;
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    if (j >= kk) break;
    const int e = __ldg(ti + j);
    if (e < 0 || e >= a.E) continue;
    const float sg = 1.0f / (1.0f + expf(-__ldg(lg + e)));
    S += sg;
    gs += part[j] * sg;
  }
  __nv_bfloat16* brow = a.dense_b + static_cast<int64_t>(t) * a.ld_b;
  for (int e = lane; e < a.ld_b - a.col_b; e += 32) {
    float dl = 0.f;
    if (e < a.E) {
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        if (j >= kk) break;
        if (__ldg(ti + j) != e) continue;
        const float sg = 1.0f / (1.0f + expf(-__ldg(lg + e)));
        const float ds = a.rsf * (part[j] / S - gs / (S * S));
        dl = ds * sg * (1.0f - sg);
      }
      if (a.dlogits) a.dlogits[static_cast<int64_t>(t) * a.E + e] = dl;
    }
    brow[a.col_b + e] = __float2bfloat16_rn(dl);
  }
}

// SwiGLU backward in place: row r of z holds [a | u] (n columns each, row
// length ld), the fc1 outputs recomputed by the backward form of the fc1
// kernel; with dh [rows, n] it becomes [da | du], and h = bf16(silu(a) u) goes
// to h_out [rows, n] when h_out is given (the fc2 weight gradient's operand).
// Rows with row_token < 0 (segment pads) are zeroed in z and h_out; a null
// row_token means every row holds a token, and rows_used (when given) bounds the
// rows.  Eight columns per thread and vector; each thread reads its a, u, dh
// before writing the same places.
__global__ void __launch_bounds__(256) swiglu_backward_kernel(
    __nv_bfloat16* __restrict__ z, int64_t ld, const __nv_bfloat16* __restrict__ dh,
    __nv_bfloat16* __restrict__ h_out, const int32_t* __restrict__ row_token,
    const int32_t* __restrict__ rows_used, int64_t rows, int n) {
  pdl_wait();
  pdl_trigger();
  const int64_t nrows = rows_used ? __ldg(rows_used) : rows;
  const int vpr = n >> 3;
  const int64_t total = nrows * vpr;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / vpr;
    const int v = static_cast<int>(i - r * vpr);
    uint4 da4 = make_uint4(0, 0, 0, 0), du4 = make_uint4(0, 0, 0, 0), h4 = make_uint4(0, 0, 0, 0);
    uint4* za = reinterpret_cast<uint4*>(z + r * ld) + v;
    uint4* zu = reinterpret_cast<uint4*>(z + r * ld + n) + v;
    if (!row_token || __ldg(row_token + r) >= 0) {
      const uint4 ar = *za, ur = *zu;
      const uint4 hr = __ldg(reinterpret_cast<const uint4*>(dh + r * n) + v);
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&ar);
      const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&ur);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&hr);
      __nv_bfloat162* da2 = reinterpret_cast<__nv_bfloat162*>(&da4);
      __nv_bfloat162* du2 = reinterpret_cast<__nv_bfloat162*>(&du4);
      __nv_bfloat162* hh2 = reinterpret_cast<__nv_bfloat162*>(&h4);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 av = __bfloat1622float2(a2[q]), uv = __bfloat1622float2(u2[q]),
                     gv = __bfloat1622float2(g2[q]);
        const float s0 = 1.0f / (1.0f + expf(-av.x)), s1 = 1.0f / (1.0f + expf(-av.y));
        const float d0 = s0 * (1.0f + av.x * (1.0f - s0)), d1 = s1 * (1.0f + av.y * (1.0f - s1));
        da2[q] = __floats2bfloat162_rn(gv.x * uv.x * d0, gv.y * uv.y * d1);
        du2[q] = __floats2bfloat162_rn(gv.x * av.x * s0, gv.y * av.y * s1);
        hh2[q] = __floats2bfloat162_rn(av.x * s0 * uv.x, av.y * s1 * uv.y);
      }
    }
    *za = da4;
    *zu = du4;
    if (h_out) reinterpret_cast<uint4*>(h_out + r * n)[v] = h4;
  }
}

// Weight preparation for the backward: a tile-major matrix (tiles of 128 rows
// x 64 columns, as the forward's prepared weights) whose element (r, c) is
// taken, transposed, from up to three row-major bf16 sources laid side by side
// along c: for the segment s holding column c, source row c - start_s and
// source column r % rows_per_group of group r / rows_per_group (each group a
// block of group_stride elements).  Columns past the last segment are zero.
// A block moves one 64 x 64 square through shared memory, so that both the
// reads (along a source row) and the writes (along a tile row) are coalesced.
struct TransposeSeg {
  const __nv_bfloat16* src;
  int64_t group_stride;  // elements between consecutive groups (experts)
  int ld;                // source row length (elements)
  int start, width;      // destination columns [start, start + width)
};
struct TransposeArgs {
  TransposeSeg seg[3];
  int nseg;
  __nv_bfloat16* dst;
  int64_t rows;          // destination rows (a multiple of 128)
  int cols;              // destination columns (a multiple of 64)
  int rows_per_group;    // a multiple of 64
};

__global__ void __launch_bounds__(256) transpose_tiles_kernel(TransposeArgs a) {
  __shared__ __nv_bfloat16 sq[64][66];
  const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int c0 = blockIdx.y * 64;
  const int64_t grp = r0 / a.rows_per_group, rl0 = r0 - grp * a.rows_per_group;
  for (int cc = ty; cc < 64; cc += 4) {
    const int c = c0 + cc;
    __nv_bfloat16 v = __float2bfloat16_rn(0.f);
    for (int s = 0; s < a.nseg; ++s) {
      const TransposeSeg& g = a.seg[s];
      if (c >= g.start && c < g.start + g.width)
        v = g.src[grp * g.group_stride + static_cast<int64_t>(c - g.start) * g.ld + rl0 + tx];
    }
    sq[cc][tx] = v;
  }
  __syncthreads();
  for (int rr = ty; rr < 64; rr += 4) {
    const int64_t r = r0 + rr;
    const int c = c0 + tx;
    const int64_t tile = (r >> 7) * (a.cols >> 6) + (c >> 6);
    a.dst[tile * 8192 + (r & 127) * 64 + (c & 63)] = sq[tx][rr];
  }
}

}  // namespace moe
