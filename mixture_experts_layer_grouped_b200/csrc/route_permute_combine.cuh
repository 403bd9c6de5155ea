// Memory-bound steps of the layer: grouped top-k selection, the permute into
// padded expert-major order (histogram, scan, stable ranks, row gather) and
// the gate-weighted combine.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kPermTile = 256;  // (t, j) entries per histogram / rank tile
constexpr int kMaxExpertsPerm = 1024;

// ---------------------------------------------------------------------------
// Selection: one warp per token.
// s = sigmoid(logit), b = s + bias; group score = sum of the two largest b in
// each contiguous group of E/G experts; keep the topk_group best groups; pick
// the top_k largest b among their experts (ties to the lower index, listed by
// b descending); gate_j = s_j / sum_j s_j * rsf.
// (TransformerEngine PR "DeepSeekV3Layer", Description, DeepSeekV3MoE bullet.)
// ---------------------------------------------------------------------------
constexpr int kSelMaxPerLane = 32;  // E <= 1024
constexpr int kMaxSplits = 4;       // router GEMM K splits summed by the selection
constexpr int kSelWarps = 4;

struct SelArgs {
  const float* logits;    // [T, E] (when n_splits == 0)
  const float* partials;  // [n_splits, T, E] router GEMM partial sums (n_splits > 0)
  float* logits_out;      // [T, E] sum of the partials, in split order (n_splits > 0)
  int n_splits;
  const float* bias;      // [E]
  int32_t* topk_idx;    // [T, k]
  float* topk_w;        // [T, k]
  int T, E, G, g, k;
  float rsf;
  uint32_t gs_magic;  // ceil(2^32 / (E / G)): e / (E / G) == umulhi(e, gs_magic) for e < 1024
};

// Warp arg-max of (v, i): larger v wins, ties to the smaller i.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
  }
}

template <int PER>
__global__ void __launch_bounds__(kSelWarps * 32) route_select_kernel(SelArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sb[kSelWarps][kSelMaxPerLane * 32];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kSelWarps + w;
  if (t >= a.T) return;
  const int gs = a.E / a.G;
  const int64_t row = static_cast<int64_t>(t) * a.E;
  const int64_t split_stride = static_cast<int64_t>(a.T) * a.E;

  float s[PER], b[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    if (e < a.E) {
      float l;
      if (a.n_splits > 0) {
        // fixed summation order over the K splits (at most kMaxSplits): deterministic
        // logits; all partial loads are issued before the additions
        float part[kMaxSplits];
#pragma unroll
        for (int sp = 0; sp < kMaxSplits; ++sp)
          part[sp] = sp < a.n_splits ? a.partials[sp * split_stride + row + e] : 0.f;
        l = part[0];
#pragma unroll
        for (int sp = 1; sp < kMaxSplits; ++sp)
          if (sp < a.n_splits) l += part[sp];
        a.logits_out[row + e] = l;
      } else {
        l = a.logits[row + e];
      }
      s[i] = 1.0f / (1.0f + expf(-l));
      b[i] = s[i] + a.bias[e];
      sb[w][e] = b[i];
    } else {
      s[i] = 0.f;
      b[i] = -INFINITY;
    }
  }
  __syncwarp();
  // group scores: lpg = 32 / G lanes per group when G divides 32 (else one),
  // each scanning a strided share of the group's experts for its two largest
  // values, merged across the group's lanes by shuffles; group q's score ends
  // in lane q
  const int lpg = (32 % a.G == 0) ? 32 / a.G : 1;
  float gscore = -INFINITY;
  {
    const int q = lane / lpg, sub = lane - q * lpg;
    float m1 = -INFINITY, m2 = -INFINITY;
    if (q < a.G) {
      for (int e = q * gs + sub; e < (q + 1) * gs; e += lpg) {
        const float v = sb[w][e];
        if (v > m1) { m2 = m1; m1 = v; } else if (v > m2) { m2 = v; }
      }
    }
    for (int o = 1; o < lpg; o <<= 1) {  // top-2 of two top-2 pairs (a multiset)
      const float o1 = __shfl_xor_sync(0xffffffffu, m1, o);
      const float o2 = __shfl_xor_sync(0xffffffffu, m2, o);
      const float hi = fmaxf(m1, o1);
      m2 = fmaxf(fminf(m1, o1), fmaxf(m2, o2));
      m1 = hi;
    }
    const float s_q = m1 + m2;  // in every lane of group q
    gscore = __shfl_sync(0xffffffffu, s_q, (lane < a.G ? lane : 0) * lpg);
    if (lane >= a.G) gscore = -INFINITY;
  }
  // keep the best g groups
  uint32_t keep = 0;
  float gv = gscore;
  for (int r = 0; r < a.g; ++r) {
    float v = gv;
    int i = (lane < a.G) ? lane : 1 << 30;
    warp_argmax(v, i);
    keep |= 1u << i;
    if (lane == i) gv = -INFINITY;
  }
  // eligible keys
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    if (e >= a.E || !((keep >> __umulhi(static_cast<uint32_t>(e), a.gs_magic)) & 1u))
      b[i] = -INFINITY;
  }
  float sel_s = 0.f;
  int sel_e = 0;
  float ssum = 0.f;
  for (int r = 0; r < a.k; ++r) {
    float v = -INFINITY;
    int idx = 1 << 30;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      if (b[i] > v || (b[i] == v && e < idx)) { v = b[i]; idx = e; }
    }
    warp_argmax(v, idx);
    // the owner lane removes it and broadcasts s
    float sv = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (lane + 32 * i == idx) { sv = s[i]; b[i] = -INFINITY; }
    sv = __shfl_sync(0xffffffffu, sv, idx & 31);
    ssum += sv;
    if (lane == r) { sel_s = sv; sel_e = idx; }
  }
  if (lane < a.k) {
    a.topk_idx[static_cast<int64_t>(t) * a.k + lane] = sel_e;
    a.topk_w[static_cast<int64_t>(t) * a.k + lane] = sel_s / ssum * a.rsf;
  }
}

// ---------------------------------------------------------------------------
// Permute.
//   hist:  per tile of kPermTile entries, per-expert counts;
//   scan:  per-expert running bases across tiles, counts, padded offsets,
//          -1 for pad rows and rows past the last segment;
//   rank:  stable slot of every (t, j) (ascending t inside each expert);
//   gather: dst[r] = src[row_token[r]] or zeros.
// (TransformerEngine PR "DeepSeekV3Layer", Performance, "NCCL EP local
//  permute": expert-major staging buffer with zero-filled padding.)
// ---------------------------------------------------------------------------
struct PermArgs {
  const int32_t* topk_idx;  // [T*k]
  int32_t* hist;            // [ntiles, E] workspace
  int32_t* counts;          // [E]
  int32_t* offsets;         // [E+1]
  int32_t* row_token;       // [r_cap]
  int32_t* token_row;       // [T*k]
  int32_t* status;
  int n, k, E, P, r_cap, ntiles;
};

__global__ void __launch_bounds__(256) permute_hist_kernel(PermArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t h[];
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) h[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kPermTile;
  for (int i = threadIdx.x; i < kPermTile; i += blockDim.x) {
    const int f = base + i;
    if (f < a.n) {
      const int e = a.topk_idx[f];
      if (e >= 0 && e < a.E) atomicAdd(&h[e], 1);
      else set_status(a.status, MOE_ERR_CAPACITY);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x)
    a.hist[static_cast<int64_t>(e) * a.ntiles + blockIdx.x] = h[e];
}

// A warp per expert: exclusive scan of the expert's tile counts (hist row
// [e][0..ntiles), contiguous) into tile bases, and counts[e].
__global__ void __launch_bounds__(256) permute_scan_kernel(PermArgs a) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (e >= a.E) return;
  int32_t* row = a.hist + static_cast<int64_t>(e) * a.ntiles;
  int run = 0;
  for (int b0 = 0; b0 < a.ntiles; b0 += 32) {
    const int b = b0 + lane;
    const int v = (b < a.ntiles) ? row[b] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (b < a.ntiles) row[b] = run + incl - v;  // the tile's base rank for this expert
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) a.counts[e] = run;
}

// One block per tile.  Every block derives the padded segment offsets; block
// 0 publishes them; all blocks mark pad rows and rows past the last segment
// with -1 (a grid-stride pass over r_cap); then warp 0 walks the tile's
// entries in order and assigns stable slots.
__global__ void __launch_bounds__(256) permute_rank_kernel(PermArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t s_off[kMaxExpertsPerm + 1];
  __shared__ int32_t run[kMaxExpertsPerm];
  block_scan_padded(a.counts, a.E, a.P, s_off);
  const int tid = threadIdx.x;
  if (blockIdx.x == 0)
    for (int e = tid; e <= a.E; e += blockDim.x) a.offsets[e] = s_off[e];
  const int total = s_off[a.E];
  const int64_t gstride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * blockDim.x + tid; r < a.r_cap; r += gstride) {
    bool pad = r >= total;
    if (!pad) {
      int lo = 0, hi = a.E;  // s_off[lo] <= r < s_off[lo + 1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_off[mid] <= r) lo = mid; else hi = mid;
      }
      pad = (r - s_off[lo]) >= a.counts[lo];
    }
    if (pad) a.row_token[r] = -1;
  }
  if (tid >= 32) return;
  const int lane = tid;
  for (int e = lane; e < a.E; e += 32)
    run[e] = s_off[e] + a.hist[static_cast<int64_t>(e) * a.ntiles + blockIdx.x];
  const int base = blockIdx.x * kPermTile;
  int ev[kPermTile / 32];
#pragma unroll
  for (int c = 0; c < kPermTile / 32; ++c) {
    const int f = base + c * 32 + lane;
    int e = -1;
    if (f < a.n) {
      e = a.topk_idx[f];
      if (e < 0 || e >= a.E) e = -1;
    }
    ev[c] = e;
  }
  __syncwarp();
#pragma unroll
  for (int c = 0; c < kPermTile / 32; ++c) {
    const int f = base + c * 32 + lane;
    const int e = ev[c];
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int slot = run[e] + __popc(peers & ((1u << lane) - 1u));
      a.token_row[f] = slot;
      a.row_token[slot] = f / a.k;
    } else if (f < a.n) {
      a.token_row[f] = -1;
    }
    __syncwarp();
    if (e >= 0 && lane == 31 - __clz(peers)) run[e] += __popc(peers);
    __syncwarp();
  }
}

// Row gather: one warp per destination row, 16-byte vectors.
struct GatherArgs {
  const uint8_t* src;     // [T, row_bytes]
  uint8_t* dst;           // [r_cap, row_bytes]
  const int32_t* row_token;
  const int32_t* offsets; // offsets[E] = rows in use
  int E, row_bytes;       // row_bytes % 16 == 0
};

__global__ void __launch_bounds__(256) permute_gather_kernel(GatherArgs a) {
  pdl_wait();
  pdl_trigger();
  const int rows = a.offsets[a.E];
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int vecs = a.row_bytes >> 4;
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int t = a.row_token[r];
    uint4* d = reinterpret_cast<uint4*>(a.dst + static_cast<int64_t>(r) * a.row_bytes);
    const uint4* s =
        t >= 0 ? reinterpret_cast<const uint4*>(a.src + static_cast<int64_t>(t) * a.row_bytes)
               : nullptr;
    warp_copy_row(d, s, vecs, threadIdx.x & 31);
  }
}

// One-round form of the row gather for rows of at most 32 * MAXV vectors: all
// loads of a row are issued before its first store and the next row's token
// index is read one row ahead (about one memory latency per row and warp).
// Plain loads keep all of them ahead of the stores (see permute_gather_bs_kernel).
template <int MAXV>
__global__ void __launch_bounds__(256) permute_gather_row_kernel(GatherArgs a) {
  pdl_wait();
  pdl_trigger();
  const int rows = a.offsets[a.E];
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  const int vecs = a.row_bytes >> 4;
  int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  int t = r < rows ? a.row_token[r] : -1;
  for (; r < rows; r += warps) {
    const int t_next = r + warps < rows ? a.row_token[r + warps] : -1;
    const uint4* src =
        t >= 0 ? reinterpret_cast<const uint4*>(a.src + static_cast<int64_t>(t) * a.row_bytes)
               : nullptr;
    uint4 buf[MAXV];
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int v = i * 32 + lane;
      buf[i] = (src && v < vecs) ? src[v] : make_uint4(0, 0, 0, 0);
    }
    uint4* d = reinterpret_cast<uint4*>(a.dst + static_cast<int64_t>(r) * a.row_bytes);
#pragma unroll
    for (int i = 0; i < MAXV; ++i)
      if (i * 32 + lane < vecs) d[i * 32 + lane] = buf[i];
    t = t_next;
  }
}

// ---------------------------------------------------------------------------
// Combine: y[t] = bf16(sum_j w[t,j] * out_rows[token_row[t*k+j]] + shared[t]),
// fp32 accumulation in j order.  One warp per token, 8 bf16 per lane-vector.
// ---------------------------------------------------------------------------
struct CombineArgs {
  const __nv_bfloat16* out_rows;  // [r_cap, H]
  const int32_t* token_row;       // [T*k]
  const float* topk_w;            // [T*k], or null: every weight 1 (the backward's dx sum)
  const __nv_bfloat16* shared;    // [T, H] or null
  __nv_bfloat16* y;               // [T, H]
  int T, H, k;
};

__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4& raw, float w) {
  const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = __bfloat1622float2(p2[q]);
    acc[2 * q] = fmaf(w, f.x, acc[2 * q]);
    acc[2 * q + 1] = fmaf(w, f.y, acc[2 * q + 1]);
  }
}

// One block per token; each thread owns 8 bf16 columns at a time and issues
// the loads of all K rows before accumulating them in j order.
template <int K>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const int kk = (K > 0) ? K : a.k;
  int rows[K > 0 ? K : 32];
  float ws[K > 0 ? K : 32];
#pragma unroll
  for (int j = 0; j < (K > 0 ? K : 32); ++j) {
    if (j < kk) {
      rows[j] = __ldg(a.token_row + static_cast<int64_t>(t) * kk + j);
      ws[j] = a.topk_w ? __ldg(a.topk_w + static_cast<int64_t>(t) * kk + j) : 1.0f;
    }
  }
  const int vecs = a.H >> 3;
  for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    if (K > 0) {
      uint4 raw[K > 0 ? K : 1];
#pragma unroll
      for (int j = 0; j < K; ++j)
        raw[j] = rows[j] >= 0 ? __ldg(reinterpret_cast<const uint4*>(
                                          a.out_rows + static_cast<int64_t>(rows[j]) * a.H) + v)
                              : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < K; ++j) acc_bf16x8(acc, raw[j], rows[j] >= 0 ? ws[j] : 0.f);
    } else {
      for (int j = 0; j < kk; ++j) {
        if (rows[j] < 0) continue;  // entry dropped by the permute (bad expert index)
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(
                                    a.out_rows + static_cast<int64_t>(rows[j]) * a.H) + v);
        acc_bf16x8(acc, raw, ws[j]);
      }
    }
    if (a.shared) {
      const uint4 raw =
          __ldg(reinterpret_cast<const uint4*>(a.shared + static_cast<int64_t>(t) * a.H) + v);
      acc_bf16x8(acc, raw, 1.0f);
    }
    uint4 o;
    __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int q = 0; q < 4; ++q) o2[q] = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
    reinterpret_cast<uint4*>(a.y + static_cast<int64_t>(t) * a.H)[v] = o;
  }
}

}  // namespace moe
