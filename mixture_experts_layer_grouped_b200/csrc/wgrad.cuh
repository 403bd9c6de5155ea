// Weight gradients of the grouped MLP, the shared expert and the router (the
// "wgrad" grouped GEMMs of the backward pass; TransformerEngine PR
// "DeepSeekV3Layer", Performance, "fused grouped MLP" row).  For each problem
// and each of its groups g:
//
//   out_g[m, n] = sum over the group's rows r of A[r, m] * B[r, n]   (fp32)
//
// with A and B row-major bf16: the contraction runs over rows (tokens).  A
// routed problem has one group per expert, over the expert's rows
// [offsets[e], offsets[e] + counts[e]) of the expert-major layout; a dense
// problem one group over rows [0, dense_rows).
//
// Both operands reach the tensor cores MN-major: a TMA box of 64 rows x 64
// columns with the 128-byte swizzle is the canonical MN-major SW128 layout
// (64 contiguous elements per 128-byte row, 8-row groups 1024 bytes apart),
// so no transposed copy of any activation is made.  Tiles are 128 (m) x 256
// (n) fp32 accumulators in TMEM, two of them, so the epilogue of one tile
// overlaps the MMAs of the next; CTAs are persistent and take tiles i, i +
// grid, ...
//
// A group's rows are read in 64-row steps, so the rows past its last one up to
// the next multiple of 64 must hold zeros in A or in B (the segment pads of a
// pad_multiple % 64 == 0 layout, or rows past the end of a dense operand, which
// TMA fills with zeros).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kWgMaxProblems = 8;
constexpr int kWgStages = 3;
constexpr int kWgBM = 128, kWgBN = 256, kWgBK = 64;
constexpr int kWgABytes = kWgBM * kWgBK * 2;  // 16 KB: two 64 x 64 boxes
constexpr int kWgBBytes = kWgBN * kWgBK * 2;  // 32 KB: four 64 x 64 boxes
constexpr int kWgStageBytes = kWgABytes + kWgBBytes;
constexpr int kWgEpiWarps = 8;  // two per TMEM lane quarter, 128 columns each
constexpr int kWgThreads = 32 * (2 + kWgEpiWarps);
// per epilogue warp, a 32 x 32 fp32 block staged with rows 36 floats apart
// (16-byte accesses of 8 threads at a time then hit distinct banks)
constexpr int kWgStgLd = 36;
constexpr int kWgStgBytes = kWgEpiWarps * 32 * kWgStgLd * 4;
constexpr int kWgSmemBytes = kWgStages * kWgStageBytes + kWgStgBytes + 256 + 1024;
constexpr uint32_t kWgTmemCols = 2 * kWgBN;

struct WgradProblem {
  CUtensorMap a;  // A: [rows, M] bf16, box 64 columns x 64 rows, 128-byte swizzle
  CUtensorMap b;  // B: [rows, N] bf16, the same boxes
  float* out;     // [groups][M][N] fp32
  int32_t M, N;
  int32_t routed;          // 1: a group per expert; 0: one group over dense_rows
  int32_t m_tiles, n_tiles;
  int32_t tile0;           // index of the problem's first tile
};

struct WgradParams {
  WgradProblem pr[kWgMaxProblems];
  int32_t nprob, total_tiles;
  const int32_t* counts;   // [E]
  const int32_t* offsets;  // [E + 1]
  int32_t E, dense_rows;
  int32_t* status;
};

struct WgTile {
  int p, g, m0, n0, row0, nrows;
};

__device__ __forceinline__ WgTile wg_decode(const WgradParams& P, int u) {
  WgTile t;
  int p = 0;
  while (p + 1 < P.nprob && u >= P.pr[p + 1].tile0) ++p;
  const WgradProblem& q = P.pr[p];
  int v = u - q.tile0;
  const int per = q.m_tiles * q.n_tiles;
  t.p = p;
  t.g = v / per;
  v -= t.g * per;
  const int mt = v / q.n_tiles;
  t.m0 = mt * kWgBM;
  t.n0 = (v - mt * q.n_tiles) * kWgBN;
  if (q.routed) {
    t.row0 = __ldg(P.offsets + t.g);
    t.nrows = __ldg(P.counts + t.g);
  } else {
    t.row0 = 0;
    t.nrows = P.dense_rows;
  }
  return t;
}

// Shared-memory descriptor of an MN-major operand staged by 64-row x
// 128-byte TMA boxes with the 128-byte swizzle: K rows 128 bytes apart, 8-row
// groups 1024 bytes apart (stride byte offset), successive 64-element MN
// blocks `mn_block_bytes` apart (leading byte offset).
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(uint32_t saddr, uint32_t mn_block_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(mn_block_bytes >> 4) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// kind::f16 instruction descriptor with A and B both MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_mn(int M, int N) {
  return idesc_bf16(M, N) | (1u << 15) | (1u << 16);
}

// ACC: add to the output's values instead of writing them (a compile-time
// choice, so the writing form carries no trace of the other).
template <bool ACC>
__global__ void __launch_bounds__(kWgThreads, 1) wgrad_kernel(const __grid_constant__ WgradParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* stg = reinterpret_cast<float*>(ring + kWgStages * kWgStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kWgStages * kWgStageBytes + kWgStgBytes);
  uint64_t* empty = full + kWgStages;
  uint64_t* acc_full = empty + kWgStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = warp_id(), lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWgStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kWgEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < P.nprob; ++i) {
      tma_prefetch_desc(&P.pr[i].a);
      tma_prefetch_desc(&P.pr[i].b);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kWgTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();  // a group's rows serve all its tiles
      int stage = 0;
      uint32_t phase = 0;
      uint32_t last[kWgStages];
#pragma unroll
      for (int s = 0; s < kWgStages; ++s) last[s] = 2;  // 2: nothing issued
      bool ok = true;
      for (int u = blockIdx.x; u < P.total_tiles && ok; u += gridDim.x) {
        const WgTile t = wg_decode(P, u);
        const WgradProblem& q = P.pr[t.p];
        const int ks = (t.nrows + kWgBK - 1) / kWgBK;
        for (int k = 0; k < ks; ++k) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, P.status)) { ok = false; break; }
          uint8_t* sa = ring + stage * kWgStageBytes;
          uint8_t* sb = sa + kWgABytes;
          mbar_arrive_expect_tx(&full[stage], kWgStageBytes);
          const int r = t.row0 + k * kWgBK;
          tma_load_2d(sa, &q.a, &full[stage], t.m0, r, pol);
          tma_load_2d(sa + 8192, &q.a, &full[stage], t.m0 + 64, r, pol);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tma_load_2d(sb + 8192 * j, &q.b, &full[stage], t.n0 + 64 * j, r, pol);
#pragma unroll
          for (int s = 0; s < kWgStages; ++s)
            if (s == stage) last[s] = phase;
          if (++stage == kWgStages) { stage = 0; phase ^= 1; }
        }
      }
      // every load issued lands before the CTA may leave (bounded: 20 ms)
      const uint64_t t0 = global_timer_ns();
#pragma unroll
      for (int s = 0; s < kWgStages; ++s) {
        if (last[s] > 1) continue;
        while (!mbar_try_wait(&full[s], last[s]) && global_timer_ns() - t0 < 20000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_mn(kWgBM, kWgBN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < P.total_tiles && ok; u += gridDim.x) {
        const WgTile t = wg_decode(P, u);
        const int ks = (t.nrows + kWgBK - 1) / kWgBK;
        if (ks == 0) continue;  // the epilogue writes the zero gradient itself
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag, P.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * kWgBN;
        for (int k = 0; k < ks; ++k) {
          if (!mbar_wait(&full[stage], phase, abort_flag, P.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + stage * kWgStageBytes);
          const uint32_t sb = sa + kWgABytes;
#pragma unroll
          for (int kk = 0; kk < kWgBK / 16; ++kk)  // 16 rows (2 groups of 8) per MMA
            mma_bf16(d, sdesc_mnmajor_sw128(sa + kk * 2048, 8192),
                     sdesc_mnmajor_sw128(sb + kk * 2048, 8192), idesc, (k | kk) != 0 ? 1u : 0u);
          mma_commit(&empty[stage]);
          if (++stage == kWgStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(&acc_full[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      mma_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 20000000ull) {
      }
    }
  } else {
    // ---------------- epilogue: TMEM -> fp32 rows of the output ----------------
    const int quarter = warp & 3;          // TMEM lanes 32 * quarter ..
    const int half = (warp - 2) >> 2;      // columns 128 * half ..
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < P.total_tiles; u += gridDim.x) {
      const WgTile t = wg_decode(P, u);
      const WgradProblem& q = P.pr[t.p];
      float* out = q.out + static_cast<int64_t>(t.g) * q.M * q.N;
      const int m = t.m0 + quarter * 32 + lane;
      const int nb = t.n0 + half * 128;
      if (t.nrows == 0) {
        // an expert no token picked: its gradient is zero (nothing to add)
        if (m < q.M && !ACC) {
          for (int c = 0; c < 128; c += 4)
            if (nb + c < q.N)
              *reinterpret_cast<float4*>(out + static_cast<int64_t>(m) * q.N + nb + c) =
                  make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag, P.status)) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kWgBN + half * 128;
      // lane = row in TMEM; through shared memory each store instruction then
      // writes four whole 128-byte row segments
      float* my = stg + (warp - 2) * 32 * kWgStgLd;
      const int m_base = t.m0 + quarter * 32;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + c * 32, r);
        tmem_ld_wait();
        const int n = nb + c * 32;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(my + lane * kWgStgLd + 4 * j) =
              make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                          __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
        __syncwarp();
        if (n < q.N) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int row = 4 * i + (lane >> 3), col = 4 * (lane & 7);
            if (m_base + row < q.M) {
              float4* dst = reinterpret_cast<float4*>(out + static_cast<int64_t>(m_base + row) * q.N +
                                                      n + col);
              float4 v = *reinterpret_cast<const float4*>(my + row * kWgStgLd + col);
              if constexpr (ACC) {
                const float4 o = *dst;
                v.x += o.x;
                v.y += o.y;
                v.z += o.z;
                v.w += o.w;
              }
              *dst = v;
            }
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kWgTmemCols);
  }
}

// Zeroes the pad rows (row_token < 0) below offsets[E] of an expert-major
// bf16 matrix [rows, n]: a warp per row.
__global__ void __launch_bounds__(256) zero_pad_rows_kernel(__nv_bfloat16* __restrict__ m, int n,
                                                            const int32_t* __restrict__ row_token,
                                                            const int32_t* __restrict__ rows_used) {
  pdl_wait();
  pdl_trigger();
  const int64_t nrows = __ldg(rows_used);
  const int lane = threadIdx.x & 31;
  const int64_t w0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t r = w0; r < nrows; r += nw) {
    if (__ldg(row_token + r) >= 0) continue;
    uint4* row = reinterpret_cast<uint4*>(m + r * n);
    for (int v = lane; v < n / 8; v += 32) row[v] = make_uint4(0, 0, 0, 0);
  }
}

}  // namespace moe
