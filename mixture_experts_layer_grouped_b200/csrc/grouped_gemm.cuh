// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent kernel per GEMM.  The work is a list of tiles over two
// groups: the routed experts (expert-major rows, per-expert token counts read
// on the device) and an optional dense group (token-order rows: the shared
// expert, or the router).  Operands are swapped with respect to the usual
// "tokens x features" orientation: the MMA's M operand (128 rows) is a slab of
// the expert's weight matrix and its N operand (16..256 columns) is the
// expert's tokens.  So every weight slab streams from HBM once per
// 256-token chunk of its expert, an expert with few tokens costs an N of
// ceil16(tokens) rather than a 128-row M tile, and the fp32 accumulator sits in
// TMEM as [weight row = TMEM lane, token = TMEM column].
//
// Warp roles (192 threads): warp 0 issues TMA loads into an smem ring, warp 1
// allocates TMEM and issues tcgen05.mma from one thread, warps 2-5 drain the
// accumulator (tcgen05.ld), apply the epilogue (fp32 store, SwiGLU, or bf16
// store) and write the outputs through a per-warp staging tile.
//
// Epilogue per mode:
//   kRouter: logits[t, e] = acc (fp32);
//   kFc1   : two accumulators (W1 slab and W3 slab against the same tokens),
//            h[row, f] = bf16(silu(gate) * up);
//   kFc2   : out[row, f] = bf16(acc).
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kBM = 128;        // weight rows per tile (MMA M)
constexpr int kBK = 64;         // bf16 elements per k-step: one 128-byte row
constexpr int kBoxRows = 32;    // token rows per TMA box
constexpr int kMaxTileN = 256;  // tokens per tile (MMA N max)
constexpr int kGemmThreads = 192;
constexpr int kMaxExperts = 1024;

enum GemmMode { kRouter = 0, kFc1 = 1, kFc2 = 2 };

struct GemmGroup {
  int32_t a_rows_per_expert;  // rows of each expert's A in the 2-D view
  int32_t a_valid_rows;       // valid A rows per expert (epilogue mask)
  int32_t n_slabs;            // ceil(a_valid_rows / 128)
  int32_t k_tiles;            // K / 64
  void* out;                  // output base (rows x columns)
  int64_t out_ld;             // output row stride, elements
};

struct GemmParams {
  CUtensorMap a0[2];  // [routed, dense]: W1 (fc1), W2 (fc2), W_r (router)
  CUtensorMap a1[2];  // [routed, dense]: W3 (fc1 only)
  CUtensorMap b[2];   // [routed, dense]: token rows
  GemmGroup g[2];
  const int32_t* counts;   // [E]
  const int32_t* offsets;  // [E+1]
  int32_t E;               // routed experts (0: no routed group)
  int32_t dense_rows;      // rows of the dense group (0: none)
  int32_t tile_n;          // tokens per tile, multiple of 32, <= 256
  int32_t* status;
};

template <int MODE>
struct GemmCfg {
  static constexpr int NA = (MODE == kFc1) ? 2 : 1;
  static constexpr int A_BYTES = kBM * 128;
  static constexpr int B_BYTES = kMaxTileN * 128;
  static constexpr int STAGE_BYTES = NA * A_BYTES + B_BYTES;
  static constexpr int STAGES = (MODE == kFc1) ? 3 : 4;
  static constexpr int STG_BYTES = 4 * 32 * 32 * 2;  // 4 warps x 32x32 bf16
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES =
      1024 + STAGES * STAGE_BYTES + STG_BYTES + BAR_BYTES + 4 * (kMaxExperts + 1);
  static constexpr uint32_t TMEM_COLS = (MODE == kFc1) ? 512 : 256;
};

struct Tile {
  int grp, e, slab, row0, n_tok, k_tiles, a_row;
};

__device__ __forceinline__ Tile decode_tile(int u, const GemmParams& p, const int* prefix,
                                            int units_routed) {
  Tile t;
  if (u < units_routed) {
    const int ns = p.g[0].n_slabs;
    const int q = u / ns;
    t.slab = u - q * ns;
    int lo = 0, hi = p.E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= q) lo = mid; else hi = mid;
    }
    const int chunk = q - prefix[lo];
    t.grp = 0;
    t.e = lo;
    t.row0 = __ldg(p.offsets + lo) + chunk * p.tile_n;
    t.n_tok = min(p.tile_n, __ldg(p.counts + lo) - chunk * p.tile_n);
    t.a_row = lo * p.g[0].a_rows_per_expert + t.slab * kBM;
  } else {
    const int v = u - units_routed;
    const int ns = p.g[1].n_slabs;
    const int chunk = v / ns;
    t.slab = v - chunk * ns;
    t.grp = 1;
    t.e = 0;
    t.row0 = chunk * p.tile_n;
    t.n_tok = min(p.tile_n, p.dense_rows - t.row0);
    t.a_row = t.slab * kBM;
  }
  t.k_tiles = p.g[t.grp].k_tiles;
  return t;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1) grouped_gemm_kernel(
    const __grid_constant__ GemmParams p) {
  using C = GemmCfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint8_t* stg = ring + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + C::STG_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* prefix = reinterpret_cast<int*>(stg + C::STG_BYTES + C::BAR_BYTES);

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < 2; ++i) {
      tma_prefetch_desc(&p.a0[i]);
      tma_prefetch_desc(&p.b[i]);
      if (MODE == kFc1) tma_prefetch_desc(&p.a1[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2) {
    // prefix[e] = number of token chunks of experts < e
    const int E = p.E;
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int local = 0;
    for (int e = e0; e < e1; ++e) {
      int c = __ldg(p.counts + e);
      local += (c + p.tile_n - 1) / p.tile_n;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    if (lane == 0) prefix[0] = 0;
    for (int e = e0; e < e1; ++e) {
      int c = __ldg(p.counts + e);
      run += (c + p.tile_n - 1) / p.tile_n;
      prefix[e + 1] = run;
    }
    if (E == 0 && lane == 0) prefix[0] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int units_routed = (p.E > 0) ? prefix[p.E] * p.g[0].n_slabs : 0;
  const int units_dense =
      (p.dense_rows > 0) ? ((p.dense_rows + p.tile_n - 1) / p.tile_n) * p.g[1].n_slabs : 0;
  const int units = units_routed + units_dense;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int last_phase[C::STAGES];
#pragma unroll
      for (int s = 0; s < C::STAGES; ++s) last_phase[s] = -1;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Tile t = decode_tile(u, p, prefix, units_routed);
        const int nbox = (t.n_tok + kBoxRows - 1) / kBoxRows;
        const uint32_t bytes = C::NA * C::A_BYTES + nbox * kBoxRows * 128;
        for (int kt = 0; kt < t.k_tiles; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status)) { ok = false; break; }
          uint8_t* sa = ring + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_2d(sa, &p.a0[t.grp], &full[stage], kt * kBK, t.a_row, pol_w);
          if (MODE == kFc1)
            tma_load_2d(sa + C::A_BYTES, &p.a1[t.grp], &full[stage], kt * kBK, t.a_row, pol_w);
          uint8_t* sb = sa + C::NA * C::A_BYTES;
          for (int bx = 0; bx < nbox; ++bx)
            tma_load_2d(sb + bx * kBoxRows * 128, &p.b[t.grp], &full[stage], kt * kBK,
                        t.row0 + bx * kBoxRows, pol_x);
          last_phase[stage] = phase;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // Let in-flight copies land before the CTA can exit.
        for (int s = 0; s < C::STAGES; ++s)
          if (last_phase[s] >= 0) {
            uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&full[s], last_phase[s]) && global_timer_ns() - t0 < 20000000ull) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const Tile t = decode_tile(u, p, prefix, units_routed);
        const int n_mma = (t.n_tok + 15) & ~15;
        const uint32_t idesc = idesc_bf16(kBM, n_mma);
        if (!mbar_wait(acc_empty, acc_phase ^ 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        for (int kt = 0; kt < t.k_tiles; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::NA * C::A_BYTES;
          const uint64_t da0 = sdesc_kmajor_sw128(sa);
          const uint64_t db = sdesc_kmajor_sw128(sb);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t acc = (kt | kk) ? 1u : 0u;
            // advance 16 bf16 = 32 bytes along K inside the swizzle atom
            mma_bf16(tmem_base, da0 + 2 * kk, db + 2 * kk, idesc, acc);
            if (MODE == kFc1) {
              const uint64_t da1 = sdesc_kmajor_sw128(sa + C::A_BYTES);
              mma_bf16(tmem_base + 256, da1 + 2 * kk, db + 2 * kk, idesc, acc);
            }
          }
          mma_commit(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        mma_commit(acc_full);
        acc_phase ^= 1;
      }
      // Drain: all issued MMAs complete before TMEM is released.
      mma_commit(drain);
      uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 20000000ull) {
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;  // TMEM lane quarter this warp may access
    uint8_t* my_stg = stg + (warp - 2) * (32 * 32 * 2);
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const Tile t = decode_tile(u, p, prefix, units_routed);
      if (!mbar_wait(acc_full, acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const GemmGroup& G = p.g[t.grp];
      const int f0 = t.slab * kBM + quarter * 32;  // first feature row of this warp
      const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
      for (int c0 = 0; c0 < t.n_tok; c0 += 32) {
        uint32_t r0[32];
        tmem_ld_32x32b_x32(lane_addr + c0, r0);
        if (MODE == kFc1) {
          uint32_t r1[32];
          tmem_ld_32x32b_x32(lane_addr + 256 + c0, r1);
          tmem_ld_wait();
          __nv_bfloat16* s = reinterpret_cast<__nv_bfloat16*>(my_stg);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float g = __uint_as_float(r0[j]);
            const float up = __uint_as_float(r1[j]);
            s[j * 32 + lane] = __float2bfloat16_rn(silu_f(g) * up);
          }
        } else if (MODE == kFc2) {
          tmem_ld_wait();
          __nv_bfloat16* s = reinterpret_cast<__nv_bfloat16*>(my_stg);
#pragma unroll
          for (int j = 0; j < 32; ++j) s[j * 32 + lane] = __float2bfloat16_rn(__uint_as_float(r0[j]));
        } else {
          tmem_ld_wait();
        }
        __syncwarp();
        const int rows_here = min(32, t.n_tok - c0);
        if (MODE == kRouter) {
          // thread = expert, register j = token: 32 consecutive fp32 per token
          float* out = static_cast<float*>(G.out);
          const int e = f0 + lane;
          if (e < G.a_valid_rows) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < rows_here)
                out[static_cast<int64_t>(t.row0 + c0 + j) * G.out_ld + e] = __uint_as_float(r0[j]);
          }
        } else {
          // [32 tokens][32 features] bf16: 64 bytes per token row, 4 x 16 B
          const uint4* s = reinterpret_cast<const uint4*>(my_stg);
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(G.out);
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int c = it * 32 + lane;
            const int j = c >> 2, part = c & 3;
            if (j < rows_here && f0 < G.a_valid_rows) {
              uint4 v = s[j * 4 + part];
              *reinterpret_cast<uint4*>(out + static_cast<int64_t>(t.row0 + c0 + j) * G.out_ld +
                                        f0 + part * 8) = v;
            }
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace moe
