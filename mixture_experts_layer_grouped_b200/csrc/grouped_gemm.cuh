// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// One persistent kernel per GEMM.  The work is a list of tiles over two
// groups: the routed experts (expert-major rows, per-expert token counts read
// on the device) and an optional dense group (token-order rows: the shared
// expert, or the router).  Operands are swapped with respect to the usual
// "tokens x features" orientation: the MMA's M operand (128 rows) is a slab of
// an expert's weight matrix and its N operand (16..TILE_N columns) is the
// expert's tokens.  So every weight slab streams from HBM once per TILE_N
// token chunk of its expert, an expert with few tokens costs an N of
// ceil16(tokens) rather than a 128-row M tile, and the fp32 accumulator sits
// in TMEM as [weight row = TMEM lane, token = TMEM column].
//
// Each tile issues two MMAs per K step against the same token operand (NA=2):
//   kFc1   : a W1 slab and the W3 slab of the same 128 features; the epilogue
//            forms h = bf16(silu(gate) * up) thread-locally (same TMEM lane);
//   kFc2   : two adjacent 128-row slabs of W2 (256 output features);
//   kRouter: one W_r slab (NA=1), with the K range optionally split across
//            tiles; each split writes its own fp32 partial logits.
//
// Warp roles (320 threads): warp 0 issues TMA loads into an smem ring, warp 1
// owns TMEM and issues tcgen05.mma from one thread, warps 2-9 drain the
// accumulators (tcgen05.ld; two warps per TMEM lane quarter, alternating
// 32-column chunks) and write the outputs.  When the accumulators of
// one tile use at most half of TMEM they are double-buffered, so the epilogue
// of tile i overlaps the MMAs of tile i+1; otherwise fc1 and fc2 read their
// accumulators into registers and release them before storing.
//
// Tiles are claimed at run time from a counter (or taken statically), and fc2
// may start before fc1 ends: its producer waits, per token chunk, for fc1's
// epilogue warps to have stored that chunk of h (see GemmParams::chunk_done).
//
// CTA pairs (PAIR): clusters of two CTAs run one tile together with M = 256
// MMAs (cta_group::2) issued by rank 0.  Each CTA holds its own 128 weight rows
// and half of the tile's token rows, so a stage carries half the token bytes
// and the ring gets a fourth stage; the accumulator of a CTA's 128 features
// sits in its own TMEM.
//
// The ring is latency-bound: a stage slot cycles through TMA issue, arrival
// (about 1.5-2 us under full HBM load), MMA and release, so the bytes of
// weights in flight per SM set the streaming rate.  Stage layouts therefore
// favour weight bytes (two 16 KB weight boxes per stage) over TMEM double
// buffering.
#pragma once

#include "common.cuh"

namespace moe {

constexpr int kBM = 128;      // weight rows per MMA (M)
constexpr int kBK = 64;       // bf16 elements per k-step: one 128-byte row
constexpr int kBoxRows = 32;  // token rows per TMA box
constexpr int kEpiWarps = 8;  // two warps per TMEM lane quarter, alternating 32-column chunks
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxExperts = 1024;
constexpr int kRingBytes = 192 * 1024;

enum GemmMode { kRouter = 0, kFc1 = 1, kFc2 = 2 };
enum GemmDtype { kBF16 = 0, kMXF8 = 1, kNVF4 = 2 };

struct GemmGroup {
  int32_t a_rows_per_expert;  // rows of each expert's A (row-major or tile-major view)
  int32_t a_valid_rows;       // valid output features per expert (epilogue mask)
  int32_t n_slabs;            // tiles along the features of one expert
  int32_t k_tiles;            // K / 64
  int32_t k_splits;           // K-range splits (router only; 1 otherwise)
  void* out;                  // output base (rows x columns)
  int64_t out_ld;             // output row stride, elements
  int64_t split_stride;       // elements between the partial outputs of splits
};

struct GemmParams {
  CUtensorMap a0[2];  // [routed, dense]: W1 (fc1), W2 (fc2), W_r (router)
  CUtensorMap a1[2];  // [routed, dense]: W3 (fc1 only)
  CUtensorMap b[2];   // [routed, dense]: token rows
  GemmGroup g[2];
  // block scales (MXFP8 / NVFP4) in the 128x4-chunk MMA layout, per group
  const uint8_t* sfa0[2];   // scales of a0's rows
  const uint8_t* sfa1[2];   // scales of a1's rows
  const uint8_t* sfb[2];    // scales of the token rows
  // CTA pairs: the same scale buffers as 2-D maps of 512-byte chunks (uint32 x 128)
  CUtensorMap sfa0_map[2];
  CUtensorMap sfa1_map[2];
  CUtensorMap sfb_map[2];
  int32_t kb4[2];           // chunk columns per row chunk (K/128 MXFP8, K/64 NVFP4)
  // NVFP4 global scales: acc * 1 / (ga[e * ga_stride] * gw[e * gw_stride])
  const float* ga[2];
  int32_t ga_stride[2];
  const float* gw[2];
  int32_t gw_stride[2];
  float* amax_out[2];       // fc1 NVFP4: per-expert amax of h (atomic max)
  int32_t amax_stride[2];
  // routed token rows gathered straight from token-order x: b[0] is then a map
  // over x with one-row boxes, and tile row j is x[row_token[row0 + j]]
  const int32_t* row_token;
  // fc1 with quantized output: h codes [rows, ld] and scales (MMA layout, KB = ld/32)
  uint8_t* q_out[2];
  uint8_t* q_sf[2];
  const int32_t* counts;   // [E]
  const int32_t* offsets;  // [E+1]
  int32_t E;               // routed experts (0: no routed group)
  int32_t dense_rows;      // rows of the dense group (0: none)
  int32_t* status;
  // fc1 -> fc2 hand-off per token chunk (null: none).  Chunk ids number the
  // TILE_N-token chunks of the routed experts in order, then the dense group's.
  // fc1 adds one per epilogue warp to chunk_done[id] once the warp's h rows of
  // the tile are stored; fc2 starts without waiting for fc1 as a whole and
  // loads a chunk's h only after chunk_done[id] reached chunk_target[group]
  // (fc1 slabs x epilogue warps per tile).
  int32_t* chunk_done;
  int32_t chunk_target[2];
  // dynamic tile order (null: CTA i takes tiles i, i + grid, ...): the next
  // tile index is claimed from this zeroed counter
  int32_t* unit_counter;
  // backward form of fc1 (the BWD kernel): per group, the column of `out` where
  // u's features start (a at the feature's own column)
  int32_t bwd_u_col[2];
};

constexpr int pow2_at_least(int v) {
  int p = 32;
  while (p < v) p <<= 1;
  return p;
}

template <int MODE, int TILE_N, int DT = kBF16, bool PAIR = false>
struct GemmCfg {
  static constexpr int NA = (MODE == kRouter) ? 1 : 2;
  static constexpr int A_BYTES = kBM * 128;
  // a CTA pair splits the token rows of a tile: each CTA holds TILE_N / 2
  static constexpr int B_ROWS = PAIR ? TILE_N / 2 : TILE_N;
  static constexpr int B_BYTES = B_ROWS * 128;
  static constexpr int SF_CHUNK = 512;                          // one 128x4 scale chunk
  static constexpr int SF_KCH = (DT == kNVF4) ? 4 : 1;          // scale chunks per k-step
  // token row chunks of scales: a tile starts at a row that is a multiple of 64
  // (segments are 64-aligned, tiles TILE_N apart, TILE_N % 64 == 0), so it spans
  // at most ceil((TILE_N + 64) / 128) chunks.  (The MMA's scale address must sit
  // on an even TMEM column: the base shifts by (row0 % 128) / 32, i.e. 0 or 2.)
  static_assert(DT == kBF16 || TILE_N % 64 == 0, "block-scaled tiles are 64-row multiples");
  static constexpr int SFB_CHUNKS = (TILE_N + 64 + 127) / 128;
  static constexpr int SF_BYTES = (DT != kBF16) ? (NA + SFB_CHUNKS) * SF_KCH * SF_CHUNK : 0;
  static constexpr int STAGE_BYTES = (NA * A_BYTES + B_BYTES + SF_BYTES + 1023) / 1024 * 1024;
  static constexpr int STG_WARP = 32 * 34 * 2;                 // per warp 32 x 34 bf16
  static constexpr int STG_BYTES = kEpiWarps * STG_WARP;
  static constexpr int BAR_BYTES = 512;  // ring / accumulator barriers, then the tile queue
  // CTA pairs take every byte the epilogue staging, barriers and tile prefix leave
  static constexpr int RING = PAIR ? (232448 - 1024 - STG_BYTES - BAR_BYTES - 4 * (kMaxExperts + 1))
                                   : ((DT == kNVF4) ? 198 * 1024 : kRingBytes);
  static constexpr int STAGES = (RING / STAGE_BYTES) > 8 ? 8 : (RING / STAGE_BYTES);
  static constexpr int ACC_COLS = NA * TILE_N;  // TMEM columns of one tile
  static constexpr int SF_COLS = (DT != kBF16) ? 4 * SF_KCH * (NA + SFB_CHUNKS) : 0;
  static constexpr int ACC_BUFS = (2 * ACC_COLS + SF_COLS <= 512) ? 2 : 1;
  static constexpr int SF_TMEM = ACC_BUFS * ACC_COLS;  // first scale-factor column
  // scale factors alternate between two TMEM regions by stage when they fit, so
  // the copies of stage s+1 do not overwrite columns stage s's MMAs still read
  static constexpr int SF_BUFS = (SF_COLS > 0 && ACC_BUFS * ACC_COLS + 2 * SF_COLS <= 512) ? 2 : 1;
  static constexpr uint32_t TMEM_COLS = pow2_at_least(ACC_BUFS * ACC_COLS + SF_BUFS * SF_COLS);
  static constexpr int SLAB_ROWS = (MODE == kFc2) ? 2 * kBM : kBM;  // features per CTA tile
  static constexpr int SLAB_SPAN = PAIR ? 2 * SLAB_ROWS : SLAB_ROWS;  // features per tile
  static constexpr int SMEM_BYTES =
      1024 + STAGES * STAGE_BYTES + STG_BYTES + BAR_BYTES + 4 * (kMaxExperts + 1);
  static_assert(TMEM_COLS <= 512, "TMEM overflow");
  static_assert(SMEM_BYTES <= 232448, "smem overflow");
  static_assert(STAGE_BYTES % 1024 == 0 || DT != kBF16, "stage alignment");
};

struct Tile {
  int grp, e, slab, row0, n_tok, k_begin, k_end, a_row, split;
  int f0;  // first output feature of this CTA's rows within the expert
  int chunk_id;  // token chunk over both groups (routed chunks, then dense)
};

// `rank` is the CTA's rank in its pair (0 without pairs): its A rows start
// SLAB_ROWS into the tile's SLAB_SPAN features.
template <int MODE, int TILE_N, int DT, bool PAIR>
__device__ __forceinline__ Tile decode_tile(int u, const GemmParams& p, const int* prefix,
                                            int units_routed, int rank = 0) {
  using C = GemmCfg<MODE, TILE_N, DT, PAIR>;
  Tile t;
  if (u < units_routed) {
    // expert e owns units [prefix[e] * ns, prefix[e + 1] * ns), slab-major: the
    // token chunks of one weight slab are adjacent, so they run at about the same
    // time and the slab's later reads hit L2
    const int ns = p.g[0].n_slabs;
    int lo = 0, hi = p.E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] * ns <= u) lo = mid; else hi = mid;
    }
    const int nch = prefix[lo + 1] - prefix[lo];
    const int v = u - prefix[lo] * ns;
    t.slab = v / nch;
    const int chunk = v - t.slab * nch;
    t.grp = 0;
    t.e = lo;
    t.chunk_id = prefix[lo] + chunk;
    t.row0 = __ldg(p.offsets + lo) + chunk * TILE_N;
    t.n_tok = min(TILE_N, __ldg(p.counts + lo) - chunk * TILE_N);
    t.f0 = t.slab * C::SLAB_SPAN + rank * C::SLAB_ROWS;
    t.a_row = lo * p.g[0].a_rows_per_expert + t.f0;
    t.split = 0;
    t.k_begin = 0;
    t.k_end = p.g[0].k_tiles;
  } else {
    const GemmGroup& G = p.g[1];
    int v = u - units_routed;
    t.split = v % G.k_splits;
    v /= G.k_splits;
    const int ns = G.n_slabs;
    const int chunk = v / ns;
    t.slab = v - chunk * ns;
    t.grp = 1;
    t.e = 0;
    t.chunk_id = (p.E > 0 ? prefix[p.E] : 0) + chunk;
    t.row0 = chunk * TILE_N;
    t.n_tok = min(TILE_N, p.dense_rows - t.row0);
    t.f0 = t.slab * C::SLAB_SPAN + rank * C::SLAB_ROWS;
    t.a_row = t.f0;
    const int kps = (G.k_tiles + G.k_splits - 1) / G.k_splits;
    t.k_begin = t.split * kps;
    t.k_end = min(G.k_tiles, t.k_begin + kps);
  }
  return t;
}

// fc1 epilogue warp, after its rows of a tile are stored: count the warp done
// on the tile's token chunk.  Every lane fences its own stores at GPU scope,
// the warp barrier orders the fences before lane 0's counter update, so an fc2
// producer that acquires the full count sees every h row of the chunk.
__device__ __forceinline__ void signal_chunk(const GemmParams& p, const Tile& t, int lane) {
  if (p.chunk_done == nullptr) return;
  __threadfence();
  __syncwarp();
  if (lane == 0) atomicAdd(p.chunk_done + t.chunk_id, 1);
}

// The sequence of tiles a CTA (or CTA pair) works on.  Static: first, first +
// stride, ...  Dynamic (p.unit_counter set): the producer thread (rank 0's in
// a pair) claims the next tile from the global counter when it is ready to
// load one and publishes the index through a kSched-slot queue in shared
// memory (in both CTAs of a pair); the other roles (the MMA thread, the eight
// epilogue warps, rank 1's producer) read it and release the slot.  CTAs that
// start late or run short tiles simply claim fewer tiles.  Tiles are claimed
// in list order, so a claimed fc2 tile's fc1 chunk was claimed before by a
// running fc1 CTA.
constexpr int kSched = 4;

struct TileQueue {
  uint64_t* full;      // [kSched], one arrival (the claimer)
  uint64_t* empty;     // [kSched], one arrival per consumer of both CTAs
  volatile int* slot_u;
  int slot;
  uint32_t phase;
  int next_static, stride;
  bool dynamic;
};

// Producer of rank 0 (or of a single CTA): the next tile, or `units` at the end.
template <bool PAIR>
__device__ __forceinline__ int claim_tile(TileQueue& q, const GemmParams& p, int units,
                                          volatile int* abort, bool& ok) {
  if (!q.dynamic) {
    const int u = q.next_static;
    q.next_static += q.stride;
    return u;
  }
  const bool free_slot = PAIR ? mbar_wait_cluster(&q.empty[q.slot], q.phase ^ 1, abort, p.status)
                              : mbar_wait(&q.empty[q.slot], q.phase ^ 1, abort, p.status);
  if (!free_slot) { ok = false; return units; }
  int u = atomicAdd(p.unit_counter, 1);
  if (u > units) u = units;
  q.slot_u[q.slot] = u;
  if constexpr (PAIR) {
    st_shared_cluster_s32(cluster_addr(const_cast<int*>(&q.slot_u[q.slot]), 1), u);
    mbar_arrive_release_cluster(cluster_addr(&q.full[q.slot], 1));
  }
  mbar_arrive(&q.full[q.slot]);
  if (++q.slot == kSched) { q.slot = 0; q.phase ^= 1; }
  return u;
}

// Any other role: the next tile, or `units` at the end (or on a time-out).
// A warp calls it with all lanes (one release per warp), a thread alone with
// warp_wide = false.
template <bool PAIR>
__device__ __forceinline__ int next_tile(TileQueue& q, const GemmParams& p, int units, int rank,
                                         bool warp_wide, volatile int* abort) {
  if (!q.dynamic) {
    const int u = q.next_static;
    q.next_static += q.stride;
    return u;
  }
  const bool got = (PAIR && rank == 1)
                       ? mbar_wait_cluster(&q.full[q.slot], q.phase, abort, p.status)
                       : mbar_wait(&q.full[q.slot], q.phase, abort, p.status);
  const int u = got ? q.slot_u[q.slot] : units;
  if (warp_wide) __syncwarp();
  if (!warp_wide || lane_id() == 0) {
    if constexpr (PAIR) mbar_arrive_release_cluster(cluster_addr(&q.empty[q.slot], 0));
    else mbar_arrive(&q.empty[q.slot]);
  }
  if (++q.slot == kSched) { q.slot = 0; q.phase ^= 1; }
  return u;
}

// One-CTA or CTA-pair (cta_group::2) forms of the MMA issuer's instructions.
template <bool PAIR>
__device__ __forceinline__ void mma_bf16_x(uint32_t d, uint64_t a, uint64_t b, uint32_t id,
                                           uint32_t acc) {
  if constexpr (PAIR) mma_bf16_pair(d, a, b, id, acc); else mma_bf16(d, a, b, id, acc);
}
template <bool PAIR>
__device__ __forceinline__ void mma_mxf8_x(uint32_t d, uint64_t a, uint64_t b, uint32_t id,
                                           uint32_t sfa, uint32_t sfb, uint32_t acc) {
  if constexpr (PAIR) mma_mxf8_pair(d, a, b, id, sfa, sfb, acc);
  else mma_mxf8(d, a, b, id, sfa, sfb, acc);
}
template <bool PAIR>
__device__ __forceinline__ void mma_nvf4_x(uint32_t d, uint64_t a, uint64_t b, uint32_t id,
                                           uint32_t sfa, uint32_t sfb, uint32_t acc) {
  if constexpr (PAIR) mma_nvf4_pair(d, a, b, id, sfa, sfb, acc);
  else mma_nvf4(d, a, b, id, sfa, sfb, acc);
}
template <bool PAIR>
__device__ __forceinline__ void tmem_cp_sf_chunk_x(uint32_t taddr, uint64_t sdesc) {
  if constexpr (PAIR) tmem_cp_sf_chunk_pair(taddr, sdesc); else tmem_cp_sf_chunk(taddr, sdesc);
}
// Arrive on `bar` once the issued tcgen05 work completes; pairs arrive on the
// barrier of both CTAs (two commits, no multicast form).
template <bool PAIR>
__device__ __forceinline__ void commit_x(uint64_t* bar) {
  if constexpr (PAIR) {
    mma_commit_pair(cluster_addr(bar, 0));
    mma_commit_pair(cluster_addr(bar, 1));
  } else {
    mma_commit(bar);
  }
}

// Seed of the reciprocal 1/d for d >= 1: an fp32 bit pattern read as an
// integer is, up to an offset and a scale, a piecewise-linear approximation
// of log2 of the value, so subtracting it from a constant approximates
// log2(1/d) and the result, read back as fp32, approximates 1/d (the idea
// behind the well-known bit-level inverse square root).  0x7EF311C2 is the
// constant that minimises the largest relative error of that seed over a
// binade: 5.05%, found by a search over all 2^23 mantissas of [1, 2) (the
// error repeats in every binade).  Three Newton-Raphson steps take it below
// 1e-10 in exact arithmetic, i.e. to fp32 rounding.
constexpr int kRcpSeed = 0x7EF311C2;

// silu(g) = g / (1 + e^-g).  e^-g comes from the hardware exponential (one
// multi-function-unit op); 1 / (1 + e^-g) is refined from the kRcpSeed seed by
// three Newton-Raphson steps r <- r (2 - d r) on the FMA pipe, which leaves it
// within about one fp32 ulp.  Arguments below -80 are clamped there (silu is
// then below 1e-32 in magnitude either way).  Keeping the epilogue to one
// multi-function op per element (plus one packed bf16 conversion per two) is
// what bounds its time.
__device__ __forceinline__ float silu_f(float g) {
  const float d = 1.0f + __expf(-fmaxf(g, -80.0f));
  float r = __int_as_float(kRcpSeed - __float_as_int(d));
#pragma unroll
  for (int i = 0; i < 3; ++i) r = fmaf(r, fmaf(-d, r, 1.0f), r);
  return g * r;
}

// bf16 pair (a in the low half) as one 32-bit word, one packed conversion.
__device__ __forceinline__ uint32_t bf16x2_bits(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Two fp32 values in one 64-bit register pair, for the sm_100 packed f32x2
// add / mul / fma: one instruction computes both halves, each rounded exactly
// as its scalar form would be.
__device__ __forceinline__ uint64_t f32x2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// bf16(silu(g0) * u0) and bf16(silu(g1) * u1) as one word: silu_f's steps for
// two accumulator columns at once -- the exponentials one by one, then the
// add, the three Newton-Raphson steps and both products as packed f32x2
// instructions.  Same operations and roundings as silu_f(g) * u (bit-identical
// results) in about half the FMA-pipe issue slots, which bound the fc1
// epilogue and with it the gap between two tiles' MMAs.
__device__ __forceinline__ uint32_t swiglu_bf16x2(float g0, float g1, float u0, float u1) {
  const float e0 = __expf(-fmaxf(g0, -80.0f)), e1 = __expf(-fmaxf(g1, -80.0f));
  const uint64_t one = f32x2_pack(1.0f, 1.0f);
  const uint64_t d = f32x2_add(one, f32x2_pack(e0, e1));
  float d0, d1;
  f32x2_unpack(d, d0, d1);
  uint64_t r = f32x2_pack(__int_as_float(kRcpSeed - __float_as_int(d0)),
                          __int_as_float(kRcpSeed - __float_as_int(d1)));
  const uint64_t nd = f32x2_pack(-d0, -d1);
#pragma unroll
  for (int i = 0; i < 3; ++i) r = f32x2_fma(r, f32x2_fma(nd, r, one), r);
  float h0, h1;
  f32x2_unpack(f32x2_mul(f32x2_mul(f32x2_pack(g0, g1), r), f32x2_pack(u0, u1)), h0, h1);
  return bf16x2_bits(h0, h1);
}

// Scale chunks of one stage, shared memory -> TMEM (in order with the MMAs
// issued after them).  NVFP4: chunk kk of each weight operand and token chunk
// cb of MMA kk (at sf_b + 4 * (kk * SFB + cb)); MXFP8: one chunk per operand
// and token chunk.  Only the first NB token chunks are copied: a tile whose
// token rows lie in one 128-row chunk reads no other (NB = 1); NB is a
// compile-time count so that the copies stay straight-line (a data-dependent
// loop around tcgen05.cp measured several times slower).
template <bool PAIR, int NA, int SFB, int NB>
__device__ __forceinline__ void sf_copies_nvf4(uint32_t sf_a0, uint32_t sf_a1, uint32_t sf_b,
                                               uint32_t ssf, uint32_t cb_bytes) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    tmem_cp_sf_chunk_x<PAIR>(sf_a0 + 4 * kk, sdesc_sf_chunk(ssf + kk * 512));
    if (NA == 2) tmem_cp_sf_chunk_x<PAIR>(sf_a1 + 4 * kk, sdesc_sf_chunk(ssf + cb_bytes + kk * 512));
#pragma unroll
    for (int cb = 0; cb < NB; ++cb)
      tmem_cp_sf_chunk_x<PAIR>(sf_b + 4 * (kk * SFB + cb),
                               sdesc_sf_chunk(ssf + (NA + cb) * cb_bytes + kk * 512));
  }
}
template <bool PAIR, int NA, int NB>
__device__ __forceinline__ void sf_copies_mxf8(uint32_t sf_a0, uint32_t sf_a1, uint32_t sf_b,
                                               uint32_t ssf) {
  tmem_cp_sf_chunk_x<PAIR>(sf_a0, sdesc_sf_chunk(ssf));
  if (NA == 2) tmem_cp_sf_chunk_x<PAIR>(sf_a1, sdesc_sf_chunk(ssf + 512));
#pragma unroll
  for (int cb = 0; cb < NB; ++cb)
    tmem_cp_sf_chunk_x<PAIR>(sf_b + 4 * cb, sdesc_sf_chunk(ssf + (NA + cb) * 512));
}

// PAIR: the kernel runs as clusters of two CTAs; rank 0 issues M = 256 MMAs
// over both CTAs' shared memory (cta_group::2), each CTA loads its own 128
// weight rows and half of the tile's token rows, and the loads of both count
// on rank 0's full barrier.
// BWD (fc1, bf16 only): the backward's recomputation of a = X W1^T and
// u = X W3^T, both stored (see the fc2-shaped epilogue branch).
template <int MODE, int TILE_N, int DT, bool PAIR = false, bool BWD = false>
__global__ void __launch_bounds__(kGemmThreads, 1) grouped_gemm_kernel(
    const __grid_constant__ GemmParams p) {
  using C = GemmCfg<MODE, TILE_N, DT, PAIR>;
  static_assert(!BWD || (MODE == kFc1 && DT == kBF16), "the backward form is bf16 fc1");
  static_assert(!PAIR || MODE != kRouter, "CTA pairs serve fc1 and fc2");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = smem;
  uint8_t* stg = ring + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(stg + C::STG_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* acc_full = empty + C::STAGES;   // [ACC_BUFS]
  uint64_t* acc_empty = acc_full + 2;       // [ACC_BUFS]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // tile queue in the second half of the barrier area
  uint64_t* sched_full = reinterpret_cast<uint64_t*>(stg + C::STG_BYTES + 256);
  uint64_t* sched_empty = sched_full + kSched;
  volatile int* sched_u = reinterpret_cast<volatile int*>(sched_empty + kSched);
  int* prefix = reinterpret_cast<int*>(stg + C::STG_BYTES + C::BAR_BYTES);

  const int warp = warp_id();
  const int lane = lane_id();
  const int rank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const int n_groups = PAIR ? gridDim.x / 2 : gridDim.x;  // CTAs or CTA pairs
  const int group_id = PAIR ? blockIdx.x / 2 : blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      // pairs: both CTAs' epilogue warps release rank 0's accumulator barrier
      mbar_init(&acc_empty[b], PAIR ? 2 * kEpiWarps : kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < kSched; ++i) {
      mbar_init(&sched_full[i], 1);
      // consumers: rank 0's MMA thread and epilogue warps, rank 1's producer
      // and epilogue warps (one CTA: MMA thread and epilogue warps)
      mbar_init(&sched_empty[i], PAIR ? 2 * (1 + kEpiWarps) : 1 + kEpiWarps);
    }
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
    // (one cta_group per kernel: pair kernels use only cta_group::2 tcgen05 forms)
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  // everything above touches only this CTA's shared memory and TMEM; from here
  // on the kernel reads what the previous kernel wrote (token counts, rows).
  // An fc2 fed chunk by chunk does not wait for fc1 as a whole: the counts it
  // reads were final before fc1 let it launch, and its producer waits for each
  // chunk of h (chunk_done) before loading it.
  if (!(MODE == kFc2 && p.chunk_done != nullptr)) pdl_wait();
  pdl_trigger();
  if (warp == 2) {
    // prefix[e] = number of TILE_N-token chunks of experts < e
    const int E = p.E;
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int local = 0;
    for (int e = e0; e < e1; ++e) local += (__ldg(p.counts + e) + TILE_N - 1) / TILE_N;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int run = incl - local;
    if (lane == 0) prefix[0] = 0;
    for (int e = e0; e < e1; ++e) {
      run += (__ldg(p.counts + e) + TILE_N - 1) / TILE_N;
      prefix[e + 1] = run;
    }
  }
  tc_fence_before();
  // pairs: the peer's barriers and TMEM must exist before any cross-CTA access
  if (PAIR) cluster_sync_all(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int units_routed = (p.E > 0) ? prefix[p.E] * p.g[0].n_slabs : 0;
  const int units_dense = (p.dense_rows > 0)
                              ? ((p.dense_rows + TILE_N - 1) / TILE_N) * p.g[1].n_slabs *
                                    p.g[1].k_splits
                              : 0;
  const int units = units_routed + units_dense;
  TileQueue tq{sched_full, sched_empty, sched_u, 0, 0u, group_id, n_groups,
               p.unit_counter != nullptr};

  // gathered token rows: the whole producer warp issues the row gathers
  const bool warp_loads = !PAIR && (MODE == kFc1) && p.row_token != nullptr;
  if (PAIR && warp == 0) {
    // ---------------- TMA producer of a CTA pair (lane 0 of each CTA) ----------
    // Both CTAs walk the same tiles.  Each loads its 128 rows of every weight
    // operand, its half of the token rows (N/2 each) and all token scale chunks
    // (each CTA's TMEM needs every token's scales), and every load completes on
    // rank 0's full barrier, whose expected bytes count both CTAs.
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      constexpr uint32_t cb_bytes = C::SF_KCH * C::SF_CHUNK;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      while (ok) {
        const int u = (rank == 0) ? claim_tile<PAIR>(tq, p, units, abort_flag, ok)
                                  : next_tile<PAIR>(tq, p, units, rank, false, abort_flag);
        if (u >= units) break;
        const Tile t = decode_tile<MODE, TILE_N, DT, PAIR>(u, p, prefix, units_routed, rank);
        const int half = ((t.n_tok + 15) & ~15) / 2;  // token rows per CTA (multiple of 8)
        const int nbox = (half + kBoxRows - 1) / kBoxRows;
        const int nsfb = ((t.row0 & 127) + t.n_tok + 127) / 128;
        // identical in both CTAs; weight and scale rows past the expert read the
        // next expert's or the map's zero fill, and only feed masked outputs
        const uint32_t bytes = C::NA * C::A_BYTES + nbox * kBoxRows * 128 +
                               (DT != kBF16 ? (C::NA + nsfb) * cb_bytes : 0);
        const int kt_all = p.g[t.grp].k_tiles;
        const int tile_base = (t.a_row / kBM) * kt_all;
        const int kb4 = p.kb4[t.grp];
        if (MODE == kFc2 && p.chunk_done != nullptr) {
          if (!counter_wait(p.chunk_done + t.chunk_id, p.chunk_target[t.grp], abort_flag,
                            p.status)) { ok = false; break; }
          fence_proxy_async_global();
        }
        for (int kt = t.k_begin; kt < t.k_end; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status)) { ok = false; break; }
          const uint32_t fb = cluster_addr(&full[stage], 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * bytes);
          uint8_t* sa = ring + stage * C::STAGE_BYTES;
          tma_load_3d_pair(sa, &p.a0[t.grp], fb, 0, 0, tile_base + kt, pol_w);
          if (MODE == kFc1)
            tma_load_3d_pair(sa + C::A_BYTES, &p.a1[t.grp], fb, 0, 0, tile_base + kt, pol_w);
          else
            tma_load_3d_pair(sa + C::A_BYTES, &p.a0[t.grp], fb, 0, 0, tile_base + kt + kt_all,
                             pol_w);
          uint8_t* sb = sa + C::NA * C::A_BYTES;
          const int col = kt * (DT == kBF16 ? kBK : 128);
#pragma unroll
          for (int bx = 0; bx < C::B_ROWS / kBoxRows; ++bx)
            if (bx < nbox)
              tma_load_2d_pair(sb + bx * kBoxRows * 128, &p.b[t.grp], fb, col,
                               t.row0 + rank * half + bx * kBoxRows, pol_x);
          if (DT != kBF16) {
            uint8_t* ssf = sb + C::B_BYTES;
            const int ca = (t.a_row / 128) * kb4 + kt * C::SF_KCH;
            tma_load_2d_pair(ssf, &p.sfa0_map[t.grp], fb, 0, ca, pol_w);
            if (MODE == kFc1)
              tma_load_2d_pair(ssf + cb_bytes, &p.sfa1_map[t.grp], fb, 0, ca, pol_w);
            else
              tma_load_2d_pair(ssf + cb_bytes, &p.sfa0_map[t.grp], fb, 0, ca + kb4, pol_w);
#pragma unroll
            for (int cb = 0; cb < C::SFB_CHUNKS; ++cb)
              if (cb < nsfb)
                tma_load_2d_pair(ssf + (C::NA + cb) * cb_bytes, &p.sfb_map[t.grp], fb, 0,
                                 (t.row0 / 128 + cb) * kb4 + kt * C::SF_KCH, pol_x);
          }
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // No drain here: rank 0's MMA issuer waits for every stage either CTA loads
      // (or gives up after its own bounded wait), and the closing cluster barrier
      // keeps both CTAs resident until then.
    }
  } else if (warp == 0) {
    // ---------------- TMA producer (lane 0, or the whole warp when gathering) ----
    if (lane == 0 || warp_loads) {
      const uint64_t pol_w = l2_policy_evict_first();
      const uint64_t pol_x = l2_policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      int last_phase[C::STAGES];
#pragma unroll
      for (int s = 0; s < C::STAGES; ++s) last_phase[s] = -1;
      bool ok = true;
      while (ok) {
        int u = units;
        if (lane == 0) u = claim_tile<PAIR>(tq, p, units, abort_flag, ok);
        if (warp_loads) u = __shfl_sync(0xffffffffu, u, 0);
        if (u >= units) break;
        const Tile t = decode_tile<MODE, TILE_N, DT, PAIR>(u, p, prefix, units_routed);
        const bool gather = (MODE == kFc1) && t.grp == 0 && p.row_token != nullptr;
        // gathered rows: lane l owns tile rows [8l, 8l + 8); rows past the MMA's N
        // are not loaded, and rows between the tile's tokens and N repeat its first
        // token (those accumulator columns are never stored)
        const int n_load = (t.n_tok + 15) & ~15;
        int ids[8];
        if (gather) {
          const int first = __ldg(p.row_token + t.row0);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int j = lane * 8 + i;
            ids[i] = j < t.n_tok ? __ldg(p.row_token + t.row0 + j) : first;
          }
        }
        const int nbox = (t.n_tok + kBoxRows - 1) / kBoxRows;
        const int nsfb = ((t.row0 & 127) + t.n_tok + 127) / 128;
        // fc2's second 128-row slab may lie past the expert's last row (odd number of
        // slabs): its outputs are masked, and its scale chunk (no bounds check on a bulk
        // copy) is not loaded
        const bool slab1 = (MODE != kFc2) ||
                           (t.slab * C::SLAB_ROWS + kBM < p.g[t.grp].a_valid_rows);
        const int n_sfa = (MODE == kRouter) ? 1 : (slab1 ? 2 : 1);
        const uint32_t bytes = C::NA * C::A_BYTES + (gather ? n_load : nbox * kBoxRows) * 128 +
                               (DT != kBF16 ? (n_sfa + nsfb) * C::SF_KCH * C::SF_CHUNK : 0);
        if (MODE == kFc2 && p.chunk_done != nullptr) {  // lane 0 only (no gather in fc2)
          if (!counter_wait(p.chunk_done + t.chunk_id, p.chunk_target[t.grp], abort_flag,
                            p.status)) { ok = false; break; }
          fence_proxy_async_global();
        }
        for (int kt = t.k_begin; kt < t.k_end; ++kt) {
          // lane 0 waits and sets the expected bytes; the decision is shared so the
          // warp stays converged
          int okw = 1;
          if (lane == 0) {
            okw = mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status) ? 1 : 0;
            if (okw) mbar_arrive_expect_tx(&full[stage], bytes);
          }
          if (warp_loads) okw = __shfl_sync(0xffffffffu, okw, 0);
          if (!okw) { ok = false; break; }
          uint8_t* sa = ring + stage * C::STAGE_BYTES;
          if (gather) {
            uint8_t* sbg = sa + C::NA * C::A_BYTES;
            const int col = kt * (DT == kBF16 ? kBK : 128);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const int j = lane * 8 + g * 4;
              if (j < n_load)
                tma_gather4(sbg + j * 128, &p.b[0], &full[stage], col, ids[4 * g],
                            ids[4 * g + 1], ids[4 * g + 2], ids[4 * g + 3], pol_x);
            }
          }
          if (lane != 0) {
            if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
            continue;
          }
          if (MODE == kRouter) {
            tma_load_2d(sa, &p.a0[t.grp], &full[stage], kt * kBK, t.a_row, pol_w);
          } else {
            // tile-major weights: tile (row slab, k-step) is one contiguous 16 KB box
            const int kt_all = p.g[t.grp].k_tiles;
            const int tile0 = (t.a_row / kBM) * kt_all + kt;
            tma_load_3d(sa, &p.a0[t.grp], &full[stage], 0, 0, tile0, pol_w);
            if (MODE == kFc1)
              tma_load_3d(sa + C::A_BYTES, &p.a1[t.grp], &full[stage], 0, 0, tile0, pol_w);
            else
              tma_load_3d(sa + C::A_BYTES, &p.a0[t.grp], &full[stage], 0, 0, tile0 + kt_all,
                          pol_w);
          }
          uint8_t* sb = sa + C::NA * C::A_BYTES;
          // fixed-count loops with a predicate (straight-line async copies)
          if (!gather)
#pragma unroll
            for (int bx = 0; bx < TILE_N / kBoxRows; ++bx)
              if (bx < nbox) tma_load_2d(sb + bx * kBoxRows * 128, &p.b[t.grp], &full[stage],
                          kt * (DT == kBF16 ? kBK : 128), t.row0 + bx * kBoxRows, pol_x);
          if (DT != kBF16) {
            // scale chunks of this k-step (SF_KCH consecutive chunks per 128-row chunk):
            // A rows [a_row, +128) (and the second operand), then the token row chunks
            constexpr uint32_t cb_bytes = C::SF_KCH * C::SF_CHUNK;
            uint8_t* ssf = sb + C::B_BYTES;
            const int kb4 = p.kb4[t.grp];
            const int64_t ca = (static_cast<int64_t>(t.a_row) / 128) * kb4 + kt * C::SF_KCH;
            bulk_load(ssf, p.sfa0[t.grp] + ca * C::SF_CHUNK, cb_bytes, &full[stage], pol_w);
            if (MODE == kFc1)
              bulk_load(ssf + cb_bytes, p.sfa1[t.grp] + ca * C::SF_CHUNK, cb_bytes, &full[stage],
                        pol_w);
            else if (MODE == kFc2 && slab1)
              bulk_load(ssf + cb_bytes, p.sfa0[t.grp] + (ca + kb4) * C::SF_CHUNK, cb_bytes,
                        &full[stage], pol_w);
#pragma unroll
            for (int cb = 0; cb < C::SFB_CHUNKS; ++cb) if (cb < nsfb) {
              const int64_t cbi = (static_cast<int64_t>(t.row0) / 128 + cb) * kb4 + kt * C::SF_KCH;
              bulk_load(ssf + (C::NA + cb) * cb_bytes, p.sfb[t.grp] + cbi * C::SF_CHUNK, cb_bytes,
                        &full[stage], pol_x);
            }
          }
          last_phase[stage] = phase;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // Let in-flight copies land before the CTA can exit.
        for (int s = 0; s < C::STAGES; ++s)
          if (last_phase[s] >= 0) {
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(&full[s], last_phase[s]) &&
                   global_timer_ns() - t0 < 20000000ull) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // (pairs: rank 0 only; its MMAs span both CTAs)
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      constexpr int M_MMA = PAIR ? 2 * kBM : kBM;
      while (ok) {
        const int u = next_tile<PAIR>(tq, p, units, 0, false, abort_flag);
        if (u >= units) break;
        const Tile t = decode_tile<MODE, TILE_N, DT, PAIR>(u, p, prefix, units_routed, 0);
        const int n_mma = (t.n_tok + 15) & ~15;
        const uint32_t idesc = idesc_bf16(M_MMA, n_mma);
        // token j's scale sits at chunk row (row0 % 128) + j: shift the TMEM base
        const uint32_t sfb_shift = static_cast<uint32_t>((t.row0 & 127) >> 5);
        // the MMA reads token scales of rows (row0 % 128) .. + n_mma - 1
        const bool one_chunk = (t.row0 & 127) + n_mma <= 128;
        const uint32_t d0 = tmem_base + acc * C::ACC_COLS;
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        for (int kt = t.k_begin; kt < t.k_end; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(ring + stage * C::STAGE_BYTES);
          const uint32_t sb = sa + C::NA * C::A_BYTES;
          const uint64_t da0 = sdesc_kmajor_sw128(sa);
          const uint64_t da1 = sdesc_kmajor_sw128(sa + C::A_BYTES);
          const uint64_t db = sdesc_kmajor_sw128(sb);
          if (DT == kBF16) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t accum = (kt > t.k_begin || kk) ? 1u : 0u;
              // advance 16 bf16 = 32 bytes along K inside the swizzle atom
              mma_bf16_x<PAIR>(d0, da0 + 2 * kk, db + 2 * kk, idesc, accum);
              if (C::NA == 2) mma_bf16_x<PAIR>(d0 + TILE_N, da1 + 2 * kk, db + 2 * kk, idesc, accum);
            }
          } else if (DT == kNVF4) {
            // scale factors: chunk kk of each operand feeds MMA kk (one 32-bit word
            // of four 16-element block scales per row); token row chunk cb of MMA kk
            // sits at sf_b + 4 * (kk * SFB_CHUNKS + cb)
            constexpr uint32_t cb_bytes = C::SF_KCH * C::SF_CHUNK;
            const uint32_t ssf = sb + C::B_BYTES;
            const uint32_t sf_a0 = tmem_base + C::SF_TMEM + (C::SF_BUFS == 2 ? (kt & 1) : 0) * C::SF_COLS;
            const uint32_t sf_a1 = sf_a0 + 4 * C::SF_KCH;
            const uint32_t sf_b = sf_a0 + 4 * C::SF_KCH * C::NA;
            // a multi-chunk tile copies every token chunk slot, also past the ones
            // its rows reach (those slots feed only columns that are never stored)
            if (one_chunk)
              sf_copies_nvf4<PAIR, C::NA, C::SFB_CHUNKS, 1>(sf_a0, sf_a1, sf_b, ssf, cb_bytes);
            else
              sf_copies_nvf4<PAIR, C::NA, C::SFB_CHUNKS, C::SFB_CHUNKS>(sf_a0, sf_a1, sf_b, ssf,
                                                                       cb_bytes);
            const uint32_t id = idesc_nvf4(M_MMA, n_mma);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t accum = (kt > t.k_begin || kk) ? 1u : 0u;
              const uint32_t sfb = sf_b + 4 * kk * C::SFB_CHUNKS + sfb_shift;
              // advance 64 e2m1 = 32 bytes along K
              mma_nvf4_x<PAIR>(d0, da0 + 2 * kk, db + 2 * kk, id, sf_a0 + 4 * kk, sfb, accum);
              if (C::NA == 2)
                mma_nvf4_x<PAIR>(d0 + TILE_N, da1 + 2 * kk, db + 2 * kk, id, sf_a1 + 4 * kk, sfb, accum);
            }
          } else {
            // scale factors of this stage: smem -> TMEM (in order with the MMAs below)
            const uint32_t ssf = sb + C::B_BYTES;
            const uint32_t sf_a0 = tmem_base + C::SF_TMEM + (C::SF_BUFS == 2 ? (kt & 1) : 0) * C::SF_COLS;
            const uint32_t sf_a1 = sf_a0 + 4;
            const uint32_t sf_b = sf_a0 + 4 * C::NA;
            if (one_chunk) sf_copies_mxf8<PAIR, C::NA, 1>(sf_a0, sf_a1, sf_b, ssf);
            else sf_copies_mxf8<PAIR, C::NA, C::SFB_CHUNKS>(sf_a0, sf_a1, sf_b, ssf);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t accum = (kt > t.k_begin || kk) ? 1u : 0u;
              const uint32_t id = idesc_mxf8(M_MMA, n_mma, kk);
              const uint32_t byte = static_cast<uint32_t>(kk) << 30;
              // advance 32 e4m3 = 32 bytes along K; k-block kk of the scale words
              const uint32_t sfb = (sf_b + sfb_shift) | byte;
              mma_mxf8_x<PAIR>(d0, da0 + 2 * kk, db + 2 * kk, id, sf_a0 | byte, sfb, accum);
              if (C::NA == 2)
                mma_mxf8_x<PAIR>(d0 + TILE_N, da1 + 2 * kk, db + 2 * kk, id, sf_a1 | byte, sfb, accum);
            }
          }
          commit_x<PAIR>(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        commit_x<PAIR>(&acc_full[acc]);
        if (++acc == C::ACC_BUFS) { acc = 0; acc_phase ^= 1; }
      }
      // Drain: all issued MMAs complete before TMEM is released.
      if constexpr (PAIR) mma_commit_pair(cluster_addr(drain, 0)); else mma_commit(drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < 20000000ull) {
      }
    }
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    const int quarter = warp & 3;          // TMEM lane quarter this warp may access
    const int member = (warp - 2) >> 2;    // which of the quarter's two warps
    uint8_t* my_stg = stg + (warp - 2) * C::STG_WARP;
    int acc = 0;
    uint32_t acc_phase = 0;
    while (true) {
      const int u = next_tile<PAIR>(tq, p, units, rank, true, abort_flag);
      if (u >= units) break;
      const Tile t = decode_tile<MODE, TILE_N, DT, PAIR>(u, p, prefix, units_routed, rank);
      // per-tile values in registers, loaded while the MMAs still run: the
      // parameter block is reached through a generic pointer once indexed by
      // t.grp, and loads through it could not be hoisted past the epilogue's
      // global stores
      const GemmGroup G = p.g[t.grp];
      uint8_t* const q_out = p.q_out[t.grp];
      uint8_t* const q_sf = p.q_sf[t.grp];
      float* const amax_out = p.amax_out[t.grp] + t.e * p.amax_stride[t.grp];
      const uint32_t lane_addr =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * C::ACC_COLS;
      const int f_base = t.f0 + quarter * 32;
      // NVFP4: undo the global encode scales of both operands
      float alpha = 1.0f;
      if (DT == kNVF4)
        alpha = 1.0f / (__ldg(p.ga[t.grp] + t.e * p.ga_stride[t.grp]) *
                        __ldg(p.gw[t.grp] + t.e * p.gw_stride[t.grp]));
      if (!mbar_wait(&acc_full[acc], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      float hmax = 0.f;  // fc1 NVFP4: amax of this warp's bf16 h values
      if constexpr (MODE == kFc1 && DT != kMXF8 && !BWD) {
        // h of this warp's chunks (32 tokens each) goes from TMEM straight into
        // registers as bf16 pairs, the accumulator is released, and only then
        // are the rows staged and stored: the next tile's MMAs wait for the
        // TMEM reads and the SwiGLU, not for the stores
        constexpr int NCH = (TILE_N + 63) / 64;
        uint32_t hp[NCH][16];
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          const int c0 = member * 32 + 64 * i;
          if (c0 < t.n_tok) {
            const int rows_here = min(32, t.n_tok - c0);
            uint32_t r0[32], r1[32];
            tmem_ld_32x32b_x32(lane_addr + c0, r0);
            tmem_ld_32x32b_x32(lane_addr + TILE_N + c0, r1);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              float g0 = __uint_as_float(r0[j]), g1 = __uint_as_float(r0[j + 1]);
              float u0 = __uint_as_float(r1[j]), u1 = __uint_as_float(r1[j + 1]);
              if constexpr (DT == kNVF4) {  // bf16: alpha is 1
                g0 *= alpha; g1 *= alpha; u0 *= alpha; u1 *= alpha;
              }
              const uint32_t w = swiglu_bf16x2(g0, g1, u0, u1);
              if (DT == kNVF4) {  // bf16 -> fp32 is a shift
                if (j < rows_here) hmax = fmaxf(hmax, fabsf(__uint_as_float(w << 16)));
                if (j + 1 < rows_here) hmax = fmaxf(hmax, fabsf(__uint_as_float(w & 0xFFFF0000u)));
              }
              hp[i][j >> 1] = w;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR) mbar_arrive_cluster(cluster_addr(&acc_empty[acc], 0));  // rank 0's barrier
          else mbar_arrive(&acc_empty[acc]);
        }
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(G.out);
        const uint4* s4 = reinterpret_cast<const uint4*>(my_stg);
        uint16_t* s = reinterpret_cast<uint16_t*>(my_stg);
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          const int c0 = member * 32 + 64 * i;
          if (c0 < t.n_tok) {
            const int rows_here = min(32, t.n_tok - c0);
            // staged [32 tokens][32 features], then 16-byte row stores
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              s[j * 32 + lane] = static_cast<uint16_t>(hp[i][j >> 1] & 0xFFFFu);
              s[(j + 1) * 32 + lane] = static_cast<uint16_t>(hp[i][j >> 1] >> 16);
            }
            __syncwarp();
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int c = it * 32 + lane;
              const int j = c >> 2, part = c & 3;
              if (j < rows_here && f_base < G.a_valid_rows)
                *reinterpret_cast<uint4*>(out + static_cast<int64_t>(t.row0 + c0 + j) * G.out_ld +
                                          f_base + part * 8) = s4[j * 4 + part];
            }
            __syncwarp();
          }
        }
        if (DT == kNVF4) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
            hmax = fmaxf(hmax, __shfl_xor_sync(0xffffffffu, hmax, o));
          if (lane == 0 && hmax > 0.f && f_base < G.a_valid_rows)
            atomic_max_nonneg(amax_out, hmax);
        }
        signal_chunk(p, t, lane);
        if (++acc == C::ACC_BUFS) { acc = 0; acc_phase ^= 1; }
      } else if constexpr (MODE == kFc2 || (MODE == kFc1 && DT == kMXF8) || BWD) {
        // As above: TMEM -> registers (packed bf16), release the accumulator,
        // then stage and store.  fc2 keeps both 128-feature halves of its chunks
        // (128 registers for 256-token tiles, which therefore read 16 columns
        // at a time: 16 raw registers live instead of 64, within the 168 a
        // thread gets); MXFP8 fc1 keeps h, quantized after the release.  The
        // backward form of fc1 stores its two accumulators, a and u, as the two
        // halves: a at the feature's column of `out`, u bwd_u_col further.
        constexpr bool TWO = (MODE == kFc2) || BWD;
        constexpr int NCH = (TILE_N + 63) / 64;
        constexpr int NH = TWO ? 2 : 1;
        uint32_t hp[NCH][NH][16];
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          const int c0 = member * 32 + 64 * i;
          if (TWO && TILE_N > 192 && c0 < t.n_tok) {
#pragma unroll
            for (int q = 0; q < 2 * NH; ++q) {  // (half, 16-column part)
              uint32_t r[16];
              tmem_ld_32x32b_x16(lane_addr + (q >> 1) * TILE_N + c0 + (q & 1) * 16, r);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 16; j += 2)
                hp[i][q >> 1][(q & 1) * 8 + (j >> 1)] =
                    bf16x2_bits(__uint_as_float(r[j]) * alpha, __uint_as_float(r[j + 1]) * alpha);
            }
          } else if (c0 < t.n_tok) {
            uint32_t r0[32], r1[32];
            tmem_ld_32x32b_x32(lane_addr + c0, r0);
            tmem_ld_32x32b_x32(lane_addr + TILE_N + c0, r1);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              if (TWO) {
                hp[i][0][j >> 1] = bf16x2_bits(__uint_as_float(r0[j]) * alpha,
                                               __uint_as_float(r0[j + 1]) * alpha);
                hp[i][NH - 1][j >> 1] = bf16x2_bits(__uint_as_float(r1[j]) * alpha,
                                                    __uint_as_float(r1[j + 1]) * alpha);
              } else {
                hp[i][0][j >> 1] = swiglu_bf16x2(__uint_as_float(r0[j]), __uint_as_float(r0[j + 1]),
                                                 __uint_as_float(r1[j]), __uint_as_float(r1[j + 1]));
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR) mbar_arrive_cluster(cluster_addr(&acc_empty[acc], 0));  // rank 0's barrier
          else mbar_arrive(&acc_empty[acc]);
        }
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          const int c0 = member * 32 + 64 * i;
          if (c0 >= t.n_tok) continue;
          const int rows_here = min(32, t.n_tok - c0);
          if constexpr (TWO) {
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(G.out);
            const uint4* s4 = reinterpret_cast<const uint4*>(my_stg);
            uint16_t* s16 = reinterpret_cast<uint16_t*>(my_stg);
#pragma unroll
            for (int half = 0; half < NH; ++half) {
              const int f0 = f_base + half * (BWD ? p.bwd_u_col[t.grp] : kBM);
              const bool fvalid = (BWD ? f_base : f0) < G.a_valid_rows;
#pragma unroll
              for (int j = 0; j < 32; j += 2) {
                s16[j * 32 + lane] = static_cast<uint16_t>(hp[i][half][j >> 1] & 0xFFFFu);
                s16[(j + 1) * 32 + lane] = static_cast<uint16_t>(hp[i][half][j >> 1] >> 16);
              }
              __syncwarp();
#pragma unroll
              for (int it = 0; it < 4; ++it) {
                const int c = it * 32 + lane;
                const int j = c >> 2, part = c & 3;
                if (j < rows_here && fvalid)
                  *reinterpret_cast<uint4*>(out + static_cast<int64_t>(t.row0 + c0 + j) *
                                                      G.out_ld + f0 + part * 8) = s4[j * 4 + part];
              }
              __syncwarp();
            }
          } else {
            // h staged [32 tokens][32 features] (row stride 34 bf16 to spread banks);
            // then lane j takes token j: the warp's 32 features are one MXFP8 block,
            // quantized from registers without cross-lane work
            constexpr int RS = 34;
            uint16_t* hs16 = reinterpret_cast<uint16_t*>(my_stg);
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              hs16[j * RS + lane] = static_cast<uint16_t>(hp[i][0][j >> 1] & 0xFFFFu);
              hs16[(j + 1) * RS + lane] = static_cast<uint16_t>(hp[i][0][j >> 1] >> 16);
            }
            __syncwarp();
            if (lane < rows_here && f_base < G.a_valid_rows) {
              float v[32];
              float amax = 0.f;
              const __nv_bfloat162* row =
                  reinterpret_cast<const __nv_bfloat162*>(hs16 + lane * RS);
#pragma unroll
              for (int q = 0; q < 16; ++q) {
                const float2 f = __bfloat1622float2(row[q]);
                v[2 * q] = f.x;
                v[2 * q + 1] = f.y;
                amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
              }
              const uint32_t code = mx_scale_code(amax);
              const float inv = mx_inv_scale(code);
              uint32_t w[8];
#pragma unroll
              for (int q = 0; q < 8; ++q)
                w[q] = static_cast<uint32_t>(to_e4m3(v[4 * q] * inv)) |
                       (static_cast<uint32_t>(to_e4m3(v[4 * q + 1] * inv)) << 8) |
                       (static_cast<uint32_t>(to_e4m3(v[4 * q + 2] * inv)) << 16) |
                       (static_cast<uint32_t>(to_e4m3(v[4 * q + 3] * inv)) << 24);
              const int64_t r = t.row0 + c0 + lane;
              uint4* dst = reinterpret_cast<uint4*>(q_out + r * G.out_ld + f_base);
              dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
              dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
              q_sf[sf_offset(r, f_base / 32, static_cast<int>(G.out_ld) / 32)] =
                  static_cast<uint8_t>(code);
            }
            __syncwarp();
          }
        }
        if constexpr (MODE == kFc1) signal_chunk(p, t, lane);
        if (++acc == C::ACC_BUFS) { acc = 0; acc_phase ^= 1; }
      } else {
        // router logits, the one mode left: thread = expert, register j = token
        // (32 consecutive fp32 per token), into the tile's K-split partials
        static_assert(MODE == kRouter, "fc1 and fc2 release their accumulator early");
        float* out = static_cast<float*>(G.out) + t.split * G.split_stride;
        const int e = f_base + lane;
        for (int c0 = member * 32; c0 < t.n_tok; c0 += 64) {
          const int rows_here = min(32, t.n_tok - c0);
          uint32_t r0[32];
          tmem_ld_32x32b_x32(lane_addr + c0, r0);
          tmem_ld_wait();
          if (e < G.a_valid_rows) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < rows_here)
                out[static_cast<int64_t>(t.row0 + c0 + j) * G.out_ld + e] = __uint_as_float(r0[j]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
        if (++acc == C::ACC_BUFS) { acc = 0; acc_phase ^= 1; }
      }
    }
  }

  tc_fence_before();
  // pairs: neither CTA leaves while the other may still touch its shared memory,
  // barriers or TMEM
  if (PAIR) cluster_sync_all(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace moe
