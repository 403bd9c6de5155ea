// C ABI entry points: argument checks, workspace layout, TMA descriptors and
// kernel launches.  See include/moe_b200.h for the contract of each call.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "backward.cuh"
#include "grouped_gemm.cuh"
#include "prepare.cuh"
#include "quantize.cuh"
#include "route_permute_combine.cuh"
#include "wgrad.cuh"

using namespace moe;

namespace {

constexpr size_t kAlign = 256;

inline size_t align_up(size_t v, size_t a = kAlign) { return (v + a - 1) / a * a; }
inline int64_t pad128(int64_t v) { return (v + 127) / 128 * 128; }

// ---------------------------------------------------------------------------
// Workspace layout of the step calls.
// ---------------------------------------------------------------------------
struct StepLayout {
  // h: fc1 output (bf16; MXFP8: e4m3 codes); h_q: NVFP4 codes of h; h_sf: scales
  size_t status, hist, h, h_q, h_sf, h_shared, h_shared_q, h_shared_sf, g_h, chunk_done,
      router_partials, total;
  int32_t r_cap, ntiles, router_splits;
};

// Router GEMM tiling: 256-token tiles for long batches (W_r re-read per tile
// is then negligible), 64 otherwise; K split into at most kMaxSplits parts,
// the count that minimises the rounds of units over the 148 SMs times the
// k-steps of one unit (ties to fewer splits: less partial-sum traffic).
int router_tile_of(const moe_config& c) { return c.T >= 4096 ? 256 : 64; }

int router_splits_of(const moe_config& c) {
  const int tn = router_tile_of(c);
  const int units = ((c.T + tn - 1) / tn) * ((c.E + kBM - 1) / kBM);
  const int k_tiles = c.H / kBK;
  int best = 1;
  int64_t best_cost = -1;
  for (int s = 1; s <= kMaxSplits && s <= (k_tiles / 4 > 0 ? k_tiles / 4 : 1); ++s) {
    const int64_t rounds = (static_cast<int64_t>(units) * s + 147) / 148;
    const int64_t cost = rounds * ((k_tiles + s - 1) / s);
    if (best_cost < 0 || cost < best_cost) { best = s; best_cost = cost; }
  }
  return best;
}

// Upper bound on the token chunks of the grouped GEMMs (tiles of at least 64
// tokens): each expert's ceil(count / TILE_N) summed over experts, plus the
// dense group's.
int max_token_chunks(const moe_config& c) {
  return c.E + (c.T * c.top_k) / 64 + 1 + (c.T + 63) / 64;
}

// fc1 and fc2 CTAs claim their tiles from a counter (MOE_DYNAMIC_TILES=0:
// CTA i takes tiles i, i + grid, ...).
bool dynamic_tiles() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("MOE_DYNAMIC_TILES");
    v = (e && atoi(e) == 0) ? 0 : 1;
  }
  return v == 1;
}

// Failure-path test hook: MOE_TEST_FC2_NEVER_READY=1 (read on every call)
// raises fc2's chunk targets by one, a count fc1 never reaches, so every fc2
// producer's bounded wait runs out, the kernel records MOE_ERR_TIMEOUT and
// exits in order.  Nothing sets it outside that test.
bool test_fc2_never_ready() {
  const char* e = getenv("MOE_TEST_FC2_NEVER_READY");
  return e && atoi(e) == 1;
}

// fc2 starts on the SMs fc1 frees and waits per token chunk (bf16, MXFP8;
// NVFP4 quantizes h between the two).  MOE_FC2_EARLY=0 makes fc2 wait for fc1
// as a whole instead.
bool fc2_early(const moe_config& c) {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("MOE_FC2_EARLY");
    v = (e && atoi(e) == 0) ? 0 : 1;
  }
  return v == 1 && c.dtype != MOE_NVFP4;
}

int32_t r_cap_of(const moe_config& c) {
  const int64_t P = c.pad_multiple;
  const int64_t r = static_cast<int64_t>(c.T) * c.top_k + static_cast<int64_t>(c.E) * (P - 1);
  return static_cast<int32_t>((r + P - 1) / P * P);
}

StepLayout step_layout(const moe_config& c) {
  StepLayout L;
  L.r_cap = r_cap_of(c);
  L.ntiles = (c.T * c.top_k + kPermTile - 1) / kPermTile;
  size_t o = 0;
  L.status = o; o = align_up(o + 4);
  L.hist = o; o = align_up(o + static_cast<size_t>(L.ntiles) * c.E * 4);
  const bool mx = c.dtype == MOE_MXFP8, nv = c.dtype == MOE_NVFP4;
  const size_t eb = mx ? 1 : 2;  // bytes per element of h as fc1 writes it
  const size_t Is = c.I_shared > 0 ? c.I_shared : 0;
  const size_t Tp = static_cast<size_t>(pad128(c.T));
  const size_t Rp = static_cast<size_t>(pad128(L.r_cap));
  const size_t blk = mx ? 32 : 16;  // elements per scale
  L.h = o; o = align_up(o + static_cast<size_t>(L.r_cap) * c.I * eb);
  L.h_q = o; o = align_up(o + (nv ? static_cast<size_t>(L.r_cap) * c.I / 2 : 0));
  L.h_sf = o; o = align_up(o + ((mx || nv) ? Rp * c.I / blk : 0));
  L.h_shared = o; o = align_up(o + Tp * Is * eb);
  L.h_shared_q = o; o = align_up(o + (nv ? Tp * Is / 2 : 0));
  L.h_shared_sf = o; o = align_up(o + ((mx || nv) ? Tp * Is / blk : 0));
  L.g_h = o; o = align_up(o + (nv ? (static_cast<size_t>(c.E) + 1) * 4 : 0));
  // two tile-claim counters (fc1, fc2), then the per-chunk counters
  L.chunk_done = o; o = align_up(o + (2 + static_cast<size_t>(max_token_chunks(c))) * 4);
  L.router_splits = router_splits_of(c);
  L.router_partials = o;
  o = align_up(o + static_cast<size_t>(L.router_splits) * c.T * c.E * 4);
  L.total = o;
  return L;
}

struct FwdLayout {
  StepLayout step;
  size_t logits, topk_idx, topk_w, counts, offsets, row_token, token_row, rows, rows_sf,
      out_rows, shared_out, x, x_q, x_sf, x_g, y, total;
};

FwdLayout fwd_layout(const moe_config& c) {
  FwdLayout F;
  F.step = step_layout(c);
  const size_t T = c.T, H = c.H, E = c.E, k = c.top_k, R = F.step.r_cap;
  size_t o = F.step.total;
  F.logits = o; o = align_up(o + T * E * 4);
  F.topk_idx = o; o = align_up(o + T * k * 4);
  F.topk_w = o; o = align_up(o + T * k * 4);
  F.counts = o; o = align_up(o + E * 4);
  F.offsets = o; o = align_up(o + (E + 1) * 4);
  F.row_token = o; o = align_up(o + R * 4);
  F.token_row = o; o = align_up(o + T * k * 4);
  const bool mx = c.dtype == MOE_MXFP8, nv = c.dtype == MOE_NVFP4, q = mx || nv;
  const size_t Tp = static_cast<size_t>(pad128(c.T));
  const size_t row_b = mx ? H : (nv ? H / 2 : 2 * H);  // bytes per permuted row
  const size_t sf_b = mx ? H / 32 : H / 16;            // scale bytes per row
  F.rows = o; o = align_up(o + R * row_b);
  F.rows_sf = o; o = align_up(o + (q ? static_cast<size_t>(pad128(R)) * sf_b : 0));
  F.out_rows = o; o = align_up(o + R * H * 2);
  F.shared_out = o; o = align_up(o + (c.I_shared > 0 ? T * H * 2 : 0));
  F.x = o; o = align_up(o + T * H * 2);
  F.x_q = o; o = align_up(o + (q ? T * row_b : 0));
  F.x_sf = o; o = align_up(o + (q ? Tp * sf_b : 0));
  F.x_g = o; o = align_up(o + (nv ? 4 : 0));
  F.y = o; o = align_up(o + T * H * 2);
  F.total = o;
  return F;
}

moe_status check_config(const moe_config* c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  if (c->T < 1 || c->H < 1 || c->I < 1 || c->E < 1 || c->n_group < 1 || c->topk_group < 1 ||
      c->top_k < 1 || c->pad_multiple < 1 || c->I_shared < 0)
    return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_BF16 && c->dtype != MOE_MXFP8 && c->dtype != MOE_NVFP4)
    return MOE_ERR_INVALID_ARG;
  if (c->H % 128 || c->I % 128 || (c->I_shared % 128)) return MOE_ERR_UNSUPPORTED;
  if (c->E > kMaxExperts || c->E % c->n_group || c->E / c->n_group < 2 || c->n_group > 32)
    return MOE_ERR_UNSUPPORTED;
  if (c->topk_group > c->n_group) return MOE_ERR_UNSUPPORTED;
  if (c->top_k > 32 || c->top_k > c->topk_group * (c->E / c->n_group)) return MOE_ERR_UNSUPPORTED;
  const int64_t rcap = static_cast<int64_t>(c->T) * c->top_k +
                       static_cast<int64_t>(c->E) * (c->pad_multiple - 1);
  if (rcap > (int64_t(1) << 30)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Block-scaled paths need expert segments to start on 64-row boundaries: the
// GEMM shifts its TMEM scale base by (row % 128) / 32 columns, and that address
// must be even.  So pad_multiple % 64 == 0.  NVFP4 k-steps are 256 wide.
moe_status check_dtype(const moe_config* c) {
  if (c->dtype == MOE_BF16) return MOE_OK;
  if (c->pad_multiple % 64) return MOE_ERR_UNSUPPORTED;
  if (c->dtype == MOE_NVFP4 && (c->H % 256 || c->I % 256 || c->I_shared % 256))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

inline bool is_mx(const moe_config& c) { return c.dtype == MOE_MXFP8; }
inline bool is_nv(const moe_config& c) { return c.dtype == MOE_NVFP4; }
inline bool is_bf16(const moe_config& c) { return c.dtype == MOE_BF16; }

inline moe_status cuda_check(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  fprintf(stderr, "moe_b200: CUDA error %s\n", cudaGetErrorString(e));
  return MOE_ERR_CUDA;
}

#define MOE_TRY(expr)                      \
  do {                                     \
    moe_status _s = (expr);                \
    if (_s != MOE_OK) return _s;           \
  } while (0)

#define MOE_CUDA(expr) MOE_TRY(cuda_check(expr))

inline moe_status launch_check() { return cuda_check(cudaGetLastError()); }

// ---------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched through the runtime).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Programmatic dependent launch is on unless MOE_PDL=0 (plain stream order,
// e.g. for profilers that replay kernels one at a time).
bool pdl_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("MOE_PDL");
    v = (e && atoi(e) == 0) ? 0 : 1;
  }
  return v == 1;
}

// Launch with programmatic dependent launch allowed: the kernel's CTAs may
// start while the previous kernel in the stream is finishing (every library
// kernel waits in pdl_wait() before it touches global memory), which hides the
// gap between the many short kernels of one layer.
template <typename... KArgs, typename... Args>
moe_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                      Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  MOE_CUDA(cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...));
  return MOE_OK;
}

// 2-D K-major tile map over [rows, inner] elements with a 128-byte swizzle.
// The box is (128 bytes of K) x box_rows.
moe_status make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes,
                    uint64_t inner, uint64_t rows, uint64_t row_stride_bytes, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return MOE_ERR_CUDA;
  if (reinterpret_cast<uintptr_t>(base) % 16 || row_stride_bytes % 16) return MOE_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fprintf(stderr, "moe_b200: cuTensorMapEncodeTiled failed (%d)\n", static_cast<int>(r));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// 3-D map over a tile-major matrix of `rows` rows and `k_bytes` bytes per row:
// tiles of 128 rows x 128 bytes, box = one tile.
moe_status make_tiled_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t k_bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return MOE_ERR_CUDA;
  if (reinterpret_cast<uintptr_t>(base) % 16) return MOE_ERR_INVALID_ARG;
  cuuint64_t dims[3] = {128, 128, (rows / 128) * (k_bytes / 128)};
  cuuint64_t strides[2] = {128, 128 * 128};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fprintf(stderr, "moe_b200: cuTensorMapEncodeTiled (3-D) failed (%d)\n", static_cast<int>(r));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

// 2-D map over a block-scale buffer as rows of 512-byte chunks (uint32 x 128):
// a box of `box_rows` consecutive chunks; chunks past n_chunks read as zeros.
moe_status make_sf_map(CUtensorMap* m, const void* base, uint64_t n_chunks, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return MOE_ERR_CUDA;
  if (reinterpret_cast<uintptr_t>(base) % 16 || n_chunks < 1) return MOE_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {128, n_chunks};
  cuuint64_t strides[1] = {512};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    fprintf(stderr, "moe_b200: cuTensorMapEncodeTiled (scales) failed (%d)\n", static_cast<int>(r));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// One persistent CTA per SM, or (PAIR) one two-CTA cluster per SM pair, as
// many as can be resident at once, capped by the number of tiles.
template <int MODE, int TILE_N, int DT, bool PAIR = false, bool BWD = false>
moe_status launch_gemm(const GemmParams& p, int max_units, cudaStream_t s) {
  using C = GemmCfg<MODE, TILE_N, DT, PAIR>;
  auto kern = grouped_gemm_kernel<MODE, TILE_N, DT, PAIR, BWD>;
  MOE_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
  if (!PAIR) {
    int grid = sm_count();
    if (max_units < grid) grid = max_units;
    if (grid < 1) return MOE_OK;
    return launch_pdl(kern, dim3(grid), dim3(kGemmThreads), C::SMEM_BYTES, s, p);
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // as in launch_pdl
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kGemmThreads);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // cluster shape only for the occupancy query
  // resident clusters, once per device for this kernel
  static int cached[64];
  static std::mutex mu;
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  int n = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 0 && dev < 64 && cached[dev] > 0) {
      n = cached[dev];
    } else {
      cfg.gridDim = dim3(2 * (sm_count() / 2));
      MOE_CUDA(cudaOccupancyMaxActiveClusters(&n, kern, &cfg));
      if (dev >= 0 && dev < 64) cached[dev] = n;
    }
  }
  if (n < 1) return MOE_ERR_UNSUPPORTED;
  int clusters = n < max_units ? n : max_units;
  if (clusters < 1) return MOE_OK;
  cfg.gridDim = dim3(2 * clusters);
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  MOE_CUDA(cudaLaunchKernelEx(&cfg, kern, p));
  return launch_check();
}

int32_t* status_ptr(void* ws) { return static_cast<int32_t*>(ws); }

// ---------------------------------------------------------------------------
// Step implementations (arguments already validated).
// ---------------------------------------------------------------------------
moe_status do_route(const moe_config& c, const void* x, const void* w_router, const float* bias,
                    const float* logits_in, float* logits_out, int32_t* topk_idx, float* topk_w,
                    void* ws, cudaStream_t s) {
  SelArgs a;
  memset(&a, 0, sizeof(a));
  if (!logits_in) {
    const StepLayout L = step_layout(c);
    float* partials = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + L.router_partials);
    GemmParams p;
    memset(&p, 0, sizeof(p));
    MOE_TRY(make_map(&p.a0[1], w_router, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c.H, c.E,
                     static_cast<uint64_t>(c.H) * 2, kBM));
    MOE_TRY(make_map(&p.b[1], x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c.H, c.T,
                     static_cast<uint64_t>(c.H) * 2, kBoxRows));
    p.a0[0] = p.a1[0] = p.a1[1] = p.a0[1];
    p.b[0] = p.b[1];
    GemmGroup g;
    g.a_rows_per_expert = 0;
    g.a_valid_rows = c.E;
    g.n_slabs = (c.E + kBM - 1) / kBM;
    g.k_tiles = c.H / kBK;
    g.k_splits = L.router_splits;
    g.out = partials;
    g.out_ld = c.E;
    g.split_stride = static_cast<int64_t>(c.T) * c.E;
    p.g[0] = p.g[1] = g;
    p.E = 0;
    p.dense_rows = c.T;
    p.status = status_ptr(ws);
    const int tn = router_tile_of(c);
    const int units = ((c.T + tn - 1) / tn) * g.n_slabs * g.k_splits;
    if (tn == 256) MOE_TRY((launch_gemm<kRouter, 256, kBF16>(p, units, s)));
    else MOE_TRY((launch_gemm<kRouter, 64, kBF16>(p, units, s)));
    a.partials = partials;
    a.n_splits = L.router_splits;
    a.logits_out = logits_out;
  } else {
    a.logits = logits_in;
    a.n_splits = 0;
  }
  a.bias = bias;
  a.topk_idx = topk_idx;
  a.topk_w = topk_w;
  a.T = c.T;
  a.E = c.E;
  a.G = c.n_group;
  a.g = c.topk_group;
  a.k = c.top_k;
  a.rsf = c.routed_scaling_factor;
  a.gs_magic = static_cast<uint32_t>(((1ull << 32) + (c.E / c.n_group) - 1) / (c.E / c.n_group));
  const int per = (c.E + 31) / 32;
  const dim3 grid((c.T + kSelWarps - 1) / kSelWarps), block(kSelWarps * 32);
  if (per <= 1) MOE_TRY(launch_pdl(route_select_kernel<1>, dim3(grid), dim3(block), 0, s, a));
  else if (per <= 2) MOE_TRY(launch_pdl(route_select_kernel<2>, dim3(grid), dim3(block), 0, s, a));
  else if (per <= 4) MOE_TRY(launch_pdl(route_select_kernel<4>, dim3(grid), dim3(block), 0, s, a));
  else if (per <= 8) MOE_TRY(launch_pdl(route_select_kernel<8>, dim3(grid), dim3(block), 0, s, a));
  else if (per <= 12) MOE_TRY(launch_pdl(route_select_kernel<12>, dim3(grid), dim3(block), 0, s, a));
  else if (per <= 16) MOE_TRY(launch_pdl(route_select_kernel<16>, dim3(grid), dim3(block), 0, s, a));
  else MOE_TRY(launch_pdl(route_select_kernel<32>, dim3(grid), dim3(block), 0, s, a));
  return launch_check();
}

// Histogram, padded offsets and the two row maps (no row is copied).
moe_status do_permute_maps(const moe_config& c, const int32_t* topk_idx, int32_t* counts,
                           int32_t* offsets, int32_t* row_token, int32_t* token_row, void* ws,
                           cudaStream_t s) {
  const StepLayout L = step_layout(c);
  PermArgs a;
  a.topk_idx = topk_idx;
  a.hist = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + L.hist);
  a.counts = counts;
  a.offsets = offsets;
  a.row_token = row_token;
  a.token_row = token_row;
  a.status = status_ptr(ws);
  a.n = c.T * c.top_k;
  a.k = c.top_k;
  a.E = c.E;
  a.P = c.pad_multiple;
  a.r_cap = L.r_cap;
  a.ntiles = L.ntiles;
  const size_t hsm = static_cast<size_t>(c.E) * 4;
  MOE_TRY(launch_pdl(permute_hist_kernel, dim3(L.ntiles), dim3(256), hsm, s, a));
  MOE_TRY(launch_check());
  MOE_TRY(launch_pdl(permute_scan_kernel, dim3((c.E + 7) / 8), dim3(256), 0, s, a));
  MOE_TRY(launch_check());
  MOE_TRY(launch_pdl(permute_rank_kernel, dim3(L.ntiles), dim3(256), 0, s, a));
  return launch_check();
}

moe_status do_permute(const moe_config& c, const int32_t* topk_idx, const void* src_rows,
                      const void* src_scales, int32_t* counts, int32_t* offsets,
                      int32_t* row_token, int32_t* token_row, void* dst_rows, void* dst_scales,
                      void* ws, cudaStream_t s) {
  const StepLayout L = step_layout(c);
  PermArgs a;
  a.topk_idx = topk_idx;
  a.hist = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + L.hist);
  a.counts = counts;
  a.offsets = offsets;
  a.row_token = row_token;
  a.token_row = token_row;
  a.status = status_ptr(ws);
  a.n = c.T * c.top_k;
  a.k = c.top_k;
  a.E = c.E;
  a.P = c.pad_multiple;
  a.r_cap = L.r_cap;
  a.ntiles = L.ntiles;
  const size_t hsm = static_cast<size_t>(c.E) * 4;
  MOE_TRY(launch_pdl(permute_hist_kernel, dim3(L.ntiles), dim3(256), hsm, s, a));
  MOE_TRY(launch_check());
  MOE_TRY(launch_pdl(permute_scan_kernel, dim3((c.E + 7) / 8), dim3(256), 0, s, a));
  MOE_TRY(launch_check());
  MOE_TRY(launch_pdl(permute_rank_kernel, dim3(L.ntiles), dim3(256), 0, s, a));
  MOE_TRY(launch_check());
  if (is_mx(c) || is_nv(c)) {
    GatherMxArgs g;
    g.src_codes = static_cast<const uint8_t*>(src_rows);
    g.src_scales = static_cast<const uint8_t*>(src_scales);
    g.dst_codes = static_cast<uint8_t*>(dst_rows);
    g.dst_scales = static_cast<uint8_t*>(dst_scales);
    g.row_token = row_token;
    g.offsets = offsets;
    g.E = c.E;
    g.H = c.H;
    const int row_bytes = is_nv(c) ? c.H / 2 : c.H;
    const int KB = is_nv(c) ? c.H / 16 : c.H / 32;
    const int vpl = (row_bytes / 16 + 31) / 32;  // 16-byte vectors per lane
    const dim3 grid(sm_count() * 4), block(256);
    if (KB / 4 <= 256 && vpl <= 8)
      MOE_TRY(launch_pdl(permute_gather_bs_kernel<8>, grid, block, 0, s, g, row_bytes, KB));
    else if (KB / 4 <= 256 && vpl <= 16)
      MOE_TRY(launch_pdl(permute_gather_bs_kernel<16>, grid, block, 0, s, g, row_bytes, KB));
    else if (is_nv(c))
      MOE_TRY(launch_pdl(permute_gather_nv_kernel, grid, block, 0, s, g));
    else
      MOE_TRY(launch_pdl(permute_gather_mx_kernel, grid, block, 0, s, g));
    return launch_check();
  }
  if (!dst_rows) return MOE_OK;  // rows are gathered later by the grouped GEMM
  GatherArgs g;
  g.src = static_cast<const uint8_t*>(src_rows);
  g.dst = static_cast<uint8_t*>(dst_rows);
  g.row_token = row_token;
  g.offsets = offsets;
  g.E = c.E;
  g.row_bytes = c.H * 2;
  const int vpl = (g.row_bytes / 16 + 31) / 32;  // 16-byte vectors per lane
  const dim3 grid(sm_count() * 4), block(256);
  if (vpl <= 8) MOE_TRY(launch_pdl(permute_gather_row_kernel<8>, grid, block, 0, s, g));
  else if (vpl <= 16) MOE_TRY(launch_pdl(permute_gather_row_kernel<16>, grid, block, 0, s, g));
  else if (vpl <= 32) MOE_TRY(launch_pdl(permute_gather_row_kernel<32>, grid, block, 0, s, g));
  else MOE_TRY(launch_pdl(permute_gather_kernel, grid, block, 0, s, g));
  return launch_check();
}

// Quantized inputs of the grouped MLP (MXFP8): row scales, token-order x codes
// and scales for the shared expert.
struct MlpQuant {
  const void* row_scales;
  const void* x_scales;
  const float* x_global;     // NVFP4 global encode scale of x
  const int32_t* row_token;  // with rows == nullptr: fc1 gathers token rows from x
};

// PAIR: fc1 and fc2 run as two-CTA clusters (M = 256 MMAs; each CTA holds
// half of a tile's token rows), which leaves room for a deeper load ring.
// The grouped MLP's counters (tile claims, fc1 -> fc2 chunks) and NVFP4's
// per-expert amax of h start every call at zero.  A memset between two kernels
// breaks their programmatic launch overlap, so the one-call forward issues it
// first, before the routing kernels, and tells the grouped MLP so.
moe_status zero_mlp_scratch(const moe_config& c, void* ws, cudaStream_t s) {
  const StepLayout L = step_layout(c);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  MOE_CUDA(cudaMemsetAsync(wsb + L.chunk_done, 0,
                           (2 + static_cast<size_t>(max_token_chunks(c))) * 4, s));
  if (c.dtype == MOE_NVFP4)
    MOE_CUDA(cudaMemsetAsync(wsb + L.g_h, 0, (static_cast<size_t>(c.E) + 1) * 4, s));
  return MOE_OK;
}

template <int TILE_N, int DT, bool PAIR>
moe_status grouped_mlp_tiles(const moe_config& c, const moe_weights& w, const void* rows,
                             const void* x, const MlpQuant& q, const int32_t* counts,
                             const int32_t* offsets, void* out_rows, void* shared_out, void* ws,
                             cudaStream_t s, bool scratch_zeroed) {
  const StepLayout L = step_layout(c);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  void* h = wsb + L.h;
  void* hs = wsb + L.h_shared;
  const bool sh = c.I_shared > 0;
  const bool mx = DT == kMXF8, nv = DT == kNVF4, qz = mx || nv;
  const auto tok_t = qz ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // operand bytes per K element (NVFP4 packs two per byte), map element bytes
  auto kbytes = [&](uint64_t k) -> uint64_t { return nv ? k / 2 : (mx ? k : 2 * k); };
  const int me = qz ? 1 : 2;                  // tensor-map element bytes
  const int kstep = nv ? 256 : (mx ? 128 : kBK);  // K elements per k-step
  const int kb4_div = nv ? 64 : 128;          // K elements per scale chunk column
  float* g_h = reinterpret_cast<float*>(wsb + L.g_h);
  if (!scratch_zeroed) MOE_TRY(zero_mlp_scratch(c, ws, s));
  const bool early = fc2_early(c);
  const bool dyn = dynamic_tiles();
  int32_t* unit_counters = reinterpret_cast<int32_t*>(wsb + L.chunk_done);
  int32_t* chunk_done = unit_counters + 2;
  int fc1_slabs[2] = {0, 0};
  const uint64_t H = c.H, I = c.I, Is = c.I_shared, E = c.E, T = c.T;
  const int max_chunks = c.E + (c.T * c.top_k) / TILE_N + 1;
  const int dense_chunks = (c.T + TILE_N - 1) / TILE_N;
  constexpr int span1 = GemmCfg<kFc1, TILE_N, DT, PAIR>::SLAB_SPAN;  // features per fc1 tile
  constexpr int span2 = GemmCfg<kFc2, TILE_N, DT, PAIR>::SLAB_SPAN;  // features per fc2 tile
  constexpr uint32_t sf_box = DT == kNVF4 ? 4 : 1;                    // scale chunks per k-step
  const uint64_t Rp128 = static_cast<uint64_t>(pad128(L.r_cap)) / 128;
  const uint64_t Tp128 = static_cast<uint64_t>(pad128(c.T)) / 128;
  // fc1 + SwiGLU: one 128-feature slab of W1 and of W3 per tile
  {
    GemmParams p;
    memset(&p, 0, sizeof(p));
    MOE_TRY(make_tiled_map(&p.a0[0], w.w1, E * I, kbytes(H)));
    MOE_TRY(make_tiled_map(&p.a1[0], w.w3, E * I, kbytes(H)));
    if (rows) {
      MOE_TRY(make_map(&p.b[0], rows, tok_t, me, kbytes(H) / me, L.r_cap, kbytes(H), kBoxRows));
    } else {
      // gathered: one-row boxes over token-order x, rows picked by row_token
      MOE_TRY(make_map(&p.b[0], x, tok_t, me, kbytes(H) / me, c.T, kbytes(H), 1));
      p.row_token = q.row_token;
    }
    if (sh) {
      MOE_TRY(make_tiled_map(&p.a0[1], w.ws1, Is, kbytes(H)));
      MOE_TRY(make_tiled_map(&p.a1[1], w.ws3, Is, kbytes(H)));
      MOE_TRY(make_map(&p.b[1], x, tok_t, me, kbytes(H) / me, T, kbytes(H), kBoxRows));
    } else {
      p.a0[1] = p.a0[0];
      p.a1[1] = p.a1[0];
      p.b[1] = p.b[0];
    }
    p.g[0] = GemmGroup{c.I, c.I, (c.I + span1 - 1) / span1, c.H / kstep, 1, h, c.I, 0};
    p.g[1] = GemmGroup{0, c.I_shared, (c.I_shared + span1 - 1) / span1, c.H / kstep, 1, hs,
                       c.I_shared, 0};
    if (qz) {
      p.sfa0[0] = static_cast<const uint8_t*>(w.w1_scales);
      p.sfa1[0] = static_cast<const uint8_t*>(w.w3_scales);
      p.sfb[0] = static_cast<const uint8_t*>(q.row_scales);
      p.sfa0[1] = static_cast<const uint8_t*>(w.ws1_scales);
      p.sfa1[1] = static_cast<const uint8_t*>(w.ws3_scales);
      p.sfb[1] = static_cast<const uint8_t*>(q.x_scales);
      p.kb4[0] = p.kb4[1] = c.H / kb4_div;
      if (PAIR) {
        const uint64_t kb4 = c.H / kb4_div;
        MOE_TRY(make_sf_map(&p.sfa0_map[0], w.w1_scales, E * I / 128 * kb4, sf_box));
        MOE_TRY(make_sf_map(&p.sfa1_map[0], w.w3_scales, E * I / 128 * kb4, sf_box));
        MOE_TRY(make_sf_map(&p.sfb_map[0], q.row_scales, Rp128 * kb4, sf_box));
        if (sh) {
          MOE_TRY(make_sf_map(&p.sfa0_map[1], w.ws1_scales, Is / 128 * kb4, sf_box));
          MOE_TRY(make_sf_map(&p.sfa1_map[1], w.ws3_scales, Is / 128 * kb4, sf_box));
          MOE_TRY(make_sf_map(&p.sfb_map[1], q.x_scales, Tp128 * kb4, sf_box));
        } else {
          p.sfa0_map[1] = p.sfa0_map[0];
          p.sfa1_map[1] = p.sfa1_map[0];
          p.sfb_map[1] = p.sfb_map[0];
        }
      }
    }
    if (mx) {
      p.q_out[0] = static_cast<uint8_t*>(h);
      p.q_sf[0] = wsb + L.h_sf;
      p.q_out[1] = static_cast<uint8_t*>(hs);
      p.q_sf[1] = wsb + L.h_shared_sf;
    }
    if (nv) {
      p.ga[0] = p.ga[1] = q.x_global;
      p.ga_stride[0] = p.ga_stride[1] = 0;
      p.gw[0] = w.w13_global;
      p.gw_stride[0] = 1;
      p.gw[1] = sh ? w.ws13_global : w.w13_global;
      p.gw_stride[1] = 0;
      p.amax_out[0] = g_h;
      p.amax_stride[0] = 1;
      p.amax_out[1] = g_h + c.E;
      p.amax_stride[1] = 0;
    }
    p.counts = counts;
    p.offsets = offsets;
    p.E = c.E;
    p.dense_rows = sh ? c.T : 0;
    p.status = status_ptr(ws);
    if (early) p.chunk_done = chunk_done;
    if (dyn) p.unit_counter = unit_counters;
    const int units = max_chunks * p.g[0].n_slabs + (sh ? dense_chunks * p.g[1].n_slabs : 0);
    fc1_slabs[0] = p.g[0].n_slabs;
    fc1_slabs[1] = p.g[1].n_slabs;
    MOE_TRY((launch_gemm<kFc1, TILE_N, DT, PAIR>(p, units, s)));
  }
  // NVFP4: h's per-expert global scales from the amax fc1 gathered, then h codes
  void* h_in = h;
  void* hs_in = hs;
  if (nv) {
    MOE_TRY(launch_pdl(amax_to_global_kernel, dim3((c.E + 1 + 255) / 256), dim3(256), 0, s, g_h, c.E + 1));
    MOE_TRY(launch_check());
    MOE_TRY(launch_pdl(quantize_h_nvfp4_kernel, dim3(sm_count() * 4), dim3(256), 0, s, 
        static_cast<const __nv_bfloat16*>(h), wsb + L.h_q, wsb + L.h_sf, c.I, offsets, counts,
        c.E, g_h, 0));
    MOE_TRY(launch_check());
    if (sh) {
      MOE_TRY(launch_pdl(quantize_h_nvfp4_kernel, dim3(sm_count() * 2), dim3(256), 0, s, 
          static_cast<const __nv_bfloat16*>(hs), wsb + L.h_shared_q, wsb + L.h_shared_sf,
          c.I_shared, offsets, counts, c.E, g_h + c.E, c.T));
      MOE_TRY(launch_check());
    }
    h_in = wsb + L.h_q;
    hs_in = wsb + L.h_shared_q;
  }
  // fc2: two adjacent 128-row slabs of W2 (256 output features) per tile
  {
    GemmParams p;
    memset(&p, 0, sizeof(p));
    MOE_TRY(make_tiled_map(&p.a0[0], w.w2, E * H, kbytes(I)));
    MOE_TRY(make_map(&p.b[0], h_in, tok_t, me, kbytes(I) / me, L.r_cap, kbytes(I), kBoxRows));
    if (sh) {
      MOE_TRY(make_tiled_map(&p.a0[1], w.ws2, H, kbytes(Is)));
      MOE_TRY(make_map(&p.b[1], hs_in, tok_t, me, kbytes(Is) / me, T, kbytes(Is), kBoxRows));
    } else {
      p.a0[1] = p.a0[0];
      p.b[1] = p.b[0];
    }
    p.a1[0] = p.a0[0];
    p.a1[1] = p.a0[1];
    const int slabs = (c.H + span2 - 1) / span2;
    p.g[0] = GemmGroup{c.H, c.H, slabs, c.I / kstep, 1, out_rows, c.H, 0};
    p.g[1] = GemmGroup{0, c.H, slabs, (sh ? c.I_shared : kstep) / kstep, 1, shared_out, c.H, 0};
    if (qz) {
      p.sfa0[0] = static_cast<const uint8_t*>(w.w2_scales);
      p.sfb[0] = wsb + L.h_sf;
      p.sfa0[1] = static_cast<const uint8_t*>(w.ws2_scales);
      p.sfb[1] = wsb + L.h_shared_sf;
      p.kb4[0] = c.I / kb4_div;
      p.kb4[1] = sh ? c.I_shared / kb4_div : 1;
      if (PAIR) {
        MOE_TRY(make_sf_map(&p.sfa0_map[0], w.w2_scales, E * H / 128 * (I / kb4_div), sf_box));
        MOE_TRY(make_sf_map(&p.sfb_map[0], wsb + L.h_sf, Rp128 * (I / kb4_div), sf_box));
        if (sh) {
          MOE_TRY(make_sf_map(&p.sfa0_map[1], w.ws2_scales, H / 128 * (Is / kb4_div), sf_box));
          MOE_TRY(make_sf_map(&p.sfb_map[1], wsb + L.h_shared_sf, Tp128 * (Is / kb4_div), sf_box));
        } else {
          p.sfa0_map[1] = p.sfa0_map[0];
          p.sfb_map[1] = p.sfb_map[0];
        }
        p.sfa1_map[0] = p.sfa0_map[0];
        p.sfa1_map[1] = p.sfa0_map[1];
      }
    }
    if (nv) {
      p.ga[0] = g_h;
      p.ga_stride[0] = 1;
      p.ga[1] = g_h + c.E;
      p.ga_stride[1] = 0;
      p.gw[0] = w.w2_global;
      p.gw_stride[0] = 1;
      p.gw[1] = sh ? w.ws2_global : w.w2_global;
      p.gw_stride[1] = 0;
    }
    p.counts = counts;
    p.offsets = offsets;
    p.E = c.E;
    p.dense_rows = sh ? c.T : 0;
    p.status = status_ptr(ws);
    if (early) {
      // every epilogue warp of every fc1 tile of the chunk counts once
      const int warps = kEpiWarps * (PAIR ? 2 : 1);
      p.chunk_done = chunk_done;
      const int never = test_fc2_never_ready() ? 1 : 0;
      p.chunk_target[0] = fc1_slabs[0] * warps + never;
      p.chunk_target[1] = fc1_slabs[1] * warps + never;
    }
    if (dyn) p.unit_counter = unit_counters + 1;
    const int units = max_chunks * slabs + (sh ? dense_chunks * slabs : 0);
    MOE_TRY((launch_gemm<kFc2, TILE_N, DT, PAIR>(p, units, s)));
  }
  return MOE_OK;
}

// CTA pairs for fc1 and fc2 (bf16, MXFP8) unless fc1 gathers its rows from x
// (rows == NULL) or MOE_GEMM_PAIRS=0 asks for one-CTA tiles.  NVFP4 keeps
// one-CTA tiles: its scale chunks leave a pair's ring at three stages, like a
// single CTA's, and the split tiles then measured slower (prefill grouped MLP
// 3964 -> 4247 us, decode 1510 -> 1594 us on one B200).
bool use_pairs(const moe_config& c, const void* rows) {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("MOE_GEMM_PAIRS");
    v = (e && atoi(e) == 0) ? 0 : 1;
  }
  return v == 1 && rows != nullptr && c.dtype != MOE_NVFP4;
}

moe_status do_grouped_mlp(const moe_config& c, const moe_weights& w, const void* rows,
                          const void* x, const MlpQuant& q, const int32_t* counts,
                          const int32_t* offsets, void* out_rows, void* shared_out, void* ws,
                          cudaStream_t s, bool scratch_zeroed = false) {
  // Decode-sized batches (at most 32 rows per expert on average) take 64-token
  // tiles: a stage holds far fewer token bytes (a fourth stage fits) and two
  // accumulators fit TMEM, so each tile's epilogue overlaps the next tile.
  const bool small = static_cast<int64_t>(c.T) * c.top_k <= 32LL * c.E;
  const bool pairs = !small && use_pairs(c, rows);
#define MOE_MLP(TN, DT, PR)                                                                      \
  return grouped_mlp_tiles<TN, DT, PR>(c, w, rows, x, q, counts, offsets, out_rows, shared_out, \
                                       ws, s, scratch_zeroed)
  if (is_mx(c)) {
    if (small) MOE_MLP(64, kMXF8, false);
    if (pairs) MOE_MLP(192, kMXF8, true);
    MOE_MLP(192, kMXF8, false);
  }
  if (is_nv(c)) {
    if (small) MOE_MLP(64, kNVF4, false);
    MOE_MLP(192, kNVF4, false);
  }
  if (small) MOE_MLP(64, kBF16, false);
  if (pairs) MOE_MLP(256, kBF16, true);
  MOE_MLP(256, kBF16, false);
#undef MOE_MLP
}

moe_status do_combine(const moe_config& c, const void* out_rows, const int32_t* token_row,
                      const float* topk_w, const void* shared_out, void* y, cudaStream_t s) {
  CombineArgs a;
  a.out_rows = static_cast<const __nv_bfloat16*>(out_rows);
  a.token_row = token_row;
  a.topk_w = topk_w;
  a.shared = static_cast<const __nv_bfloat16*>(shared_out);
  a.y = static_cast<__nv_bfloat16*>(y);
  a.T = c.T;
  a.H = c.H;
  a.k = c.top_k;
  const int threads = (c.H / 8) < 256 ? (c.H / 8) : 256;
  switch (c.top_k) {
    case 1: MOE_TRY(launch_pdl(combine_kernel<1>, dim3(c.T), dim3(threads), 0, s, a)); break;
    case 2: MOE_TRY(launch_pdl(combine_kernel<2>, dim3(c.T), dim3(threads), 0, s, a)); break;
    case 3: MOE_TRY(launch_pdl(combine_kernel<3>, dim3(c.T), dim3(threads), 0, s, a)); break;
    case 4: MOE_TRY(launch_pdl(combine_kernel<4>, dim3(c.T), dim3(threads), 0, s, a)); break;
    case 5: MOE_TRY(launch_pdl(combine_kernel<5>, dim3(c.T), dim3(threads), 0, s, a)); break;
    case 6: MOE_TRY(launch_pdl(combine_kernel<6>, dim3(c.T), dim3(threads), 0, s, a)); break;
    case 7: MOE_TRY(launch_pdl(combine_kernel<7>, dim3(c.T), dim3(threads), 0, s, a)); break;
    case 8: MOE_TRY(launch_pdl(combine_kernel<8>, dim3(c.T), dim3(threads), 0, s, a)); break;
    default: MOE_TRY(launch_pdl(combine_kernel<0>, dim3(c.T), dim3(threads), 0, s, a)); break;
  }
  return launch_check();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

moe_status check_ws(const moe_config& c, void* ws, size_t bytes) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % kAlign) return MOE_ERR_INVALID_ARG;
  if (bytes < step_layout(c).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

moe_status check_weights(const moe_config& c, const moe_weights* w) {
  if (!w || !w->w1 || !w->w3 || !w->w2) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->w1) || !aligned16(w->w3) || !aligned16(w->w2)) return MOE_ERR_INVALID_ARG;
  if (c.I_shared > 0) {
    if (!w->ws1 || !w->ws3 || !w->ws2) return MOE_ERR_INVALID_ARG;
    if (!aligned16(w->ws1) || !aligned16(w->ws3) || !aligned16(w->ws2)) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CAPACITY: return "expert index out of range (device)";
    case MOE_ERR_TIMEOUT: return "bounded wait timed out (device)";
    case MOE_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

moe_status moe_workspace_size(const moe_config* cfg, size_t* bytes, int32_t* r_cap) {
  MOE_TRY(check_config(cfg));
  const StepLayout L = step_layout(*cfg);
  if (bytes) *bytes = L.total;
  if (r_cap) *r_cap = L.r_cap;
  return MOE_OK;
}

moe_status moe_route(const moe_config* cfg, const void* x, const void* w_router,
                     const float* bias, const float* logits_in, float* logits_out,
                     int32_t* topk_idx, float* topk_w, void* workspace, size_t workspace_bytes,
                     void* stream) {
  MOE_TRY(check_config(cfg));
  MOE_TRY(check_ws(*cfg, workspace, workspace_bytes));
  if (!bias || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!logits_in) {
    if (!x || !w_router || !logits_out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
  }
  return do_route(*cfg, x, w_router, bias, logits_in, logits_out, topk_idx, topk_w, workspace,
                  static_cast<cudaStream_t>(stream));
}

moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx, const void* src_rows,
                       const void* src_scales, int32_t* counts, int32_t* offsets,
                       int32_t* row_token, int32_t* token_row, void* dst_rows, void* dst_scales,
                       void* workspace, size_t workspace_bytes, void* stream) {
  MOE_TRY(check_config(cfg));
  MOE_TRY(check_dtype(cfg));
  MOE_TRY(check_ws(*cfg, workspace, workspace_bytes));
  if (!topk_idx || !counts || !offsets || !row_token || !token_row) return MOE_ERR_INVALID_ARG;
  if (dst_rows && (!src_rows || !aligned16(src_rows) || !aligned16(dst_rows)))
    return MOE_ERR_INVALID_ARG;
  if (!is_bf16(*cfg) && (!src_scales || !dst_scales || !aligned16(src_scales) ||
                         !aligned16(dst_scales)))
    return MOE_ERR_INVALID_ARG;
  return do_permute(*cfg, topk_idx, src_rows, src_scales, counts, offsets, row_token, token_row,
                    dst_rows, dst_scales, workspace, static_cast<cudaStream_t>(stream));
}

moe_status moe_grouped_mlp(const moe_config* cfg, const moe_weights* w, const void* rows,
                           const void* row_scales, const void* x, const void* x_scales,
                           const float* x_global, const int32_t* counts, const int32_t* offsets,
                           const int32_t* row_token, void* out_rows, void* shared_out,
                           void* workspace, size_t workspace_bytes, void* stream) {
  MOE_TRY(check_config(cfg));
  MOE_TRY(check_dtype(cfg));
  MOE_TRY(check_ws(*cfg, workspace, workspace_bytes));
  MOE_TRY(check_weights(*cfg, w));
  if (!counts || !offsets || !out_rows || !aligned16(out_rows)) return MOE_ERR_INVALID_ARG;
  if (rows ? !aligned16(rows) : (!row_token || !x || !aligned16(x))) return MOE_ERR_INVALID_ARG;
  if (cfg->I_shared > 0 && (!x || !shared_out || !aligned16(x) || !aligned16(shared_out)))
    return MOE_ERR_INVALID_ARG;
  if (!is_bf16(*cfg)) {
    if (!row_scales || !aligned16(row_scales)) return MOE_ERR_INVALID_ARG;
    if (cfg->I_shared > 0 && (!x_scales || !aligned16(x_scales))) return MOE_ERR_INVALID_ARG;
    if (!w->w1_scales || !w->w3_scales || !w->w2_scales) return MOE_ERR_INVALID_ARG;
    if (cfg->I_shared > 0 && (!w->ws1_scales || !w->ws3_scales || !w->ws2_scales))
      return MOE_ERR_INVALID_ARG;
  }
  if (is_nv(*cfg)) {
    if (!x_global || !w->w13_global || !w->w2_global) return MOE_ERR_INVALID_ARG;
    if (cfg->I_shared > 0 && (!w->ws13_global || !w->ws2_global)) return MOE_ERR_INVALID_ARG;
  }
  MlpQuant q{row_scales, x_scales, x_global, rows ? nullptr : row_token};
  return do_grouped_mlp(*cfg, *w, rows, x, q, counts, offsets, out_rows, shared_out, workspace,
                        static_cast<cudaStream_t>(stream));
}

moe_status moe_combine(const moe_config* cfg, const void* out_rows, const int32_t* token_row,
                       const float* topk_w, const void* shared_out, void* y, void* stream) {
  MOE_TRY(check_config(cfg));
  if (!out_rows || !token_row || !topk_w || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned16(out_rows) || !aligned16(y) || (shared_out && !aligned16(shared_out)))
    return MOE_ERR_INVALID_ARG;
  return do_combine(*cfg, out_rows, token_row, topk_w, shared_out, y,
                    static_cast<cudaStream_t>(stream));
}

moe_status moe_prepared_weights_size(const moe_config* cfg, moe_weight_sizes* sizes) {
  MOE_TRY(check_config(cfg));
  MOE_TRY(check_dtype(cfg));
  if (!sizes) return MOE_ERR_INVALID_ARG;
  const size_t H = cfg->H, I = cfg->I, E = cfg->E, Is = cfg->I_shared;
  // bytes per weight element x2 (NVFP4 packs two per byte), elements per scale
  const size_t e2 = is_mx(*cfg) ? 2 : (is_nv(*cfg) ? 1 : 4);
  const size_t blk = is_mx(*cfg) ? 32 : (is_nv(*cfg) ? 16 : 0);
  sizes->w13 = E * I * H * e2 / 2;
  sizes->w2 = E * H * I * e2 / 2;
  sizes->ws13 = Is * H * e2 / 2;
  sizes->ws2 = H * Is * e2 / 2;
  sizes->w13_scales = blk ? E * I * H / blk : 0;
  sizes->w2_scales = blk ? E * H * I / blk : 0;
  sizes->ws13_scales = blk ? Is * H / blk : 0;
  sizes->ws2_scales = blk ? H * Is / blk : 0;
  sizes->w_globals = is_nv(*cfg) ? E * 4 : 0;
  sizes->ws_globals = is_nv(*cfg) && Is ? 4 : 0;
  return MOE_OK;
}

moe_status moe_prepare_weights(const moe_config* cfg, int32_t which, int32_t e_begin,
                               int32_t e_count, const void* w1, const void* w3, const void* w2,
                               const moe_weights* dst, void* stream) {
  MOE_TRY(check_config(cfg));
  MOE_TRY(check_dtype(cfg));
  if (!dst || !w1 || !w3 || !w2) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w1) || !aligned16(w3) || !aligned16(w2)) return MOE_ERR_INVALID_ARG;
  const moe_config& c = *cfg;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int64_t rows13, rows2, k13, k2;
  void *d1, *d3, *d2;
  if (which == 0) {
    if (e_begin < 0 || e_count < 1 || e_begin + e_count > c.E) return MOE_ERR_INVALID_ARG;
    if (!dst->w1 || !dst->w3 || !dst->w2) return MOE_ERR_INVALID_ARG;
    rows13 = static_cast<int64_t>(e_count) * c.I;
    rows2 = static_cast<int64_t>(e_count) * c.H;
    k13 = c.H;
    k2 = c.I;
    // experts are contiguous in the tile-major layout: expert e starts at tile e*(I/128)*(H/64)
    d1 = static_cast<uint8_t*>(dst->w1) + static_cast<size_t>(e_begin) * c.I * c.H * 2;
    d3 = static_cast<uint8_t*>(dst->w3) + static_cast<size_t>(e_begin) * c.I * c.H * 2;
    d2 = static_cast<uint8_t*>(dst->w2) + static_cast<size_t>(e_begin) * c.H * c.I * 2;
  } else if (which == 1) {
    if (c.I_shared <= 0 || e_begin != 0 || e_count != 1) return MOE_ERR_INVALID_ARG;
    if (!dst->ws1 || !dst->ws3 || !dst->ws2) return MOE_ERR_INVALID_ARG;
    rows13 = c.I_shared;
    rows2 = c.H;
    k13 = c.H;
    k2 = c.I_shared;
    d1 = dst->ws1;
    d3 = dst->ws3;
    d2 = dst->ws2;
  } else {
    return MOE_ERR_INVALID_ARG;
  }
  if (!aligned16(d1) || !aligned16(d3) || !aligned16(d2)) return MOE_ERR_INVALID_ARG;
  if (is_nv(c)) {
    // per-expert global scales from the amax of W1 and W3 together, and of W2;
    // codes tile-major (128 rows x 256 elements), scales in the MMA layout
    const size_t off13 = which == 0 ? static_cast<size_t>(e_begin) * c.I * c.H : 0;
    const size_t off2 = which == 0 ? static_cast<size_t>(e_begin) * c.H * c.I : 0;
    float* g13 = which == 0 ? dst->w13_global + e_begin : dst->ws13_global;
    float* g2 = which == 0 ? dst->w2_global + e_begin : dst->ws2_global;
    uint8_t* s1 = static_cast<uint8_t*>(which == 0 ? dst->w1_scales : dst->ws1_scales);
    uint8_t* s3 = static_cast<uint8_t*>(which == 0 ? dst->w3_scales : dst->ws3_scales);
    uint8_t* s2 = static_cast<uint8_t*>(which == 0 ? dst->w2_scales : dst->ws2_scales);
    if (!s1 || !s3 || !s2 || !g13 || !g2) return MOE_ERR_INVALID_ARG;
    uint8_t* c1 = static_cast<uint8_t*>(which == 0 ? dst->w1 : dst->ws1) + off13 / 2;
    uint8_t* c3 = static_cast<uint8_t*>(which == 0 ? dst->w3 : dst->ws3) + off13 / 2;
    uint8_t* c2 = static_cast<uint8_t*>(which == 0 ? dst->w2 : dst->ws2) + off2 / 2;
    const int ng = which == 0 ? e_count : 1;
    MOE_CUDA(cudaMemsetAsync(g13, 0, ng * 4, s));
    MOE_CUDA(cudaMemsetAsync(g2, 0, ng * 4, s));
    const int64_t per13 = rows13 / ng * k13, per2 = rows2 / ng * k2;  // elements per expert
    const dim3 ga(static_cast<unsigned>((per13 / 8 + 255) / 256 < 64 ? (per13 / 8 + 255) / 256 : 64),
                  ng);
    const dim3 gb(static_cast<unsigned>((per2 / 8 + 255) / 256 < 64 ? (per2 / 8 + 255) / 256 : 64),
                  ng);
    amax_groups_kernel<<<ga, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w1), per13, g13);
    MOE_TRY(launch_check());
    amax_groups_kernel<<<ga, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w3), per13, g13);
    MOE_TRY(launch_check());
    amax_groups_kernel<<<gb, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w2), per2, g2);
    MOE_TRY(launch_check());
    amax_to_global_kernel<<<(ng + 255) / 256, 256, 0, s>>>(g13, ng);
    MOE_TRY(launch_check());
    amax_to_global_kernel<<<(ng + 255) / 256, 256, 0, s>>>(g2, ng);
    MOE_TRY(launch_check());
    const int64_t b13 = rows13 * (k13 / 16), b2 = rows2 * (k2 / 16);
    const int64_t rpg13 = rows13 / ng, rpg2 = rows2 / ng;
    quantize_nvfp4_kernel<<<static_cast<unsigned>((b13 + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(w1), c1, s1 + off13 / 16, rows13,
        static_cast<int>(k13), g13, rpg13, 1);
    MOE_TRY(launch_check());
    quantize_nvfp4_kernel<<<static_cast<unsigned>((b13 + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(w3), c3, s3 + off13 / 16, rows13,
        static_cast<int>(k13), g13, rpg13, 1);
    MOE_TRY(launch_check());
    quantize_nvfp4_kernel<<<static_cast<unsigned>((b2 + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(w2), c2, s2 + off2 / 16, rows2, static_cast<int>(k2),
        g2, rpg2, 1);
    return launch_check();
  }
  if (is_mx(c)) {
    // codes tile-major, scales in the MMA layout; byte offsets of the expert range
    const size_t off13 = which == 0 ? static_cast<size_t>(e_begin) * c.I * c.H : 0;
    const size_t off2 = which == 0 ? static_cast<size_t>(e_begin) * c.H * c.I : 0;
    uint8_t* s1 = static_cast<uint8_t*>(which == 0 ? dst->w1_scales : dst->ws1_scales);
    uint8_t* s3 = static_cast<uint8_t*>(which == 0 ? dst->w3_scales : dst->ws3_scales);
    uint8_t* s2 = static_cast<uint8_t*>(which == 0 ? dst->w2_scales : dst->ws2_scales);
    if (!s1 || !s3 || !s2) return MOE_ERR_INVALID_ARG;
    uint8_t* c1 = static_cast<uint8_t*>(which == 0 ? dst->w1 : dst->ws1) + off13;
    uint8_t* c3 = static_cast<uint8_t*>(which == 0 ? dst->w3 : dst->ws3) + off13;
    uint8_t* c2 = static_cast<uint8_t*>(which == 0 ? dst->w2 : dst->ws2) + off2;
    const int64_t b13 = rows13 * (k13 / 32), b2 = rows2 * (k2 / 32);
    quantize_mxfp8_tiles_kernel<<<static_cast<unsigned>((b13 + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(w1), c1, s1 + off13 / 32, rows13, static_cast<int>(k13));
    MOE_TRY(launch_check());
    quantize_mxfp8_tiles_kernel<<<static_cast<unsigned>((b13 + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(w3), c3, s3 + off13 / 32, rows13, static_cast<int>(k13));
    MOE_TRY(launch_check());
    quantize_mxfp8_tiles_kernel<<<static_cast<unsigned>((b2 + 255) / 256), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(w2), c2, s2 + off2 / 32, rows2, static_cast<int>(k2));
    return launch_check();
  }
  const int64_t t13 = (rows13 / 128) * (k13 / 64), t2 = (rows2 / 128) * (k2 / 64);
  tile_rows_kernel<<<static_cast<unsigned>(t13), 256, 0, s>>>(
      static_cast<const uint4*>(w1), static_cast<uint4*>(d1), rows13, static_cast<int>(k13));
  MOE_TRY(launch_check());
  tile_rows_kernel<<<static_cast<unsigned>(t13), 256, 0, s>>>(
      static_cast<const uint4*>(w3), static_cast<uint4*>(d3), rows13, static_cast<int>(k13));
  MOE_TRY(launch_check());
  tile_rows_kernel<<<static_cast<unsigned>(t2), 256, 0, s>>>(
      static_cast<const uint4*>(w2), static_cast<uint4*>(d2), rows2, static_cast<int>(k2));
  return launch_check();
}

moe_status moe_quantize(int32_t dtype, const void* in, int32_t rows, int32_t cols, void* codes,
                        void* scales, float* global_scale, void* stream) {
  if (dtype != MOE_MXFP8 && dtype != MOE_NVFP4) return MOE_ERR_INVALID_ARG;
  if (!in || !codes || !scales || rows < 1 || cols < 1) return MOE_ERR_INVALID_ARG;
  if (cols % (dtype == MOE_NVFP4 ? 256 : 128)) return MOE_ERR_UNSUPPORTED;
  if (!aligned16(in) || !aligned16(codes)) return MOE_ERR_INVALID_ARG;
  if (dtype == MOE_NVFP4) {
    if (!global_scale) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t n = static_cast<int64_t>(rows) * cols;
    MOE_CUDA(cudaMemsetAsync(global_scale, 0, 4, st));
    const unsigned nb = static_cast<unsigned>((n / 8 + 255) / 256 < 2048 ? (n / 8 + 255) / 256 : 2048);
    MOE_TRY(launch_pdl(amax_groups_kernel, dim3(dim3(nb, 1)), dim3(256), 0, st, static_cast<const __nv_bfloat16*>(in), n,
                                                    global_scale));
    MOE_TRY(launch_check());
    MOE_TRY(launch_pdl(amax_to_global_kernel, dim3(1), dim3(32), 0, st, global_scale, 1));
    MOE_TRY(launch_check());
    const int64_t blocks = static_cast<int64_t>(rows) * (cols / 16);
    MOE_TRY(launch_pdl(quantize_nvfp4_kernel, dim3(static_cast<unsigned>((blocks + 255) / 256)), dim3(256), 0, st, 
        static_cast<const __nv_bfloat16*>(in), static_cast<uint8_t*>(codes),
        static_cast<uint8_t*>(scales), rows, cols, global_scale, 0, 0));
    return launch_check();
  }
  const int64_t blocks = static_cast<int64_t>(rows) * (cols / 32);
  MOE_TRY(launch_pdl(quantize_mxfp8_rows_kernel, dim3(static_cast<unsigned>((blocks + 255) / 256)), dim3(256), 0, static_cast<cudaStream_t>(stream), 
      static_cast<const __nv_bfloat16*>(in), static_cast<uint8_t*>(codes),
      static_cast<uint8_t*>(scales), rows, cols));
  return launch_check();
}

moe_status moe_forward_workspace_size(const moe_config* cfg, size_t* bytes) {
  MOE_TRY(check_config(cfg));
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = fwd_layout(*cfg).total;
  return MOE_OK;
}

moe_status moe_forward(const moe_config* cfg, const moe_weights* w, const void* w_router,
                       const float* bias, const void* x, void* y, int32_t xy_on_host,
                       void* workspace, size_t workspace_bytes, void* stream) {
  MOE_TRY(check_config(cfg));
  MOE_TRY(check_dtype(cfg));
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % kAlign) return MOE_ERR_INVALID_ARG;
  const FwdLayout F = fwd_layout(*cfg);
  if (workspace_bytes < F.total) return MOE_ERR_WORKSPACE;
  MOE_TRY(check_weights(*cfg, w));
  if (!w_router || !bias || !x || !y || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
  const moe_config& c = *cfg;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* b = static_cast<uint8_t*>(workspace);
  const size_t xbytes = static_cast<size_t>(c.T) * c.H * 2;
  const void* xd = x;
  void* yd = y;
  if (xy_on_host) {
    MOE_CUDA(cudaMemcpyAsync(b + F.x, x, xbytes, cudaMemcpyHostToDevice, s));
    xd = b + F.x;
    yd = b + F.y;
  } else if (!aligned16(x) || !aligned16(y)) {
    return MOE_ERR_INVALID_ARG;
  }
  float* logits = reinterpret_cast<float*>(b + F.logits);
  int32_t* topk_idx = reinterpret_cast<int32_t*>(b + F.topk_idx);
  float* topk_w = reinterpret_cast<float*>(b + F.topk_w);
  int32_t* counts = reinterpret_cast<int32_t*>(b + F.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(b + F.offsets);
  int32_t* row_token = reinterpret_cast<int32_t*>(b + F.row_token);
  int32_t* token_row = reinterpret_cast<int32_t*>(b + F.token_row);
  void* out_rows = b + F.out_rows;
  void* shared_out = c.I_shared > 0 ? b + F.shared_out : nullptr;
  MOE_TRY(zero_mlp_scratch(c, workspace, s));
  MOE_TRY(do_route(c, xd, w_router, bias, nullptr, logits, topk_idx, topk_w, workspace, s));
  // an expert-major copy of the rows: fc1 reads it with 32-row TMA boxes, which
  // streams faster than per-row gathers from x (moe_grouped_mlp with rows == NULL)
  void* rows = b + F.rows;
  const void* xq = xd;
  MlpQuant q{nullptr, nullptr, nullptr, nullptr};
  if (is_bf16(c)) {
    MOE_TRY(do_permute(c, topk_idx, xd, nullptr, counts, offsets, row_token, token_row, rows,
                       nullptr, workspace, s));
  } else if (is_mx(c)) {
    // MXFP8: quantize in token order, then gather codes and scales (its top_k
    // row copies make the one-pass form below write-bound and slower on B200:
    // DeepSeek-V3 dims 103 us against 15 + 73 us)
    float* xg = reinterpret_cast<float*>(b + F.x_g);
    MOE_TRY(moe_quantize(c.dtype, xd, c.T, c.H, b + F.x_q, b + F.x_sf, xg, s));
    xq = b + F.x_q;
    q = MlpQuant{b + F.rows_sf, b + F.x_sf, xg, nullptr};
    MOE_TRY(do_permute(c, topk_idx, xq, q.x_scales, counts, offsets, row_token, token_row, rows,
                       b + F.rows_sf, workspace, s));
  } else {
    // NVFP4: each token is quantized once and its codes and scales go straight
    // to its expert-major rows (and to token order for the shared expert),
    // after x's global scale is taken from its amax
    float* xg = reinterpret_cast<float*>(b + F.x_g);
    {
      const int64_t n = static_cast<int64_t>(c.T) * c.H;
      MOE_CUDA(cudaMemsetAsync(xg, 0, 4, s));
      const unsigned nb = static_cast<unsigned>((n / 8 + 255) / 256 < 2048 ? (n / 8 + 255) / 256 : 2048);
      MOE_TRY(launch_pdl(amax_groups_kernel, dim3(nb, 1), dim3(256), 0, s,
                         static_cast<const __nv_bfloat16*>(xd), n, xg));
      MOE_TRY(launch_check());
      MOE_TRY(launch_pdl(amax_to_global_kernel, dim3(1), dim3(32), 0, s, xg, 1));
      MOE_TRY(launch_check());
    }
    MOE_TRY(do_permute_maps(c, topk_idx, counts, offsets, row_token, token_row, workspace, s));
    const bool sh = c.I_shared > 0;
    QScatterArgs qa;
    qa.x = static_cast<const __nv_bfloat16*>(xd);
    qa.token_row = token_row;
    qa.row_token = row_token;
    qa.offsets = offsets;
    qa.rows = static_cast<uint8_t*>(rows);
    qa.rows_sf = b + F.rows_sf;
    qa.xq = sh ? b + F.x_q : nullptr;
    qa.xq_sf = sh ? b + F.x_sf : nullptr;
    qa.g = xg;
    qa.T = c.T;
    qa.H = c.H;
    qa.k = c.top_k;
    qa.E = c.E;
    const dim3 grid(sm_count() * 8), block(256);
    MOE_TRY(launch_pdl(quantize_scatter_nvfp4_kernel, grid, block, 0, s, qa));
    MOE_TRY(launch_check());
    xq = b + F.x_q;
    q = MlpQuant{b + F.rows_sf, b + F.x_sf, xg, nullptr};
  }
  MOE_TRY(do_grouped_mlp(c, *w, rows, xq, q, counts, offsets, out_rows, shared_out, workspace,
                         s, /*scratch_zeroed=*/true));
  MOE_TRY(do_combine(c, out_rows, token_row, topk_w, shared_out, yd, s));
  if (xy_on_host) MOE_CUDA(cudaMemcpyAsync(y, yd, xbytes, cudaMemcpyDeviceToHost, s));
  return MOE_OK;
}

moe_status moe_get_device_status(void* workspace, int32_t* device_status, void* stream) {
  if (!workspace || !device_status) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  MOE_CUDA(cudaMemcpyAsync(&v, workspace, 4, cudaMemcpyDeviceToHost, s));
  MOE_CUDA(cudaStreamSynchronize(s));
  MOE_CUDA(cudaMemsetAsync(workspace, 0, 4, s));
  MOE_CUDA(cudaStreamSynchronize(s));
  *device_status = v;
  return MOE_OK;
}

}  // extern "C"

// ===========================================================================
// moe_permute_noalloc: the permute with its histogram scratch in a fixed
// device array compiled into the library, for callers that cannot hand the
// library a workspace.
// ===========================================================================
namespace {

// Histogram scratch: one int32 per (tile of 256 (t, j) entries, expert).
constexpr int kNoAllocScratchInts = 1 << 18;  // 1 MiB per device

}  // namespace

static __device__ __align__(256) int32_t moe_noalloc_permute_scratch[kNoAllocScratchInts];

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
int32_t* g_noalloc_ptr[kNoAllocMaxDevices] = {};
unsigned long long g_noalloc_ctx[kNoAllocMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the current CUDA context (ids are never reused, so a context
// re-created after a device reset gets a new one); 0 if it cannot be read.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (!get_current || !get_id) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &a, 12000, cudaEnableDefault, &qa) !=
            cudaSuccess || qa != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPointByVersion("cuCtxGetId", &b, 12000, cudaEnableDefault, &qb) !=
            cudaSuccess || qb != cudaDriverEntryPointSuccess)
      return 0;
    get_current = reinterpret_cast<CtxGetCurrentFn>(a);
    get_id = reinterpret_cast<CtxGetIdFn>(b);
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device.  Host code must
// not use the array's name as a pointer: on the host it is only a stand-in
// for the symbol.  The address is looked up with the device current, once
// per device and CUDA context (again after a device reset re-creates the
// context), and cached.
moe_status noalloc_scratch(int32_t** out) {
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_UNSUPPORTED;
  // 0 before the device's context exists; the symbol lookup then creates it
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    MOE_CUDA(cudaGetSymbolAddress(&p, moe_noalloc_permute_scratch));
    g_noalloc_ptr[dev] = static_cast<int32_t*>(p);
    g_noalloc_ctx[dev] = current_context_id();
  }
  *out = g_noalloc_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx,
                                          const void* src_rows, const void* src_scales,
                                          int32_t* counts, int32_t* offsets, int32_t* row_token,
                                          int32_t* token_row, void* dst_rows, void* dst_scales,
                                          void* stream) {
  MOE_TRY(check_config(cfg));
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;  // gathers bf16 rows only
  if (src_scales || dst_scales) return MOE_ERR_INVALID_ARG;  // bf16 rows carry no scales
  if (!topk_idx || !src_rows || !counts || !offsets || !row_token || !token_row || !dst_rows)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(src_rows) || !aligned16(dst_rows)) return MOE_ERR_INVALID_ARG;
  const moe_config& c = *cfg;
  const StepLayout L = step_layout(c);
  const int64_t need = static_cast<int64_t>(L.ntiles) * c.E;
  if (need > kNoAllocScratchInts) {
    fprintf(stderr,
            "moe_permute_noalloc: ceil(T*top_k/256)*E = %lld exceeds the built-in scratch of "
            "%d entries; use moe_permute with a workspace\n",
            static_cast<long long>(need), kNoAllocScratchInts);
    return MOE_ERR_WORKSPACE;
  }
  int32_t* scratch = nullptr;
  MOE_TRY(noalloc_scratch(&scratch));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PermArgs a;
  a.topk_idx = topk_idx;
  a.hist = scratch;  // every entry read is first written by this call's histogram kernel
  a.counts = counts;
  a.offsets = offsets;
  a.row_token = row_token;
  a.token_row = token_row;
  a.status = nullptr;  // bad indices are dropped (token_row = -1) without a status word
  a.n = c.T * c.top_k;
  a.k = c.top_k;
  a.E = c.E;
  a.P = c.pad_multiple;
  a.r_cap = L.r_cap;
  a.ntiles = L.ntiles;
  const size_t hsm = static_cast<size_t>(c.E) * 4;
  permute_hist_kernel<<<L.ntiles, 256, hsm, s>>>(a);
  MOE_TRY(launch_check());
  permute_scan_kernel<<<(c.E + 7) / 8, 256, 0, s>>>(a);
  MOE_TRY(launch_check());
  permute_rank_kernel<<<L.ntiles, 256, 0, s>>>(a);
  MOE_TRY(launch_check());
  GatherArgs g;
  g.src = static_cast<const uint8_t*>(src_rows);
  g.dst = static_cast<uint8_t*>(dst_rows);
  g.row_token = row_token;
  g.offsets = offsets;
  g.E = c.E;
  g.row_bytes = c.H * 2;
  permute_gather_kernel<<<sm_count() * 4, 256, 0, s>>>(g);
  return launch_check();
}

// The backward of the bf16 layer: its host steps and its C ABI.
#include "backward_api.cuh"
