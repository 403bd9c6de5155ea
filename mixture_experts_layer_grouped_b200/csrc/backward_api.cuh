// Host side of the backward of the bf16 layer (part of moe_api.cu's translation
// unit, included at its end): the workspace layout, the dgrad and wgrad
// launches, argument checks, and the four C ABI calls of include/moe_b200.h's
// backward section.  The kernels are in backward.cuh, wgrad.cuh and
// grouped_gemm.cuh (the fc1 kernel's backward form).
#pragma once

namespace {

// ---------------------------------------------------------------------------
// Backward of the bf16 layer.
// ---------------------------------------------------------------------------
inline int64_t ceil64(int64_t v) { return (v + 63) / 64 * 64; }

// Columns of the dense operand of the last dgrad contraction, [da_s | du_s |
// bf16(dlogits) | 0]: the shared expert's dx and the router's dx come out of
// one contraction with [Ws1^T | Ws3^T | W_r^T | 0].
int64_t dense_bwd_cols(const moe_config& c) {
  return 2 * static_cast<int64_t>(c.I_shared > 0 ? c.I_shared : 0) + ceil64(c.E);
}

struct BwdLayout {
  size_t status, dO, dh, dz, h, dX, dh_s, h_s, dense_b, dx_dense, dgate, total;
  int32_t r_cap;
};

BwdLayout bwd_layout(const moe_config& c) {
  BwdLayout L;
  L.r_cap = r_cap_of(c);
  const size_t R = L.r_cap, T = c.T, H = c.H, I = c.I, Is = c.I_shared > 0 ? c.I_shared : 0;
  size_t o = 0;
  L.status = o; o = align_up(o + 4);
  L.dO = o; o = align_up(o + R * H * 2);
  L.dh = o; o = align_up(o + R * I * 2);
  L.dz = o; o = align_up(o + R * 2 * I * 2);
  L.h = o; o = align_up(o + R * I * 2);
  L.dX = o; o = align_up(o + R * H * 2);
  L.dh_s = o; o = align_up(o + T * Is * 2);
  L.h_s = o; o = align_up(o + T * Is * 2);
  L.dense_b = o; o = align_up(o + T * static_cast<size_t>(dense_bwd_cols(c)) * 2);
  L.dx_dense = o; o = align_up(o + T * H * 2);
  L.dgate = o; o = align_up(o + T * c.top_k * 4);
  L.total = o;
  return L;
}

// out_g = A_g . B_g^T per group on the grouped GEMM's fc2 mode (every tile over
// the full K): the routed group has E experts of M_r rows each (A tile-major
// [E * M_r, K_r], B the expert-major rows [r_cap, K_r], out [r_cap, M_r]); the
// dense group (a_d non-null) one tile-major [M_d, K_d] matrix against the T
// token-order rows of b_d, out [T, M_d].
template <int TILE_N, bool PAIR>
moe_status rows_gemm(const moe_config& c, const void* a_r, int M_r, int K_r, const void* b_r,
                     void* out_r, const void* a_d, int M_d, int K_d, const void* b_d, void* out_d,
                     const int32_t* counts, const int32_t* offsets, int32_t* status,
                     cudaStream_t s) {
  constexpr int span = GemmCfg<kFc2, TILE_N, kBF16, PAIR>::SLAB_SPAN;
  const int32_t r_cap = r_cap_of(c);
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  MOE_TRY(make_tiled_map(&p.a0[0], a_r, static_cast<uint64_t>(c.E) * M_r,
                         static_cast<uint64_t>(K_r) * 2));
  MOE_TRY(make_map(&p.b[0], b_r, bf, 2, K_r, r_cap, static_cast<uint64_t>(K_r) * 2, kBoxRows));
  const bool dense = a_d != nullptr;
  if (dense) {
    MOE_TRY(make_tiled_map(&p.a0[1], a_d, M_d, static_cast<uint64_t>(K_d) * 2));
    MOE_TRY(make_map(&p.b[1], b_d, bf, 2, K_d, c.T, static_cast<uint64_t>(K_d) * 2, kBoxRows));
  } else {
    p.a0[1] = p.a0[0];
    p.b[1] = p.b[0];
  }
  p.a1[0] = p.a0[0];
  p.a1[1] = p.a0[1];
  p.g[0] = GemmGroup{M_r, M_r, (M_r + span - 1) / span, K_r / kBK, 1, out_r, M_r, 0};
  if (dense)
    p.g[1] = GemmGroup{0, M_d, (M_d + span - 1) / span, K_d / kBK, 1, out_d, M_d, 0};
  else
    p.g[1] = GemmGroup{0, M_r, p.g[0].n_slabs, 1, 1, nullptr, M_r, 0};  // no rows: never run
  p.counts = counts;
  p.offsets = offsets;
  p.E = c.E;
  p.dense_rows = dense ? c.T : 0;
  p.status = status;
  const int max_chunks = c.E + (c.T * c.top_k) / TILE_N + 1;
  const int dense_chunks = (c.T + TILE_N - 1) / TILE_N;
  const int units = max_chunks * p.g[0].n_slabs + (dense ? dense_chunks * p.g[1].n_slabs : 0);
  return launch_gemm<kFc2, TILE_N, kBF16, PAIR>(p, units, s);
}

// a = X W1^T and u = X W3^T recomputed in one pass of the fc1 kernel's
// backward form (W1 and W3 slabs per stage, as in the forward), stored as
// [a | u] rows of dz (row length 2I); the shared expert's on x into the first
// 2 I_shared columns of the dense operand (row length Kd).
template <int TILE_N, bool PAIR>
moe_status fc1_recompute(const moe_config& c, const moe_weights& w, const void* rows,
                         const void* x, void* dz, void* dense_b, int Kd, const int32_t* counts,
                         const int32_t* offsets, int32_t* status, cudaStream_t s) {
  constexpr int span = GemmCfg<kFc1, TILE_N, kBF16, PAIR>::SLAB_SPAN;
  const int32_t r_cap = r_cap_of(c);
  const bool sh = c.I_shared > 0;
  const uint64_t H = c.H, I = c.I, Is = sh ? c.I_shared : 0, E = c.E;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  MOE_TRY(make_tiled_map(&p.a0[0], w.w1, E * I, H * 2));
  MOE_TRY(make_tiled_map(&p.a1[0], w.w3, E * I, H * 2));
  MOE_TRY(make_map(&p.b[0], rows, bf, 2, H, r_cap, H * 2, kBoxRows));
  if (sh) {
    MOE_TRY(make_tiled_map(&p.a0[1], w.ws1, Is, H * 2));
    MOE_TRY(make_tiled_map(&p.a1[1], w.ws3, Is, H * 2));
    MOE_TRY(make_map(&p.b[1], x, bf, 2, H, c.T, H * 2, kBoxRows));
  } else {
    p.a0[1] = p.a0[0];
    p.a1[1] = p.a1[0];
    p.b[1] = p.b[0];
  }
  p.g[0] = GemmGroup{c.I, c.I, (c.I + span - 1) / span, c.H / kBK, 1, dz, 2 * c.I, 0};
  p.g[1] = GemmGroup{0, static_cast<int32_t>(Is), static_cast<int32_t>((Is + span - 1) / span),
                     c.H / kBK, 1, dense_b, Kd, 0};
  p.bwd_u_col[0] = c.I;
  p.bwd_u_col[1] = static_cast<int32_t>(Is);
  p.counts = counts;
  p.offsets = offsets;
  p.E = c.E;
  p.dense_rows = sh ? c.T : 0;
  p.status = status;
  const int max_chunks = c.E + (c.T * c.top_k) / TILE_N + 1;
  const int dense_chunks = (c.T + TILE_N - 1) / TILE_N;
  const int units = max_chunks * p.g[0].n_slabs + (sh ? dense_chunks * p.g[1].n_slabs : 0);
  return launch_gemm<kFc1, TILE_N, kBF16, PAIR, true>(p, units, s);
}

// One wgrad contraction as the host describes it.
struct WgDesc {
  const void* a;  // [rows, lda] bf16, the operand's columns start here
  int64_t lda;
  int a_cols;     // columns the A map covers (>= M; the extra ones hold zeros)
  const void* b;
  int64_t ldb;
  int M, N;
  float* out;
  bool routed;
};

moe_status launch_wgrad(const moe_config& c, const WgDesc* d, int n, bool accumulate,
                        const int32_t* counts, const int32_t* offsets, int32_t* status,
                        cudaStream_t s) {
  if (n < 1) return MOE_OK;
  if (n > kWgMaxProblems) return MOE_ERR_INVALID_ARG;
  WgradParams P;
  memset(&P, 0, sizeof(P));
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int32_t r_cap = r_cap_of(c);
  int tiles = 0;
  for (int i = 0; i < n; ++i) {
    WgradProblem& q = P.pr[i];
    const uint64_t rows = d[i].routed ? static_cast<uint64_t>(r_cap) : static_cast<uint64_t>(c.T);
    MOE_TRY(make_map(&q.a, d[i].a, bf, 2, d[i].a_cols, rows, d[i].lda * 2, kWgBK));
    MOE_TRY(make_map(&q.b, d[i].b, bf, 2, d[i].N, rows, d[i].ldb * 2, kWgBK));
    q.out = d[i].out;
    q.M = d[i].M;
    q.N = d[i].N;
    q.routed = d[i].routed ? 1 : 0;
    q.m_tiles = (d[i].M + kWgBM - 1) / kWgBM;
    q.n_tiles = (d[i].N + kWgBN - 1) / kWgBN;
    q.tile0 = tiles;
    tiles += q.m_tiles * q.n_tiles * (d[i].routed ? c.E : 1);
  }
  P.nprob = n;
  P.total_tiles = tiles;
  P.counts = counts;
  P.offsets = offsets;
  P.E = c.E;
  P.dense_rows = c.T;
  P.status = status;
  auto kern = accumulate ? wgrad_kernel<true> : wgrad_kernel<false>;
  MOE_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kWgSmemBytes));
  const int grid = tiles < sm_count() ? tiles : sm_count();
  MOE_TRY(launch_pdl(kern, dim3(grid), dim3(kWgThreads), kWgSmemBytes, s, P));
  return launch_check();
}

bool wants_routed_wgrad(const moe_weight_grads* dw) {
  return dw && (dw->dw1 || dw->dw3 || dw->dw2);
}

template <int TILE_N, bool PAIR>
moe_status backward_steps(const moe_config& c, const moe_weights& w, const moe_bwd_weights& wb,
                          const moe_fwd_saved& f, const void* dy, void* dx, float* dlogits,
                          float* dgate, const moe_weight_grads* dw, void* ws, cudaStream_t s) {
  const BwdLayout L = bwd_layout(c);
  uint8_t* b = static_cast<uint8_t*>(ws);
  int32_t* status = status_ptr(ws);
  const bool sh = c.I_shared > 0;
  const int H = c.H, I = c.I, Is = c.I_shared;
  const int Kd = static_cast<int>(dense_bwd_cols(c));
  auto bfp = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(b + off); };
  // combine backward: dO rows, dgate, and the router's dlogits (fp32, and the
  // bf16 copy in the dense operand)
  CombineBwdArgs cb;
  cb.dy = static_cast<const __nv_bfloat16*>(dy);
  cb.out_rows = static_cast<const __nv_bfloat16*>(f.out_rows);
  cb.token_row = f.token_row;
  cb.topk_idx = f.topk_idx;
  cb.topk_w = f.topk_w;
  cb.logits = f.logits;
  cb.dO = bfp(L.dO);
  cb.dgate = dgate ? dgate : reinterpret_cast<float*>(b + L.dgate);
  cb.dlogits = dlogits;
  cb.dense_b = bfp(L.dense_b);
  cb.T = c.T;
  cb.H = H;
  cb.k = c.top_k;
  cb.E = c.E;
  cb.col_b = 2 * (sh ? Is : 0);
  cb.ld_b = Kd;
  cb.rsf = c.routed_scaling_factor;
  const dim3 cgrid((c.T + 7) / 8);  // a warp per token
  switch (c.top_k) {
    case 1: MOE_TRY(launch_pdl(combine_backward_kernel<1>, cgrid, dim3(256), 0, s, cb)); break;
    case 2: MOE_TRY(launch_pdl(combine_backward_kernel<2>, cgrid, dim3(256), 0, s, cb)); break;
    case 3: MOE_TRY(launch_pdl(combine_backward_kernel<3>, cgrid, dim3(256), 0, s, cb)); break;
    case 4: MOE_TRY(launch_pdl(combine_backward_kernel<4>, cgrid, dim3(256), 0, s, cb)); break;
    case 5: MOE_TRY(launch_pdl(combine_backward_kernel<5>, cgrid, dim3(256), 0, s, cb)); break;
    case 7: MOE_TRY(launch_pdl(combine_backward_kernel<7>, cgrid, dim3(256), 0, s, cb)); break;
    case 6: MOE_TRY(launch_pdl(combine_backward_kernel<6>, cgrid, dim3(256), 0, s, cb)); break;
    case 8: MOE_TRY(launch_pdl(combine_backward_kernel<8>, cgrid, dim3(256), 0, s, cb)); break;
    default: MOE_TRY(launch_pdl(combine_backward_kernel<0>, cgrid, dim3(256), 0, s, cb)); break;
  }
  MOE_TRY(launch_check());
  const unsigned g = static_cast<unsigned>(sm_count() * 8);
  if (wants_routed_wgrad(dw)) {
    // dO^T h contracts over the pad rows too: they must hold zeros
    MOE_TRY(launch_pdl(zero_pad_rows_kernel, dim3(g), dim3(256), 0, s, bfp(L.dO), H,
                       f.row_token, f.offsets + c.E));
    MOE_TRY(launch_check());
  }
  // dh = dO W2 (the shared expert's: dy Ws2)
  MOE_TRY((rows_gemm<TILE_N, PAIR>(c, wb.w2t, I, H, b + L.dO, b + L.dh, sh ? wb.ws2t : nullptr,
                                   Is, H, dy, b + L.dh_s, f.counts, f.offsets, status, s)));
  // [a | u] recomputed from the saved rows in one fc1 pass (the shared
  // expert's into the dense operand), then the SwiGLU backward in place:
  // [da | du] per expert-major row (pads zeroed) and h for dW2
  MOE_TRY((fc1_recompute<TILE_N, PAIR>(c, w, f.rows, f.x, b + L.dz, b + L.dense_b, Kd, f.counts,
                                       f.offsets, status, s)));
  const bool want_h = dw && dw->dw2;
  MOE_TRY(launch_pdl(swiglu_backward_kernel, dim3(g), dim3(256), 0, s, bfp(L.dz),
                     static_cast<int64_t>(2 * I), static_cast<const __nv_bfloat16*>(bfp(L.dh)),
                     want_h ? bfp(L.h) : nullptr, f.row_token, f.offsets + c.E,
                     static_cast<int64_t>(L.r_cap), I));
  MOE_TRY(launch_check());
  if (sh) {
    const bool want_hs = dw && dw->dws2;
    MOE_TRY(launch_pdl(swiglu_backward_kernel, dim3(g), dim3(256), 0, s, bfp(L.dense_b),
                       static_cast<int64_t>(Kd), static_cast<const __nv_bfloat16*>(bfp(L.dh_s)),
                       want_hs ? bfp(L.h_s) : nullptr, static_cast<const int32_t*>(nullptr),
                       static_cast<const int32_t*>(nullptr), static_cast<int64_t>(c.T), Is));
    MOE_TRY(launch_check());
  }
  // dX rows = [da | du] [W1; W3] (K = 2I); dense dx = [da_s | du_s | dlogits]
  // [Ws1; Ws3; W_r] (K = Kd)
  MOE_TRY((rows_gemm<TILE_N, PAIR>(c, wb.w13t, H, 2 * I, b + L.dz, b + L.dX, wb.wdt, H, Kd,
                                   b + L.dense_b, b + L.dx_dense, f.counts, f.offsets, status,
                                   s)));
  // dx[t] = sum_j dX[row(t, j)] + dense dx[t]
  MOE_TRY(do_combine(c, b + L.dX, f.token_row, nullptr, b + L.dx_dense, dx, s));
  if (!dw) return MOE_OK;
  // weight gradients; the long dense contractions (K = T) first
  WgDesc d[kWgMaxProblems];
  int n = 0;
  const __nv_bfloat16* db = bfp(L.dense_b);
  if (dw->dw_router)
    d[n++] = WgDesc{db + 2 * (sh ? Is : 0), Kd, static_cast<int>(ceil64(c.E)), f.x, H, c.E, H,
                    dw->dw_router, false};
  if (sh && dw->dws1) d[n++] = WgDesc{db, Kd, Is, f.x, H, Is, H, dw->dws1, false};
  if (sh && dw->dws3) d[n++] = WgDesc{db + Is, Kd, Is, f.x, H, Is, H, dw->dws3, false};
  if (sh && dw->dws2) d[n++] = WgDesc{dy, H, H, bfp(L.h_s), Is, H, Is, dw->dws2, false};
  if (dw->dw1) d[n++] = WgDesc{bfp(L.dz), 2 * I, I, f.rows, H, I, H, dw->dw1, true};
  if (dw->dw3) d[n++] = WgDesc{bfp(L.dz) + I, 2 * I, I, f.rows, H, I, H, dw->dw3, true};
  if (dw->dw2) d[n++] = WgDesc{bfp(L.dO), H, H, bfp(L.h), I, H, I, dw->dw2, true};
  return launch_wgrad(c, d, n, dw->accumulate != 0, f.counts, f.offsets, status, s);
}

moe_status check_bwd(const moe_config& c, const moe_weights* w, const moe_bwd_weights* wb,
                     const moe_fwd_saved* f, const void* dy, void* dx,
                     const moe_weight_grads* dw) {
  if (!is_bf16(c)) return MOE_ERR_UNSUPPORTED;
  MOE_TRY(check_weights(c, w));
  if (!wb || !wb->w2t || !wb->w13t || !wb->wdt) return MOE_ERR_INVALID_ARG;
  if (!aligned16(wb->w2t) || !aligned16(wb->w13t) || !aligned16(wb->wdt)) return MOE_ERR_INVALID_ARG;
  if (c.I_shared > 0 && (!wb->ws2t || !aligned16(wb->ws2t))) return MOE_ERR_INVALID_ARG;
  if (!f || !f->x || !f->rows || !f->logits || !f->topk_idx || !f->topk_w || !f->counts ||
      !f->offsets || !f->row_token || !f->token_row || !f->out_rows)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(f->x) || !aligned16(f->rows) || !aligned16(f->out_rows)) return MOE_ERR_INVALID_ARG;
  if (!dy || !dx || !aligned16(dy) || !aligned16(dx)) return MOE_ERR_INVALID_ARG;
  if (dw) {
    if (wants_routed_wgrad(dw) && c.pad_multiple % 64 != 0) return MOE_ERR_UNSUPPORTED;
    if (c.I_shared <= 0 && (dw->dws1 || dw->dws3 || dw->dws2)) return MOE_ERR_INVALID_ARG;
    const float* all[7] = {dw->dw1, dw->dw3, dw->dw2, dw->dws1, dw->dws3, dw->dws2, dw->dw_router};
    for (const float* q : all)
      if (q && !aligned16(q)) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_backward_weights_size(const moe_config* cfg, moe_bwd_weight_sizes* sizes) {
  MOE_TRY(check_config(cfg));
  if (!is_bf16(*cfg)) return MOE_ERR_UNSUPPORTED;
  if (!sizes) return MOE_ERR_INVALID_ARG;
  const size_t H = cfg->H, I = cfg->I, E = cfg->E, Is = cfg->I_shared > 0 ? cfg->I_shared : 0;
  sizes->w2t = E * I * H * 2;
  sizes->w13t = E * H * 2 * I * 2;
  sizes->ws2t = Is * H * 2;
  sizes->wdt = H * static_cast<size_t>(dense_bwd_cols(*cfg)) * 2;
  return MOE_OK;
}

moe_status moe_prepare_backward_weights(const moe_config* cfg, int32_t which, int32_t e_begin,
                                        int32_t e_count, const void* w1, const void* w3,
                                        const void* w2, const void* w_router,
                                        const moe_bwd_weights* dst, void* stream) {
  MOE_TRY(check_config(cfg));
  if (!is_bf16(*cfg)) return MOE_ERR_UNSUPPORTED;
  if (!dst) return MOE_ERR_INVALID_ARG;
  const moe_config& c = *cfg;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto bf = [](const void* p) { return static_cast<const __nv_bfloat16*>(p); };
  auto run = [&](const TransposeArgs& a) -> moe_status {
    const dim3 grid(static_cast<unsigned>(a.rows / 64), static_cast<unsigned>(a.cols / 64));
    transpose_tiles_kernel<<<grid, 256, 0, s>>>(a);
    return launch_check();
  };
  const int64_t H = c.H, I = c.I;
  if (which == 0) {
    if (e_begin < 0 || e_count < 1 || e_begin + e_count > c.E) return MOE_ERR_INVALID_ARG;
    if (!w1 || !w3 || !w2 || !dst->w2t || !dst->w13t) return MOE_ERR_INVALID_ARG;
    // the experts' rows are contiguous in both tile-major copies
    TransposeArgs a2;
    memset(&a2, 0, sizeof(a2));
    a2.seg[0] = TransposeSeg{bf(w2), H * I, static_cast<int>(I), 0, static_cast<int>(H)};
    a2.nseg = 1;
    a2.dst = static_cast<__nv_bfloat16*>(dst->w2t) + static_cast<size_t>(e_begin) * I * H;
    a2.rows = static_cast<int64_t>(e_count) * I;
    a2.cols = static_cast<int>(H);
    a2.rows_per_group = static_cast<int>(I);
    MOE_TRY(run(a2));
    TransposeArgs a13;
    memset(&a13, 0, sizeof(a13));
    a13.seg[0] = TransposeSeg{bf(w1), I * H, static_cast<int>(H), 0, static_cast<int>(I)};
    a13.seg[1] = TransposeSeg{bf(w3), I * H, static_cast<int>(H), static_cast<int>(I),
                              static_cast<int>(I)};
    a13.nseg = 2;
    a13.dst = static_cast<__nv_bfloat16*>(dst->w13t) + static_cast<size_t>(e_begin) * H * 2 * I;
    a13.rows = static_cast<int64_t>(e_count) * H;
    a13.cols = static_cast<int>(2 * I);
    a13.rows_per_group = static_cast<int>(H);
    return run(a13);
  }
  if (which != 1 || e_begin != 0 || e_count != 1) return MOE_ERR_INVALID_ARG;
  if (!w_router || !dst->wdt) return MOE_ERR_INVALID_ARG;
  const int Is = c.I_shared > 0 ? c.I_shared : 0;
  if (Is > 0) {
    if (!w1 || !w3 || !w2 || !dst->ws2t) return MOE_ERR_INVALID_ARG;
    TransposeArgs a2;
    memset(&a2, 0, sizeof(a2));
    a2.seg[0] = TransposeSeg{bf(w2), 0, Is, 0, static_cast<int>(H)};
    a2.nseg = 1;
    a2.dst = static_cast<__nv_bfloat16*>(dst->ws2t);
    a2.rows = Is;
    a2.cols = static_cast<int>(H);
    a2.rows_per_group = Is;
    MOE_TRY(run(a2));
  }
  TransposeArgs ad;
  memset(&ad, 0, sizeof(ad));
  int n = 0;
  if (Is > 0) {
    ad.seg[n++] = TransposeSeg{bf(w1), 0, static_cast<int>(H), 0, Is};
    ad.seg[n++] = TransposeSeg{bf(w3), 0, static_cast<int>(H), Is, Is};
  }
  ad.seg[n++] = TransposeSeg{bf(w_router), 0, static_cast<int>(H), 2 * Is, c.E};
  ad.nseg = n;
  ad.dst = static_cast<__nv_bfloat16*>(dst->wdt);
  ad.rows = H;
  ad.cols = static_cast<int>(dense_bwd_cols(c));
  ad.rows_per_group = static_cast<int>(H);
  return run(ad);
}

moe_status moe_backward_workspace_size(const moe_config* cfg, size_t* bytes) {
  MOE_TRY(check_config(cfg));
  if (!is_bf16(*cfg)) return MOE_ERR_UNSUPPORTED;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = bwd_layout(*cfg).total;
  return MOE_OK;
}

moe_status moe_backward(const moe_config* cfg, const moe_weights* w, const moe_bwd_weights* wb,
                        const moe_fwd_saved* saved, const void* dy, void* dx, float* dlogits,
                        float* dgate, const moe_weight_grads* dw, void* workspace,
                        size_t workspace_bytes, void* stream) {
  MOE_TRY(check_config(cfg));
  const moe_config& c = *cfg;
  MOE_TRY(check_bwd(c, w, wb, saved, dy, dx, dw));
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % kAlign) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < bwd_layout(c).total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // tiles as the forward's bf16 grouped GEMMs pick them
  const bool small = static_cast<int64_t>(c.T) * c.top_k <= 32LL * c.E;
  if (small)
    return backward_steps<64, false>(c, *w, *wb, *saved, dy, dx, dlogits, dgate, dw, workspace, s);
  if (use_pairs(c, saved->rows))
    return backward_steps<256, true>(c, *w, *wb, *saved, dy, dx, dlogits, dgate, dw, workspace, s);
  return backward_steps<256, false>(c, *w, *wb, *saved, dy, dx, dlogits, dgate, dw, workspace, s);
}

}  // extern "C"
