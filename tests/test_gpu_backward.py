"""Parity of the backward of the bf16 layer (moe_backward) with the oracle's
backward: dx, dgate, dlogits and every weight gradient, on the same seeded
inputs and the same routing (TransformerEngine PR "DeepSeekV3Layer",
Performance, "fused grouped MLP" row: the dGLU backward, the dgrad and wgrad
grouped GEMMs, and the router's gradient).

Tolerance: relative Frobenius error <= 1e-2 for every result, the bar the
forward's bf16 output meets.  The GPU stores six intermediates as bf16 on the
way to dx (dO, a, u, dh, da/du, dX) and accumulates each contraction in fp32;
each bf16 store adds a relative error of at most 2^-9 per element, about
1.1e-3 rms, so the expected error of dx is near sqrt(6) * 1.1e-3 = 2.7e-3.
The weight gradients take two bf16 operands each (about 1.6e-3 rms).
"""

import numpy as np
import pytest
import torch

import synth
from moe_testlib import f64, near_ties, rel_frob, run_steps, weights_dict
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

TOL = 1e-2

SHAPES = {
    # several 128 x 256 wgrad tiles per expert, shared expert, top_k 4
    "small_shared": synth.MoEShape(
        name="bwd_small_shared", T=256, H=512, I=256, E=16, n_group=4, topk_group=2, top_k=4,
        rsf=2.5, I_shared=256, dtype="bf16", pad_multiple=64, router_std=0.02),
    # ragged T, H not a multiple of the 256-column wgrad tile, E = 32 (a
    # partly empty router tile), top_k 6, skewed load
    "ragged_k6": synth.MoEShape(
        name="bwd_ragged_k6", T=333, H=384, I=128, E=32, n_group=8, topk_group=4, top_k=6,
        rsf=2.5, I_shared=0, dtype="bf16", pad_multiple=64, router_std=0.02, skew_experts=4,
        skew_factor=3.0),
    # decode-sized: most experts get no token (zero gradients), 64-token tiles
    "decode_shared": synth.MoEShape(
        name="bwd_decode_shared", T=8, H=256, I=128, E=16, n_group=4, topk_group=2, top_k=4,
        rsf=2.5, I_shared=128, dtype="bf16", pad_multiple=128, router_std=0.02),
    # top-8 (the DeepSeek-V3 fan-out) with a shared expert
    "top8_shared": synth.MoEShape(
        name="bwd_top8_shared", T=200, H=256, I=256, E=32, n_group=4, topk_group=4, top_k=8,
        rsf=2.5, I_shared=128, dtype="bf16", pad_multiple=64, router_std=0.02),
    # top-10: the combine kernels' generic (any top_k) form
    "top10": synth.MoEShape(
        name="bwd_top10", T=96, H=256, I=128, E=64, n_group=8, topk_group=4, top_k=10,
        rsf=1.0, I_shared=0, dtype="bf16", pad_multiple=64, router_std=0.02),
}


def _run(cfg, grads=True):
    import mixture_experts_layer_grouped_b200 as M
    d = synth.gen_all(cfg, "cuda")
    s = run_steps(cfg, d)
    assert s["status"] == 0
    c = M.config_from_shape(cfg)
    prepared = M.prepare_weights(c, weights_dict(d))
    bwd_w = M.prepare_backward_weights(c, weights_dict(d), d["w_router"])
    dy = synth.gen_dy(cfg, "cuda")
    saved = {k: s[k] for k in ("rows", "logits", "topk_idx", "topk_w", "counts", "offsets",
                               "row_token", "token_row", "out_rows")}
    saved["x"] = d["x"]
    T, H, E, I, Is, k = cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k
    dx = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    dlogits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    dgate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    g = None
    if grads:
        f32 = dict(dtype=torch.float32, device="cuda")
        g = {"dw1": torch.full((E, I, H), float("nan"), **f32),
             "dw3": torch.full((E, I, H), float("nan"), **f32),
             "dw2": torch.full((E, H, I), float("nan"), **f32),
             "dw_router": torch.full((E, H), float("nan"), **f32)}
        if Is:
            g["dws1"] = torch.full((Is, H), float("nan"), **f32)
            g["dws3"] = torch.full((Is, H), float("nan"), **f32)
            g["dws2"] = torch.full((H, Is), float("nan"), **f32)
    ws = M.binding.new_workspace(M.moe_backward_workspace_size(c), "cuda")
    M.moe_backward(c, prepared, bwd_w, saved, dy, dx, ws, dlogits=dlogits, dgate=dgate,
                   grads=g)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    return d, s, dy, dx, dlogits, dgate, g


def _oracle(cfg, d, s, dy, weight_grads=True):
    h = {k: f64(v) for k, v in d.items()}
    shared = (h["ws1"], h["ws3"], h["ws2"]) if cfg.I_shared else None
    b = O.backward(cfg, h["x"], h["w_router"], h["bias"], h["w1"], h["w3"], h["w2"], f64(dy),
                   shared=shared, logits=f64(s["logits"]), weight_grads=weight_grads)
    # the oracle routes on the GPU's fp32 logits; a near-tie could still
    # choose differently in fp64, which would make the gradients incomparable:
    # the selections must agree on every token (near-ties included)
    # the selections must agree on every token, near-ties included; a near-tie
    # may order two selected experts differently, and then the oracle's dgate
    # row is put in the GPU's order
    r = b["fwd"]["route"]
    gi = s["topk_idx"].cpu().numpy()
    same = np.all(np.sort(r["idx"], axis=1) == np.sort(gi, axis=1), axis=1)
    assert same.all(), ("routing differs", np.nonzero(~same)[0], near_ties(r).sum())
    for t in np.nonzero(np.any(r["idx"] != gi, axis=1))[0]:
        pos = {int(e): j for j, e in enumerate(r["idx"][t])}
        b["dgate"][t] = b["dgate"][t][[pos[int(e)] for e in gi[t]]]
    return b


@pytest.mark.parametrize("name", list(SHAPES))
def test_backward_matches_oracle(name):
    cfg = SHAPES[name]
    d, s, dy, dx, dlogits, dgate, g = _run(cfg)
    b = _oracle(cfg, d, s, dy)
    errs = {"dx": rel_frob(f64(dx), b["dx"]),
            "dgate": rel_frob(f64(dgate), b["dgate"]),
            "dlogits": rel_frob(f64(dlogits), b["dlogits"])}
    counts = s["counts"].cpu().numpy()
    for key in ("dw1", "dw3", "dw2"):
        got = f64(g[key])
        assert np.isfinite(got).all(), key
        ref = np.stack([b[key][e] for e in range(cfg.E)])
        errs[key] = rel_frob(got, ref)
        # experts no token picked: exactly zero
        assert not got[counts == 0].any(), key
    errs["dw_router"] = rel_frob(f64(g["dw_router"]), b["dw_router"])
    if cfg.I_shared:
        for key in ("dws1", "dws3", "dws2"):
            errs[key] = rel_frob(f64(g[key]), b[key])
    print(name, {k: f"{v:.2e}" for k, v in errs.items()})
    for key, v in errs.items():
        assert v <= TOL, (key, v)


def test_backward_without_weight_grads_matches():
    """dw = NULL: only dx, dlogits and dgate; the same values as with it."""
    cfg = SHAPES["small_shared"]
    _, _, _, dx0, dl0, dg0, _ = _run(cfg, grads=True)
    _, _, _, dx1, dl1, dg1, _ = _run(cfg, grads=False)
    assert torch.equal(dx0, dx1) and torch.equal(dl0, dl1) and torch.equal(dg0, dg1)


def test_backward_mid_size():
    """The mid bf16 layer with a shared expert (T=2048, H=2048, I=1024,
    E=64, top_k=6, skewed router), with 64-row segment pads: dx, dgate and
    dlogits over every token, the weight gradients of the most and least
    loaded experts and of the shared expert and the router."""
    cfg = synth.get_config("mid_bf16_shared_T2048").scaled(pad_multiple=64)
    d, s, dy, dx, dlogits, dgate, g = _run(cfg)
    counts = s["counts"].cpu().numpy()
    pick = [int(np.argmax(counts)), int(np.argmin(np.where(counts > 0, counts, 1 << 30)))]
    b = _oracle(cfg, d, s, dy, weight_grads=pick)
    errs = {"dx": rel_frob(f64(dx), b["dx"]),
            "dgate": rel_frob(f64(dgate), b["dgate"]),
            "dlogits": rel_frob(f64(dlogits), b["dlogits"]),
            "dw_router": rel_frob(f64(g["dw_router"]), b["dw_router"])}
    for key in ("dws1", "dws3", "dws2"):
        errs[key] = rel_frob(f64(g[key]), b[key])
    for e in pick:
        for key in ("dw1", "dw3", "dw2"):
            errs[f"{key}[{e}]"] = rel_frob(f64(g[key][e]), b[key][e])
    for key in ("dw1", "dw3", "dw2"):
        assert torch.isfinite(g[key]).all(), key
    print("mid", {k: f"{v:.2e}" for k, v in errs.items()})
    for key, v in errs.items():
        assert v <= TOL, (key, v)


@pytest.mark.slow
def test_backward_full_size_dsv4_bf16():
    """The DeepSeek-V4 routed-expert geometry in bf16 (T=4096, H=4096, I=2048,
    E=256, top-6) with 64-row pads, every token on the GPU.  The oracle routes
    from its own fp64 logits and checks, away from near-ties: the weight
    gradients of the most loaded expert and two seeded others (each from that
    expert's own rows and dO = w * dy), and dx, dgate and dlogits of eight
    tokens (their backward on their own: a token's gradients depend on no other
    token)."""
    import mixture_experts_layer_grouped_b200 as M
    from moe_testlib import check_routing, pick_tokens, prepare_streaming
    cfg = synth.get_config("dsv4_bf16_T4096").scaled(pad_multiple=64)
    c = M.config_from_shape(cfg)
    T, H, E, I, k = cfg.T, cfg.H, cfg.E, cfg.I, cfg.top_k
    x = synth.gen_x(cfg, "cuda")
    w_r, bias = synth.gen_router(cfg, "cuda")
    prepared = prepare_streaming(M, cfg)
    bw = {n: (torch.empty(v, dtype=torch.uint8, device="cuda") if v else None)
          for n, v in M.moe_backward_weights_size(c).items()}
    for e in range(E):
        M.moe_prepare_backward_weights(c, 0, e, 1, *synth.gen_expert_weights(cfg, e, "cuda"),
                                       None, bw)
    M.moe_prepare_backward_weights(c, 1, 0, 1, None, None, None, w_r, bw)
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes, "cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    sv = {"x": x, "logits": torch.empty(T, E, dtype=torch.float32, device="cuda"),
          "topk_idx": torch.empty(T, k, **i32),
          "topk_w": torch.empty(T, k, dtype=torch.float32, device="cuda"),
          "counts": torch.empty(E, **i32), "offsets": torch.empty(E + 1, **i32),
          "row_token": torch.empty(r_cap, **i32), "token_row": torch.empty(T * k, **i32),
          "rows": torch.empty(r_cap, H, dtype=torch.bfloat16, device="cuda"),
          "out_rows": torch.empty(r_cap, H, dtype=torch.bfloat16, device="cuda")}
    M.moe_route(c, x, w_r, bias, sv["topk_idx"], sv["topk_w"], ws, logits_out=sv["logits"])
    M.moe_permute(c, sv["topk_idx"], x, sv["counts"], sv["offsets"], sv["row_token"],
                  sv["token_row"], sv["rows"], ws)
    M.moe_grouped_mlp(c, prepared, sv["rows"], sv["counts"], sv["offsets"], sv["out_rows"], ws)
    dy = synth.gen_dy(cfg, "cuda")
    dx = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    dlogits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    dgate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    g = {"dw1": torch.empty(E, I, H, **f32), "dw3": torch.empty(E, I, H, **f32),
         "dw2": torch.empty(E, H, I, **f32), "dw_router": torch.empty(E, H, **f32)}
    wsb = M.binding.new_workspace(M.moe_backward_workspace_size(c), "cuda")
    M.moe_backward(c, prepared, bw, sv, dy, dx, wsb, dlogits=dlogits, dgate=dgate, grads=g)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0 and M.moe_get_device_status(wsb) == 0

    # the oracle's own routing
    xh, dyh = f64(x), f64(dy)
    wrh, bh = f64(w_r), f64(bias)
    logits = O.router_logits(xh, wrh)
    r = O.route(logits, bh, cfg.n_group, cfg.topk_group, cfg.top_k, cfg.rsf)
    idx_gpu = sv["topk_idx"].cpu().numpy()
    keep, bad = check_routing(r, idx_gpu, sv["topk_w"].cpu().numpy(), cfg.rsf)
    assert not bad, f"{len(bad)} tokens routed differently"
    bad_e = set(r["idx"][~keep].ravel().tolist()) | set(idx_gpu[~keep].ravel().tolist())
    weights = {}

    def expert(e):
        if e not in weights:
            weights[e] = tuple(f64(t) for t in synth.gen_expert_weights(cfg, e, "cuda"))
        return weights[e]

    # whole experts: weight gradients from the expert's own rows
    counts = np.bincount(r["idx"].ravel(), minlength=E)
    touched = [e for e in np.nonzero(counts)[0].tolist() if e not in bad_e]
    hot = max(touched, key=lambda e: (counts[e], -e))
    rng = np.random.default_rng(0)
    rest = [e for e in touched if e != hot]
    errs = {}
    for e in [hot] + sorted(rng.choice(rest, 2, replace=False).tolist()):
        tok, j = np.nonzero(r["idx"] == e)          # ascending tokens
        Xe = xh[tok]
        dOe = r["w"][tok, j][:, None] * dyh[tok]
        W1, W3, W2 = expert(e)
        _, mid = O.expert_backward(Xe, W1, W3, W2, dOe)
        d1, d3, d2 = O.expert_weight_grads(Xe, dOe, mid)
        errs[f"dw1[{e}]"] = rel_frob(f64(g["dw1"][e]), d1)
        errs[f"dw3[{e}]"] = rel_frob(f64(g["dw3"][e]), d3)
        errs[f"dw2[{e}]"] = rel_frob(f64(g["dw2"][e]), d2)
    # eight tokens end to end, sharing experts where they can
    cand = [t for t in np.nonzero(keep)[0].tolist() if not (set(r["idx"][t]) & bad_e)]
    toks, _ = pick_tokens(r["idx"], cand, [hot], 8, E, seed=1)
    toks = np.sort(toks)
    scfg = cfg.scaled(T=len(toks))
    w = [(lambda e, q=q: expert(e)[q]) for q in range(3)]
    b = O.backward(scfg, xh[toks], wrh, bh, w[0], w[1], w[2], dyh[toks], logits=logits[toks])
    assert np.array_equal(b["fwd"]["route"]["idx"], r["idx"][toks])
    errs["dx"] = rel_frob(f64(dx)[toks], b["dx"])
    errs["dgate"] = rel_frob(f64(dgate)[toks], b["dgate"])
    errs["dlogits"] = rel_frob(f64(dlogits)[toks], b["dlogits"])
    print("dsv4 bf16 backward", {kk: f"{v:.2e}" for kk, v in errs.items()})
    for kk, v in errs.items():
        assert v <= TOL, (kk, v)


def test_train_layer_gives_the_same_bits():
    """MoETrainLayer (forward through the step calls, then backward) gives the
    bits of the explicit calls above."""
    import mixture_experts_layer_grouped_b200 as M
    cfg = SHAPES["small_shared"]
    d, s, dy, dx, dlogits, dgate, g = _run(cfg)
    c = M.config_from_shape(cfg)
    layer = M.MoETrainLayer(c, weights_dict(d), d["w_router"], d["bias"])
    y = layer.forward(d["x"])
    res = layer.backward(dy)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(y, s["y"])
    assert torch.equal(res["dx"], dx) and torch.equal(res["dlogits"], dlogits)
    assert torch.equal(res["dgate"], dgate)
    for key in g:
        assert torch.equal(res[key], g[key]), key


def test_weight_grads_accumulate():
    """accumulate: a second backward adds its weight gradients to the first
    one's (x + x = 2x exactly in fp32), and experts no token picked keep the
    values that were there."""
    import mixture_experts_layer_grouped_b200 as M
    cfg = SHAPES["decode_shared"]  # most experts empty
    d = synth.gen_all(cfg, "cuda")
    c = M.config_from_shape(cfg)
    layer = M.MoETrainLayer(c, weights_dict(d), d["w_router"], d["bias"])
    layer.forward(d["x"])
    dy = synth.gen_dy(cfg, "cuda")
    once = layer.backward(dy)
    f32 = dict(dtype=torch.float32, device="cuda")
    acc = {k: once[k].clone() for k in ("dw1", "dw3", "dw2", "dw_router", "dws1", "dws3", "dws2")}
    empty = layer.saved["counts"] == 0
    assert bool(empty.any())
    marker = torch.full((int(empty.sum()), cfg.I, cfg.H), 7.0, **f32)
    acc["dw1"][empty] = marker
    twice = layer.backward(dy, grads=acc, accumulate=True)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(twice["dx"], once["dx"])
    full = ~empty
    assert torch.equal(acc["dw1"][full], 2 * once["dw1"][full])
    assert torch.equal(acc["dw1"][empty], marker)          # untouched
    for k in ("dw3", "dw2", "dw_router", "dws1", "dws3", "dws2"):
        assert torch.equal(acc[k], 2 * once[k]), k
