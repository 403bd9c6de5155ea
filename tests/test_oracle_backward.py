"""Pins of the oracle's backward (input gradients of the bf16 layer) by
central finite differences of its own forward, on tiny shapes where every
coordinate can be perturbed (TransformerEngine PR "DeepSeekV3Layer",
Performance, "fused grouped MLP" row: the dGLU backward and the grouped GEMMs
of the backward pass; the forward is the DeepSeekV3MoE bullet of the same PR).

The backward differentiates the smooth function (bf16 storage read as the
identity, forward with rounding=False); the selection is piecewise constant,
so the shapes are drawn with clear score margins and the step is small."""

import numpy as np

import synth
from oracle import moe_oracle as O


def _fd(f, x, eps):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        xp, xm = x.copy(), x.copy()
        xp[i] += eps
        xm[i] -= eps
        g[i] = (f(xp) - f(xm)) / (2 * eps)
    return g


def test_expert_backward_matches_finite_differences():
    rng = np.random.default_rng(0)
    m, H, I = 3, 8, 5
    X = rng.normal(size=(m, H))
    W1, W3 = rng.normal(size=(I, H)) * 0.5, rng.normal(size=(I, H)) * 0.5
    W2 = rng.normal(size=(H, I)) * 0.5
    dO = rng.normal(size=(m, H))

    def loss(Xv):
        return float(np.sum(dO * (O.swiglu(Xv @ W1.T, Xv @ W3.T) @ W2.T)))

    dX, mid = O.expert_backward(X, W1, W3, W2, dO)
    fd = _fd(loss, X, 1e-6)
    assert np.max(np.abs(dX - fd)) < 1e-7 * max(1.0, np.abs(fd).max())
    # the SwiGLU derivative on its own: d(silu(a) u)/da and /du
    a, u = mid["a"], mid["u"]
    fa = _fd(lambda av: float(np.sum(mid["dh"] * O.swiglu(av, u))), a, 1e-6)
    fu = _fd(lambda uv: float(np.sum(mid["dh"] * O.swiglu(a, uv))), u, 1e-6)
    assert np.allclose(mid["da"], fa, rtol=1e-6, atol=1e-9)
    assert np.allclose(mid["du"], fu, rtol=1e-6, atol=1e-9)


def test_gate_backward_matches_finite_differences():
    rng = np.random.default_rng(1)
    T, E, G, g, k, rsf = 5, 8, 2, 1, 3, 2.5
    logits = rng.normal(size=(T, E)) * 2
    bias = np.zeros(E)
    r = O.route(logits, bias, G, g, k, rsf)
    assert r["expert_margin"].min() > 1e-3 and r["group_margin"].min() > 1e-3
    dgate = rng.normal(size=(T, k))

    def loss(lv):
        rr = O.route(lv, bias, G, g, k, rsf)
        assert np.array_equal(rr["idx"], r["idx"])  # the selection does not move
        return float(np.sum(dgate * rr["w"]))

    dl = O.gate_backward(logits, r["idx"], rsf, dgate)
    fd = _fd(loss, logits, 1e-6)
    assert np.max(np.abs(dl - fd)) < 1e-8
    unselected = np.ones((T, E), dtype=bool)
    np.put_along_axis(unselected, r["idx"], False, axis=1)
    assert np.all(dl[unselected] == 0)


def test_layer_backward_matches_finite_differences():
    cfg = synth.MoEShape(name="bwd_tiny", T=4, H=16, I=8, E=4, n_group=2, topk_group=1,
                         top_k=2, rsf=2.5, I_shared=8, dtype="bf16", pad_multiple=1,
                         router_std=0.5)
    rng = np.random.default_rng(3)
    x = rng.normal(size=(cfg.T, cfg.H))
    wr = rng.normal(size=(cfg.E, cfg.H)) * 0.5
    bias = rng.uniform(-0.1, 0.1, size=cfg.E)
    w1 = rng.normal(size=(cfg.E, cfg.I, cfg.H)) * 0.3
    w3 = rng.normal(size=(cfg.E, cfg.I, cfg.H)) * 0.3
    w2 = rng.normal(size=(cfg.E, cfg.H, cfg.I)) * 0.3
    sh = tuple(rng.normal(size=s) * 0.3 for s in ((8, 16), (8, 16), (16, 8)))
    dy = rng.normal(size=(cfg.T, cfg.H))
    b = O.backward(cfg, x, wr, bias, w1, w3, w2, dy, shared=sh, rounding=False)
    r = b["fwd"]["route"]
    assert r["expert_margin"].min() > 1e-4 and r["group_margin"].min() > 1e-4

    def loss(xv):
        f = O.forward(cfg, xv, wr, bias, w1, w3, w2, shared=sh, rounding=False)
        assert np.array_equal(f["route"]["idx"], r["idx"])
        return float(np.sum(dy * f["y"]))

    fd = _fd(loss, x, 1e-6)
    assert np.max(np.abs(b["dx"] - fd)) < 1e-6 * max(1.0, np.abs(fd).max())
    # without the router term the gradient is wrong: the pin sees every part
    assert np.max(np.abs((b["dx"] - b["dlogits"] @ wr) - fd)) > 1e-3


def test_layer_weight_grads_match_finite_differences():
    """dW1, dW3, dW2 per expert, the shared expert's and the router's weight
    gradients, each entry against a central difference of the loss."""
    cfg = synth.MoEShape(name="bwd_tiny_w", T=5, H=16, I=8, E=4, n_group=2, topk_group=1,
                         top_k=2, rsf=2.5, I_shared=8, dtype="bf16", pad_multiple=1,
                         router_std=0.5)
    rng = np.random.default_rng(7)
    x = rng.normal(size=(cfg.T, cfg.H))
    wr = rng.normal(size=(cfg.E, cfg.H)) * 0.5
    bias = rng.uniform(-0.1, 0.1, size=cfg.E)
    W = {"w1": rng.normal(size=(cfg.E, cfg.I, cfg.H)) * 0.3,
         "w3": rng.normal(size=(cfg.E, cfg.I, cfg.H)) * 0.3,
         "w2": rng.normal(size=(cfg.E, cfg.H, cfg.I)) * 0.3,
         "ws1": rng.normal(size=(8, 16)) * 0.3, "ws3": rng.normal(size=(8, 16)) * 0.3,
         "ws2": rng.normal(size=(16, 8)) * 0.3, "wr": wr}
    dy = rng.normal(size=(cfg.T, cfg.H))

    def run(V, **kw):
        return O.backward(cfg, x, V["wr"], bias, V["w1"], V["w3"], V["w2"], dy,
                          shared=(V["ws1"], V["ws3"], V["ws2"]), rounding=False, **kw)

    b = run(W, weight_grads=True)
    r = b["fwd"]["route"]
    assert r["expert_margin"].min() > 1e-4 and r["group_margin"].min() > 1e-4
    counts = b["fwd"]["maps"]["counts"]
    assert (counts > 0).any()

    def loss(V):
        f = O.forward(cfg, x, V["wr"], bias, V["w1"], V["w3"], V["w2"],
                      shared=(V["ws1"], V["ws3"], V["ws2"]), rounding=False)
        assert np.array_equal(f["route"]["idx"], r["idx"])
        return float(np.sum(dy * f["y"]))

    analytic = {
        "w1": np.stack([b["dw1"][e] for e in range(cfg.E)]),
        "w3": np.stack([b["dw3"][e] for e in range(cfg.E)]),
        "w2": np.stack([b["dw2"][e] for e in range(cfg.E)]),
        "ws1": b["dws1"], "ws3": b["dws3"], "ws2": b["dws2"], "wr": b["dw_router"]}
    eps = 1e-6
    for name, g in analytic.items():
        # 24 entries per weight, drawn over every expert and position
        for flat in rng.choice(g.size, size=min(24, g.size), replace=False):
            i = np.unravel_index(flat, g.shape)
            Vp = dict(W); Vm = dict(W)
            Vp[name] = W[name].copy(); Vm[name] = W[name].copy()
            Vp[name][i] += eps
            Vm[name][i] -= eps
            fd = (loss(Vp) - loss(Vm)) / (2 * eps)
            assert abs(g[i] - fd) < 1e-6 * max(1.0, abs(fd)), (name, i, g[i], fd)
    # experts no token picked have zero gradients
    for e in range(cfg.E):
        if counts[e] == 0:
            assert not analytic["w1"][e].any() and not analytic["w2"][e].any()


def test_backward_closed_forms():
    """Two closed forms that need no finite differences.
    (i) Every expert the same (W1, W3, W2): y = rsf * MLP(x) for any routing, so
        dlogits = 0, dx = the single expert's input gradient for dO = rsf * dy,
        and the experts' weight gradients sum to that expert's for the same dO.
    (ii) top_k = 1: the gate is rsf whatever the logits, so dlogits = 0."""
    rng = np.random.default_rng(11)
    cfg = synth.MoEShape(name="bwd_same", T=6, H=16, I=8, E=4, n_group=2, topk_group=2,
                         top_k=2, rsf=2.5, I_shared=0, dtype="bf16", pad_multiple=1,
                         router_std=0.5)
    x = rng.normal(size=(cfg.T, cfg.H))
    wr = rng.normal(size=(cfg.E, cfg.H)) * 0.5
    bias = rng.uniform(-0.1, 0.1, size=cfg.E)
    W1 = rng.normal(size=(cfg.I, cfg.H)) * 0.3
    W3 = rng.normal(size=(cfg.I, cfg.H)) * 0.3
    W2 = rng.normal(size=(cfg.H, cfg.I)) * 0.3
    dy = rng.normal(size=(cfg.T, cfg.H))
    rep = lambda W: np.stack([W] * cfg.E)
    b = O.backward(cfg, x, wr, bias, rep(W1), rep(W3), rep(W2), dy, rounding=False,
                   weight_grads=True)
    assert np.max(np.abs(b["dlogits"])) < 1e-12
    dX, mid = O.expert_backward(x, W1, W3, W2, cfg.rsf * dy)
    assert np.allclose(b["dx"], dX, rtol=1e-10, atol=1e-12)
    d1, d3, d2 = O.expert_weight_grads(x, cfg.rsf * dy, mid, rounding=False)
    assert np.allclose(sum(b["dw1"].values()), d1, rtol=1e-10, atol=1e-12)
    assert np.allclose(sum(b["dw3"].values()), d3, rtol=1e-10, atol=1e-12)
    assert np.allclose(sum(b["dw2"].values()), d2, rtol=1e-10, atol=1e-12)
    assert np.allclose(b["dw_router"], 0.0, atol=1e-12)

    cfg1 = cfg.scaled(name="bwd_top1", top_k=1, topk_group=1)
    w1 = rng.normal(size=(cfg.E, cfg.I, cfg.H)) * 0.3
    w3 = rng.normal(size=(cfg.E, cfg.I, cfg.H)) * 0.3
    w2 = rng.normal(size=(cfg.E, cfg.H, cfg.I)) * 0.3
    b1 = O.backward(cfg1, x, wr, bias, w1, w3, w2, dy, rounding=False)
    assert np.max(np.abs(b1["dlogits"])) < 1e-12
    assert np.abs(b1["dgate"]).max() > 1e-3   # the gate's own gradient is not zero
