"""Pins of the oracle's expert math and whole-layer forward: explicit loops on
tiny shapes, and closed forms the layer must satisfy whatever the routing
(TransformerEngine PR "DeepSeekV3Layer", Description, DeepSeekV3MoE bullet:
GroupedLinear -> ScaledSwiGLU -> GroupedLinear, gate-weighted combine, optional
shared expert)."""

import math

import numpy as np
import pytest

import synth
from oracle import moe_oracle as O


def test_swiglu_closed_forms():
    assert O.silu(np.array([0.0]))[0] == 0.0
    assert abs(O.silu(np.array([50.0]))[0] - 50.0) < 1e-12
    assert abs(O.silu(np.array([-50.0]))[0]) < 1e-18
    a, u = 1.3, -0.7
    assert abs(O.swiglu(np.array([a]), np.array([u]))[0] - a * u / (1 + math.exp(-a))) < 1e-15


def test_expert_math_explicit_loops():
    rng = np.random.default_rng(0)
    m, H, I = 3, 8, 4
    X = O.round_bf16(rng.normal(size=(m, H)))
    W1 = O.round_bf16(rng.normal(size=(I, H)))
    W3 = O.round_bf16(rng.normal(size=(I, H)))
    W2 = O.round_bf16(rng.normal(size=(H, I)))
    h = O.expert_fc1(X, W1, W3)
    o = O.expert_fc2(h, W2)
    for r in range(m):
        for i in range(I):
            a = math.fsum(X[r, q] * W1[i, q] for q in range(H))
            u = math.fsum(X[r, q] * W3[i, q] for q in range(H))
            ref = a / (1 + math.exp(-a)) * u
            assert abs(h[r, i] - ref) <= abs(ref) * 2.0 ** -8 + 1e-300
        for q in range(H):
            ref = math.fsum(h[r, i] * W2[q, i] for i in range(I))
            assert abs(o[r, q] - ref) <= abs(ref) * 2.0 ** -8 + 1e-300


def _tiny(**kw):
    cfg = synth.get_config("tiny_bf16_T64").scaled(**kw)
    d = synth.gen_all(cfg)
    f = {k: O.from_bf16(v) if v.dtype != __import__("torch").float32 else v.numpy().astype(np.float64)
         for k, v in d.items()}
    return cfg, f


def _fwd(cfg, f, **over):
    g = dict(f)
    g.update(over)
    sh = (g["ws1"], g["ws3"], g["ws2"]) if "ws1" in g else None
    return O.forward(cfg, g["x"], g["w_router"], g["bias"], g["w1"], g["w3"], g["w2"], shared=sh)


def test_identical_experts_give_rsf_times_mlp():
    cfg, f = _tiny()
    w1 = np.repeat(f["w1"][:1], cfg.E, axis=0)
    w3 = np.repeat(f["w3"][:1], cfg.E, axis=0)
    w2 = np.repeat(f["w2"][:1], cfg.E, axis=0)
    out = _fwd(cfg, f, w1=w1, w3=w3, w2=w2)
    o = O.expert_fc2(O.expert_fc1(f["x"], w1[0], w3[0]), w2[0])
    ref = cfg.rsf * o
    assert np.all(np.abs(out["y"] - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)


def test_single_expert_layer():
    cfg, f = _tiny(E=1, n_group=1, topk_group=1, top_k=1)
    f["w_router"], f["bias"] = f["w_router"][:1], f["bias"][:1]
    for k in ("w1", "w3", "w2"):
        f[k] = f[k][:1]
    out = _fwd(cfg, f)
    assert np.all(out["route"]["w"] == cfg.rsf)
    o = O.expert_fc2(O.expert_fc1(f["x"], f["w1"][0], f["w3"][0]), f["w2"][0])
    assert np.array_equal(out["y"], O.round_bf16(cfg.rsf * o))


def test_w2_scaling_scales_output():
    cfg, f = _tiny()
    a = _fwd(cfg, f)
    b = _fwd(cfg, f, w2=f["w2"] * 2.0)
    assert np.array_equal(b["y"], 2.0 * a["y"])


def test_zero_input_gives_zero_output():
    cfg, f = _tiny()
    out = _fwd(cfg, f, x=np.zeros_like(f["x"]))
    assert np.all(out["y"] == 0)


def test_token_permutation_equivariance():
    cfg, f = _tiny()
    perm = np.random.default_rng(3).permutation(cfg.T)
    a = _fwd(cfg, f)
    b = _fwd(cfg, f, x=f["x"][perm])
    assert np.array_equal(b["y"], a["y"][perm])


def test_shared_expert_adds():
    cfg, f = _tiny(I_shared=128)
    sh = synth.gen_shared_weights(cfg)
    ws = [O.from_bf16(t) for t in sh]
    a = _fwd(cfg, f)
    b = _fwd(cfg, f, ws1=ws[0], ws3=ws[1], ws2=ws[2])
    s = O.expert_fc2(O.expert_fc1(f["x"], ws[0], ws[1]), ws[2])
    # y_b = bf16(routed_sum + s); compare before the final rounding
    routed = np.zeros_like(a["y"])
    tr = a["maps"]["token_row"].reshape(cfg.T, cfg.top_k)
    for j in range(cfg.top_k):
        routed += a["route"]["w"][:, j:j + 1] * a["out_rows"][tr[:, j]]
    assert np.array_equal(b["y"], O.round_bf16(routed + s))


@pytest.mark.parametrize("dtype", ["mxfp8", "nvfp4"])
def test_quantized_forward_close_to_bf16(dtype):
    # The quantized layer stays near the bf16 one (relative Frobenius), with
    # NVFP4 noisier than MXFP8.
    cfg, f = _tiny()
    ref = _fwd(cfg, f)["y"]
    q = _fwd(cfg.scaled(dtype=dtype, pad_multiple=128), f)["y"]
    rel = np.linalg.norm(q - ref) / np.linalg.norm(ref)
    assert rel < (0.08 if dtype == "mxfp8" else 0.3), rel
    assert rel > 1e-3
