"""Pins of the oracle's quantized expert composition against values worked by
hand (tests/golden/quantized_expert_hand.txt): x codes -> W1 || W3 codes under
one shared NVFP4 global -> fp64 SwiGLU -> bf16 h -> h codes and the h global ->
fc2 -> bf16 (sglang PR "Mistral Large 3 NVFP4 TRTLLM MoE support",
Modifications: W4A4 NVFP4; TransformerEngine PR "DeepSeekV3Layer",
Performance, MXFP8 rows; same PR, Description, DeepSeekV3MoE bullet).

Each stage is compared separately, so a dropped bf16 rounding of h, separate
W1 / W3 global scales or an h global taken over another scope fails here
(the fixture's comments show which values each of those would change)."""

import os

import numpy as np

import synth
from oracle import moe_oracle as O

FIXTURE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                       "quantized_expert_hand.txt")


def _fixture():
    d = {}
    with open(FIXTURE) as f:
        for line in f:
            parts = line.split("#")[0].split()
            if parts:
                d.setdefault(parts[0], []).append([float(v) for v in parts[1:]])
    return d


def _inputs(dtype):
    """The fixture's inputs: two token rows and one expert (zeros elsewhere)."""
    n = 16 if dtype == "nvfp4" else 32
    x = np.zeros((2, n))
    W1, W3, W2 = np.zeros((n, n)), np.zeros((n, n)), np.zeros((n, n))
    if dtype == "nvfp4":
        x[0, :3] = [3, 1.5, 1.25]
        x[1, :2] = [-6, 0.5]
        W1[0, 0] = 0.5
    else:
        x[0, :3] = [3, 1.5, 1.296875]
        x[1, :2] = [-1.9921875, 0.5]
        W1[0, 0] = 0.53125
    W1[1, 1] = 6.0
    W3[0, 0], W3[1, 1] = 0.6875, 0.25
    W2[0, 0], W2[1, 1] = 1.0, 0.5
    return x, W1, W3, W2


def _expect_rows(got, rows, width):
    """got[:, :width] equals the fixture rows exactly and the rest is zero."""
    ref = np.array([r[1:1 + width] for r in sorted(rows)])
    assert np.array_equal(got[:, :width], ref), (got[:, :width], ref)
    assert np.all(got[:, width:] == 0)


def _expect_weights(got, entries):
    ref = np.zeros_like(got)
    for r, c, v in entries:
        ref[int(r), int(c)] = v
    assert np.array_equal(got, ref)


def _check_expert(dtype):
    fx = _fixture()
    p = "nv" if dtype == "nvfp4" else "mx"
    x, W1, W3, W2 = _inputs(dtype)
    xq = O.quantize_dequantize(x, dtype)
    _expect_rows(xq, fx[p + "_x_deq"], 4)
    w1, w3, w2 = O.prepare_expert_weights(W1, W3, W2, dtype)
    _expect_weights(w1, fx[p + "_w1_deq"])
    _expect_weights(w3, fx[p + "_w3_deq"])
    # W2 row 0 = [1], row 1 = [0, 0.5] are exact in both formats
    _expect_weights(w2, [(0, 0, 1.0), (1, 1, 0.5)])
    h, o = O.expert_forward(xq, W1, W3, W2, dtype)
    _expect_rows(h, fx[p + "_h_bf16"], 2)
    g = None
    if dtype == "nvfp4":
        g = O.nvfp4_global_scale(np.abs(h).max())
        assert float(g) == fx["nv_h_global"][0][0]
    hq = O.quantize_dequantize(h, dtype, g)
    _expect_rows(hq, fx[p + "_h_deq"], 2)
    _expect_rows(o, fx[p + "_out"], 2)
    return x, W1, W3, W2, o


def test_nvfp4_expert_by_hand():
    _check_expert("nvfp4")


def test_mxfp8_expert_by_hand():
    _check_expert("mxfp8")


def test_nvfp4_h_global_is_per_expert():
    """In the whole layer the h global of an expert comes from that expert's
    rows only: expert 0 (the fixture's expert, tokens 0 and 1) gives the
    fixture's outputs even next to an expert whose h amax is three times
    larger (tokens 2 and 3).  One global over both experts' h would change
    expert 0's token-1 outputs (checked here too, so the case discriminates)."""
    fx = _fixture()
    x, W1, W3, W2, o_ref = _check_expert("nvfp4")
    W3b = W3.copy()
    W3b[0, 0], W3b[1, 1] = 2.0625, 0.75
    cfg = synth.MoEShape(name="hand_nv", T=4, H=16, I=16, E=2, n_group=1, topk_group=1,
                         top_k=1, rsf=1.0, I_shared=0, dtype="nvfp4", pad_multiple=1,
                         router_std=0.02)
    x4 = np.concatenate([x, x])             # same amax, so the same x global
    logits = np.array([[4.0, -4.0], [4.0, -4.0], [-4.0, 4.0], [-4.0, 4.0]])
    out = O.forward(cfg, x4, None, np.zeros(2), np.stack([W1, W1]), np.stack([W3, W3b]),
                    np.stack([W2, W2]), logits=logits)
    assert out["route"]["idx"][:, 0].tolist() == [0, 0, 1, 1]
    assert np.all(out["route"]["w"] == 1.0)
    rows_a = out["maps"]["token_row"][:2]
    _expect_rows(out["out_rows"][rows_a], fx["nv_out"], 2)
    _expect_rows(out["y"][:2], fx["nv_out"], 2)
    # the other reading, one global over both experts' h, differs
    h_b, _ = O.expert_forward(out["xq"][2:], W1, W3b, W2, "nvfp4")
    h_a = out["h_rows"][rows_a]
    g_all = O.nvfp4_global_scale(max(np.abs(h_a).max(), np.abs(h_b).max()))
    assert np.abs(h_b).max() == 10.125
    _, o_all = O.expert_forward(out["xq"][:2], W1, W3, W2, "nvfp4", h_global=g_all)
    assert not np.array_equal(o_all, o_ref)
    assert o_all[1, 0] == 0.6328125 and o_all[1, 1] == 0.158203125


def test_row_blocks_match_one_call():
    """The quantizers applied block by block (threads) give the one-call result."""
    rng = np.random.default_rng(5)
    v = O.round_bf16(rng.normal(size=(3 * O.ROW_BLOCK + 37, 512)) * 3)
    g = O.nvfp4_global_scale(np.abs(v).max())
    whole_nv = O.nvfp4_dequantize(*O.nvfp4_quantize(v, g), g)
    whole_mx = O.mxfp8_dequantize(*O.mxfp8_quantize(v))
    assert np.array_equal(O.quantize_dequantize(v, "nvfp4"), whole_nv)
    assert np.array_equal(O.quantize_dequantize(v, "mxfp8"), whole_mx)
