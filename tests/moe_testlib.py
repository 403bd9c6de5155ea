"""Helpers shared by the tests: marshalling between torch and the oracle's
numpy arrays, running the library's step calls, and the comparison rules.

Comparison rules (from the layer's statement of agreement):
* routing indices, permute maps and quantized codes: bit-exact, except tokens
  whose k-th and (k+1)-th biased scores (or g-th and (g+1)-th group scores)
  differ by less than 1e-5, which are left out of the index check and of the
  end-to-end sums;
* gates: |gpu - oracle| <= 1e-6 * routed_scaling_factor;
* end to end: relative Frobenius error <= 1e-2 (bf16), <= 2e-2 (MXFP8/NVFP4).
"""

import numpy as np
import torch

import synth
from oracle import moe_oracle as O

NEAR_TIE = 1e-5


def f64(t):
    if t.dtype == torch.bfloat16:
        return O.from_bf16(t)
    return t.detach().cpu().numpy().astype(np.float64)


def near_ties(r):
    """Boolean [T]: tokens whose selection is decided by a near-tie."""
    return (r["expert_margin"] < NEAR_TIE) | (r["group_margin"] < NEAR_TIE)


def rel_frob(a, b):
    d = np.linalg.norm(np.asarray(a, np.float64) - np.asarray(b, np.float64))
    n = np.linalg.norm(np.asarray(b, np.float64))
    return d / n if n > 0 else d


def check_routing(r, idx_gpu, w_gpu, rsf):
    """Compare a GPU routing with the oracle's on all non-near-tie tokens."""
    keep = ~near_ties(r)
    idx_o, w_o, b = r["idx"], r["w"], r["b"]
    bad = []
    for t in np.nonzero(keep)[0]:
        go, gg = idx_o[t], idx_gpu[t]
        sel_b = b[t, go]
        gaps = -np.diff(sel_b)
        if gaps.size == 0 or gaps.min() >= NEAR_TIE:
            same = np.array_equal(go, gg)
        else:
            same = np.array_equal(np.sort(go), np.sort(gg))
        if not same:
            bad.append(t)
            continue
        wo = dict(zip(go.tolist(), w_o[t].tolist()))
        for e, wv in zip(gg.tolist(), w_gpu[t].tolist()):
            if abs(wv - wo[e]) > 1e-6 * rsf:
                bad.append(t)
                break
    return keep, bad


def gen_device_inputs(cfg, device="cuda"):
    """All inputs of a workload on the device (routed weights stacked)."""
    return synth.gen_all(cfg, device)


def host_inputs(d):
    """float64 numpy copies of device inputs for the oracle."""
    return {k: f64(v) for k, v in d.items()}


def weights_dict(d):
    w = {k: d[k] for k in ("w1", "w3", "w2")}
    for k in ("ws1", "ws3", "ws2"):
        if k in d:
            w[k] = d[k]
    return w


def run_steps(cfg, d, logits_in=None):
    """Run route -> permute -> grouped MLP -> combine through the step calls."""
    import mixture_experts_layer_grouped_b200 as M
    c = M.config_from_shape(cfg)
    dev = d["x"].device
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes, dev)
    T, E, k, H = cfg.T, cfg.E, cfg.top_k, cfg.H
    i32 = dict(dtype=torch.int32, device=dev)
    out = {}
    out["logits"] = torch.empty(T, E, dtype=torch.float32, device=dev)
    out["topk_idx"] = torch.empty(T, k, **i32)
    out["topk_w"] = torch.empty(T, k, dtype=torch.float32, device=dev)
    M.moe_route(c, d["x"], d["w_router"], d["bias"], out["topk_idx"], out["topk_w"], ws,
                logits_in=logits_in, logits_out=None if logits_in is not None else out["logits"])
    out["counts"] = torch.empty(E, **i32)
    out["offsets"] = torch.empty(E + 1, **i32)
    out["row_token"] = torch.empty(r_cap, **i32)
    out["token_row"] = torch.empty(T * k, **i32)
    out["rows"] = torch.empty(r_cap, H, dtype=torch.bfloat16, device=dev)
    M.moe_permute(c, out["topk_idx"], d["x"], out["counts"], out["offsets"], out["row_token"],
                  out["token_row"], out["rows"], ws)
    out["out_rows"] = torch.zeros(r_cap, H, dtype=torch.bfloat16, device=dev)
    out["shared_out"] = (torch.empty(T, H, dtype=torch.bfloat16, device=dev)
                         if cfg.I_shared > 0 else None)
    prepared = M.prepare_weights(c, weights_dict(d))
    M.moe_grouped_mlp(c, prepared, out["rows"], out["counts"], out["offsets"],
                      out["out_rows"], ws, x=d["x"], shared_out=out["shared_out"])
    out["y"] = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    M.moe_combine(c, out["out_rows"], out["token_row"], out["topk_w"], out["y"],
                  shared_out=out["shared_out"])
    torch.cuda.synchronize()
    out["status"] = M.moe_get_device_status(ws)
    return out
