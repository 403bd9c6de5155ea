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


# ---------------------------------------------------------------------------
# Full-size layers: every token on the GPU, the oracle on samples it can take
# expert by expert.
# ---------------------------------------------------------------------------

TOL = {"bf16": 1e-2, "mxfp8": 2e-2, "nvfp4": 2e-2}


def prepare_streaming(M, cfg, device="cuda"):
    """Prepared weights of a workload, drawn and prepared one expert at a time
    (the whole bf16 layer never exists at once)."""
    c = M.config_from_shape(cfg)
    p = M.allocate_prepared_weights(c, device)
    dst = M.binding.weights_struct(p)
    for e in range(cfg.E):
        M.moe_prepare_weights(c, 0, e, 1, *synth.gen_expert_weights(cfg, e, device), dst)
    if cfg.I_shared:
        M.moe_prepare_weights(c, 1, 0, 1, *synth.gen_shared_weights(cfg, device), dst)
    return p


def run_layer_steps(M, cfg, x, w_r, bias, p):
    """The layer through the step calls (route, quantize, permute, grouped MLP,
    combine) on prepared weights; every intermediate comes back."""
    c = M.config_from_shape(cfg)
    dev = x.device
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes, dev)
    T, E, k, H = cfg.T, cfg.E, cfg.top_k, cfg.H
    i32 = dict(dtype=torch.int32, device=dev)
    o = {"logits": torch.empty(T, E, dtype=torch.float32, device=dev),
         "topk_idx": torch.empty(T, k, **i32),
         "topk_w": torch.empty(T, k, dtype=torch.float32, device=dev)}
    M.moe_route(c, x, w_r, bias, o["topk_idx"], o["topk_w"], ws, logits_out=o["logits"])
    q = cfg.dtype != "bf16"
    rb = {"bf16": 2 * H, "mxfp8": H, "nvfp4": H // 2}[cfg.dtype]
    xc = xs = xg = rows_sf = None
    if q:
        xc = torch.empty(T, rb, dtype=torch.uint8, device=dev)
        xs = torch.zeros(M.scale_bytes(T, H, cfg.dtype), dtype=torch.uint8, device=dev)
        xg = torch.empty(1, dtype=torch.float32, device=dev)
        M.moe_quantize(cfg.dtype, x, xc, xs, global_scale=xg)
        rows_sf = torch.zeros(M.scale_bytes(r_cap, H, cfg.dtype), dtype=torch.uint8, device=dev)
    o["counts"], o["offsets"] = torch.empty(E, **i32), torch.empty(E + 1, **i32)
    o["row_token"], o["token_row"] = torch.empty(r_cap, **i32), torch.empty(T * k, **i32)
    rows = torch.empty(r_cap, rb, dtype=torch.uint8, device=dev)
    M.moe_permute(c, o["topk_idx"], xc if q else x, o["counts"], o["offsets"], o["row_token"],
                  o["token_row"], rows, ws, src_scales=xs, dst_scales=rows_sf)
    o["out_rows"] = torch.zeros(r_cap, H, dtype=torch.bfloat16, device=dev)
    o["shared_out"] = (torch.empty(T, H, dtype=torch.bfloat16, device=dev)
                       if cfg.I_shared else None)
    M.moe_grouped_mlp(c, p, rows, o["counts"], o["offsets"], o["out_rows"], ws,
                      x=xc if q else x, shared_out=o["shared_out"], row_scales=rows_sf,
                      x_scales=xs, x_global=xg)
    o["y"] = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    M.moe_combine(c, o["out_rows"], o["token_row"], o["topk_w"], o["y"],
                  shared_out=o["shared_out"])
    torch.cuda.synchronize()
    o["status"] = M.moe_get_device_status(ws)
    return o


def pick_tokens(idx, candidates, start_experts, n, E, seed):
    """n tokens from `candidates`, greedily the ones whose experts are mostly
    among those already picked (seeded order breaks ties), so the oracle's
    per-expert work stays bounded.  Returns (tokens, experts needed)."""
    rng = np.random.default_rng(seed)
    order = rng.permutation(np.asarray(candidates))
    have = np.zeros(E, dtype=bool)
    have[list(start_experts)] = True
    chosen = []
    for _ in range(min(n, len(order))):
        new = (~have[idx[order]]).sum(axis=1)
        i = int(np.argmin(new))
        t = int(order[i])
        chosen.append(t)
        have[idx[t]] = True
        order = np.delete(order, i)
    return np.array(chosen), np.nonzero(have)[0]


def check_full_size(cfg, x, w_r, bias, gpu, n_experts=8, n_tokens=32, seed=0):
    """Compare a full-size GPU run with the oracle:
      * routing of every token (indices bit-exact, gates within 1e-6 * rsf,
        near-ties excluded), from the oracle's own fp64 router logits;
      * whole experts: the most loaded one and n_experts - 1 seeded others,
        their maps and every fc2 output row (rel. Frobenius per expert);
      * n_tokens tokens end to end (y, rel. Frobenius over the sample).
    Experts that hold a near-tie token, and tokens routed to one, are left out
    (a flipped selection changes the rows of the segment)."""
    dt = cfg.dtype
    tol = TOL[dt]
    xh = f64(x)
    r = O.route(O.router_logits(xh, f64(w_r)), f64(bias), cfg.n_group, cfg.topk_group,
                cfg.top_k, cfg.rsf)
    idx_gpu = gpu["topk_idx"].cpu().numpy()
    keep, bad = check_routing(r, idx_gpu, gpu["topk_w"].cpu().numpy(), cfg.rsf)
    assert not bad, f"{len(bad)} tokens routed differently, first {bad[:5]}"
    assert keep.mean() > 0.95
    idx = r["idx"]
    bad_e = set(idx[~keep].ravel().tolist()) | set(idx_gpu[~keep].ravel().tolist())
    mp = O.permute_maps(idx, cfg.E, cfg.pad_multiple)
    xq = O.quantize_dequantize(xh, dt)          # NVFP4: one global over all of x
    g_counts = gpu["counts"].cpu().numpy()
    g_off = gpu["offsets"].cpu().numpy()
    g_rt = gpu["row_token"].cpu().numpy()
    out_rows = gpu["out_rows"]
    rng = np.random.default_rng(seed)
    touched = [e for e in np.nonzero(mp["counts"] > 0)[0].tolist() if e not in bad_e]
    hot = max(touched, key=lambda e: (mp["counts"][e], -e))
    rest = [e for e in touched if e != hot]
    whole = [hot] + sorted(rng.choice(rest, min(n_experts - 1, len(rest)), replace=False).tolist())
    cand = [t for t in np.nonzero(keep)[0] if not any(int(e) in bad_e for e in idx[t])]
    tokens, needed = pick_tokens(idx, cand, whole, n_tokens, cfg.E, seed)
    acc = np.zeros((len(tokens), cfg.H))
    pos = {t: i for i, t in enumerate(tokens.tolist())}
    errs = {}
    for e in needed.tolist():
        lo, cnt = int(mp["offsets"][e]), int(mp["counts"][e])
        W = [f64(w) for w in synth.gen_expert_weights(cfg, e, x.device)]
        _, o = O.expert_forward(xq[mp["row_token"][lo:lo + cnt]], *W, dt)
        if e in whole:
            glo = int(g_off[e])
            assert int(g_counts[e]) == cnt, (e, int(g_counts[e]), cnt)
            assert np.array_equal(g_rt[glo:glo + cnt], mp["row_token"][lo:lo + cnt]), e
            errs[e] = rel_frob(f64(out_rows[glo:glo + cnt]), o)
            assert errs[e] < tol, (e, cnt, errs[e])
        for t in np.nonzero((idx[tokens] == e).any(axis=1))[0].tolist():
            tok = int(tokens[t])
            j = int(np.nonzero(idx[tok] == e)[0][0])
            acc[pos[tok]] += r["w"][tok, j] * o[mp["token_row"][tok * cfg.top_k + j] - lo]
    if cfg.I_shared:
        Ws = [f64(w) for w in synth.gen_shared_weights(cfg, x.device)]
        if dt == "nvfp4":   # h's global spans all T rows of the shared expert
            acc += O.expert_forward(xq, *Ws, dt)[1][tokens]
        else:
            acc += O.expert_forward(xq[tokens], *Ws, dt)[1]
    y_err = rel_frob(f64(gpu["y"])[tokens], O.round_bf16(acc))
    assert y_err < tol, y_err
    return {"experts_computed": len(needed), "whole_experts": whole, "hot_rows": int(mp["counts"][hot]),
            "expert_err_max": max(errs.values()), "tokens": len(tokens), "y_err": y_err}
