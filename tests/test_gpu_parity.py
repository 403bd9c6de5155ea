"""Parity of the CUDA library with the CPU oracle, through the C ABI.

Each step call is checked on identical inputs (routing from identical logits,
permute from identical indices, combine from identical rows), then the grouped
MLP and the whole layer end to end, on the six workloads and on edge shapes
(one token, ragged tails, experts with more than one 256-token chunk, empty
experts, pad multiples 1 / 8 / 128).
"""

import numpy as np
import pytest
import torch

import synth
from moe_testlib import (check_routing, f64, gen_device_inputs, host_inputs, near_ties,
                         rel_frob, run_steps, weights_dict)
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

BF16_CONFIGS = ["tiny_bf16_T64", "mid_bf16_shared_T2048"]
ALL_CONFIGS = list(synth.CONFIGS)

EDGE = {
    "one_token": synth.MoEShape(name="edge_one_token", T=1, H=256, I=128, E=16, n_group=4,
                                topk_group=2, top_k=4, rsf=2.5, I_shared=128, dtype="bf16",
                                pad_multiple=8, router_std=0.02),
    "ragged_pad1": synth.MoEShape(name="edge_ragged_pad1", T=300, H=384, I=256, E=8,
                                  n_group=2, topk_group=1, top_k=2, rsf=1.0, I_shared=128,
                                  dtype="bf16", pad_multiple=1, router_std=0.05),
    "hot_chunks": synth.MoEShape(name="edge_hot_chunks", T=1000, H=256, I=384, E=4, n_group=2,
                                 topk_group=2, top_k=2, rsf=2.5, I_shared=0, dtype="bf16",
                                 pad_multiple=128, router_std=0.02),
    "empty_experts": synth.MoEShape(name="edge_empty_experts", T=40, H=128, I=128, E=64,
                                    n_group=8, topk_group=1, top_k=3, rsf=2.5, I_shared=0,
                                    dtype="bf16", pad_multiple=16, router_std=0.02),
}


# permute-only shapes whose rows take the other gather forms: 28 and 33
# 16-byte vectors per lane (the 32-vector one-round kernel and the looping one)
WIDE = {
    "rows_h7168": synth.MoEShape(name="edge_rows_h7168", T=96, H=7168, I=128, E=16, n_group=4,
                                 topk_group=2, top_k=4, rsf=2.5, I_shared=0, dtype="bf16",
                                 pad_multiple=8, router_std=0.02),
    "rows_h8448": synth.MoEShape(name="edge_rows_h8448", T=96, H=8448, I=128, E=16, n_group=4,
                                 topk_group=2, top_k=4, rsf=2.5, I_shared=0, dtype="bf16",
                                 pad_multiple=8, router_std=0.02),
}


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import mixture_experts_layer_grouped_b200 as M
    M.lib()  # fails loudly when the library is missing
    return M


def _cfg(name):
    if name in WIDE:
        return WIDE[name]
    return EDGE[name] if name in EDGE else synth.get_config(name)


def _logits(cfg, scale=1.0):
    g = torch.Generator(device="cuda")
    g.manual_seed(1234 + cfg.E)
    return torch.randn(cfg.T, cfg.E, generator=g, device="cuda") * scale


# ---------------------------------------------------------------- routing
@pytest.mark.parametrize("name", ALL_CONFIGS + list(EDGE))
def test_route_selection_from_identical_logits(M, name):
    cfg = _cfg(name)
    c = M.config_from_shape(cfg)
    _, bias = synth.gen_router(cfg, "cuda")
    logits = _logits(cfg)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device="cuda")
    ws = M.binding.new_workspace(M.moe_workspace_size(c)[0])
    M.moe_route(c, None, None, bias, idx, w, ws, logits_in=logits)
    torch.cuda.synchronize()
    r = O.route(f64(logits), f64(bias), cfg.n_group, cfg.topk_group, cfg.top_k, cfg.rsf)
    keep, bad = check_routing(r, idx.cpu().numpy(), w.cpu().numpy(), cfg.rsf)
    assert not bad, f"{len(bad)} tokens differ, first {bad[:5]}"
    assert keep.mean() > 0.95


@pytest.mark.parametrize("name", ALL_CONFIGS)
def test_router_gemm(M, name):
    """Every workload at its full T (the 8192-token prefill splits K three ways)."""
    cfg = _cfg(name)
    c = M.config_from_shape(cfg)
    x = synth.gen_x(cfg, "cuda")
    w_r, bias = synth.gen_router(cfg, "cuda")
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device="cuda")
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device="cuda")
    ws = M.binding.new_workspace(M.moe_workspace_size(c)[0])
    M.moe_route(c, x, w_r, bias, idx, w, ws, logits_out=logits)
    torch.cuda.synchronize()
    ref = O.router_logits(f64(x), f64(w_r))
    got = f64(logits)
    assert rel_frob(got, ref) < 1e-5
    assert np.max(np.abs(got - ref)) < 1e-4 * max(1.0, np.abs(ref).max())
    # and selection on the GPU's own logits matches the oracle on those logits
    r = O.route(got, f64(bias), cfg.n_group, cfg.topk_group, cfg.top_k, cfg.rsf)
    _, bad = check_routing(r, idx.cpu().numpy(), w.cpu().numpy(), cfg.rsf)
    assert not bad


# ---------------------------------------------------------------- permute
@pytest.mark.parametrize("name", ["tiny_bf16_T64", "mid_bf16_shared_T2048", "dsv4_bf16_T4096"]
                         + list(EDGE) + list(WIDE))
def test_permute_bit_exact(M, name):
    """Counts, offsets, slots and every gather form against the oracle's maps
    and rows."""
    cfg = _cfg(name)
    c = M.config_from_shape(cfg)
    _, bias = synth.gen_router(cfg, "cuda")
    r = O.route(f64(_logits(cfg)), f64(bias), cfg.n_group, cfg.topk_group, cfg.top_k, cfg.rsf)
    m = O.permute_maps(r["idx"], cfg.E, cfg.pad_multiple)
    x = synth.gen_x(cfg, "cuda")
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes)
    i32 = dict(dtype=torch.int32, device="cuda")
    idx = torch.from_numpy(r["idx"]).to("cuda")
    counts, offsets = torch.empty(cfg.E, **i32), torch.empty(cfg.E + 1, **i32)
    row_token, token_row = torch.empty(r_cap, **i32), torch.empty(cfg.T * cfg.top_k, **i32)
    rows = torch.full((r_cap, cfg.H), 7.0, dtype=torch.bfloat16, device="cuda")
    M.moe_permute(c, idx, x, counts, offsets, row_token, token_row, rows, ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    n = int(m["offsets"][-1])
    assert np.array_equal(counts.cpu().numpy(), m["counts"])
    assert np.array_equal(offsets.cpu().numpy(), m["offsets"])
    rt = row_token.cpu().numpy()
    assert np.array_equal(rt[:n], m["row_token"]) and np.all(rt[n:] == -1)
    assert np.array_equal(token_row.cpu().numpy(), m["token_row"])
    xb = x.cpu().view(torch.int16).numpy()
    ref_rows = O.gather_rows(xb, m["row_token"])
    assert np.array_equal(rows[:n].cpu().view(torch.int16).numpy(), ref_rows)


# ---------------------------------------------------------------- combine
@pytest.mark.parametrize("name", ["tiny_bf16_T64", "mid_bf16_shared_T2048", "one_token"])
def test_combine(M, name):
    cfg = _cfg(name)
    c = M.config_from_shape(cfg)
    _, bias = synth.gen_router(cfg, "cuda")
    r = O.route(f64(_logits(cfg)), f64(bias), cfg.n_group, cfg.topk_group, cfg.top_k, cfg.rsf)
    m = O.permute_maps(r["idx"], cfg.E, cfg.pad_multiple)
    _, r_cap = M.moe_workspace_size(c)
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    out_rows = torch.randn(r_cap, cfg.H, generator=g, device="cuda").to(torch.bfloat16)
    shared = torch.randn(cfg.T, cfg.H, generator=g, device="cuda").to(torch.bfloat16)
    tr = torch.from_numpy(m["token_row"].astype(np.int32)).to("cuda")
    w = torch.from_numpy(r["w"].astype(np.float32)).to("cuda")
    y = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    M.moe_combine(c, out_rows, tr, w, y, shared_out=shared)
    torch.cuda.synchronize()
    ref = O.combine(f64(out_rows), m["token_row"], f64(w), f64(shared))
    got = f64(y)
    # fp32 vs fp64 accumulation: at most one bf16 rounding step apart
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-6)


# ---------------------------------------------------------------- grouped MLP
@pytest.mark.parametrize("gather", [False, True], ids=["rows", "gather"])
@pytest.mark.parametrize("name", BF16_CONFIGS + list(EDGE))
def test_grouped_mlp(M, name, gather):
    """gather=True: fc1 reads token rows from x through row_token (rows=None)."""
    cfg = _cfg(name)
    c = M.config_from_shape(cfg)
    d = gen_device_inputs(cfg)
    h = host_inputs(d)
    r = O.route(f64(_logits(cfg)), h["bias"], cfg.n_group, cfg.topk_group, cfg.top_k, cfg.rsf)
    m = O.permute_maps(r["idx"], cfg.E, cfg.pad_multiple)
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes)
    n = int(m["offsets"][-1])
    rows_np = np.zeros((r_cap,) + d["x"].shape[1:], dtype=np.int16)
    rows_np[:n] = O.gather_rows(d["x"].cpu().view(torch.int16).numpy(), m["row_token"])
    rows = torch.from_numpy(rows_np).to("cuda").view(torch.bfloat16)
    counts = torch.from_numpy(m["counts"].astype(np.int32)).to("cuda")
    offsets = torch.from_numpy(m["offsets"].astype(np.int32)).to("cuda")
    out_rows = torch.zeros(r_cap, cfg.H, dtype=torch.bfloat16, device="cuda")
    shared_out = (torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
                  if cfg.I_shared else None)
    rt = np.full(r_cap, -1, dtype=np.int32)
    rt[:n] = m["row_token"]
    row_token = torch.from_numpy(rt).to("cuda")
    M.moe_grouped_mlp(c, M.prepare_weights(c, weights_dict(d)), None if gather else rows, counts,
                      offsets, out_rows, ws, x=d["x"], shared_out=shared_out,
                      row_token=row_token if gather else None)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    got = f64(out_rows)
    xr = O.gather_rows(h["x"], m["row_token"])
    for e in range(cfg.E):
        lo, cnt = int(m["offsets"][e]), int(m["counts"][e])
        if cnt == 0:
            continue
        _, o = O.expert_forward(xr[lo:lo + cnt], h["w1"][e], h["w3"][e], h["w2"][e], "bf16")
        err = rel_frob(got[lo:lo + cnt], o)
        assert err < 1e-2, (e, err)
    if cfg.I_shared:
        _, so = O.expert_forward(h["x"], h["ws1"], h["ws3"], h["ws2"], "bf16")
        assert rel_frob(f64(shared_out), so) < 1e-2


# ---------------------------------------------------------------- end to end
@pytest.mark.parametrize("name", BF16_CONFIGS + list(EDGE))
def test_forward_end_to_end(M, name):
    cfg = _cfg(name)
    d = gen_device_inputs(cfg)
    h = host_inputs(d)
    out = run_steps(cfg, d)
    assert out["status"] == 0
    sh = (h["ws1"], h["ws3"], h["ws2"]) if cfg.I_shared else None
    ref = O.forward(cfg, h["x"], h["w_router"], h["bias"], h["w1"], h["w3"], h["w2"], shared=sh)
    keep = ~near_ties(ref["route"])
    assert keep.mean() > 0.95
    y = f64(out["y"])
    err = rel_frob(y[keep], ref["y"][keep])
    assert err < 1e-2, err
    # the one-call forward (device buffers, then host buffers) gives the same bits
    c = __import__("mixture_experts_layer_grouped_b200").config_from_shape(cfg)
    import mixture_experts_layer_grouped_b200 as MM
    layer = MM.MoELayer(c, weights_dict(d), d["w_router"], d["bias"])
    y_dev = layer.forward(d["x"])
    x_host = d["x"].cpu().pin_memory()
    y_host = layer.forward(x_host)
    torch.cuda.synchronize()
    assert torch.equal(y_dev.cpu().view(torch.int16), out["y"].cpu().view(torch.int16))
    assert torch.equal(y_host.view(torch.int16), out["y"].cpu().view(torch.int16))
    assert layer.device_status() == 0


@pytest.mark.parametrize("name", ["mid_bf16_shared_T2048", "hot_chunks", "tiny_mx",
                                  "ragged_mx", "tiny_nv", "hot_nv"])
def test_schedules_give_same_bits(M, name, tmp_path):
    """The default schedule (tiles claimed from a counter, fc2 started chunk by
    chunk as fc1 finishes them) gives the same bits as the static one (CTA i
    takes tiles i, i + grid, ...; fc2 waits for fc1 as a whole): only the
    order of tiles differs, never the arithmetic of one."""
    import os
    import subprocess
    import sys
    helper = os.path.join(os.path.dirname(os.path.abspath(__file__)), "forward_once.py")
    outs = []
    for early in ("1", "0"):
        path = str(tmp_path / f"y_{early}.pt")
        env = dict(os.environ, MOE_FC2_EARLY=early, MOE_DYNAMIC_TILES=early)
        r = subprocess.run([sys.executable, helper, name, path], env=env, capture_output=True,
                           text=True, timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        outs.append(torch.load(path))
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


@pytest.mark.parametrize("name", ["tiny_bf16_T64", "mid_bf16_shared_T2048"])
def test_bounded_wait_times_out_and_recovers(M, name):
    """A wait that nothing satisfies (fc2's chunk counts raised past what fc1
    produces, for one call) ends in order: the status word reads
    MOE_ERR_TIMEOUT, the context stays usable, and the next call gives the
    same bits as before.  One-CTA tiles (tiny) and CTA pairs (mid)."""
    import os
    import subprocess
    import sys
    helper = os.path.join(os.path.dirname(os.path.abspath(__file__)), "timeout_once.py")
    r = subprocess.run([sys.executable, helper, name], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [l for l in r.stdout.splitlines() if l.startswith("status")][-1].split()
    s0, s1, s2, same = int(line[1]), int(line[2]), int(line[3]), int(line[5])
    assert (s0, s1, s2, same) == (0, 5, 0, 1), line  # 5 = MOE_ERR_TIMEOUT


def test_device_status_reports_bad_index(M):
    cfg = EDGE["empty_experts"]
    c = M.config_from_shape(cfg)
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes)
    i32 = dict(dtype=torch.int32, device="cuda")
    idx = torch.zeros(cfg.T, cfg.top_k, **i32)
    idx[:, 1], idx[:, 2] = 1, 2
    idx[5, 1] = cfg.E + 3  # out of range
    x = synth.gen_x(cfg, "cuda")
    M.moe_permute(c, idx, x, torch.empty(cfg.E, **i32), torch.empty(cfg.E + 1, **i32),
                  torch.empty(r_cap, **i32), torch.empty(cfg.T * cfg.top_k, **i32),
                  torch.empty(r_cap, cfg.H, dtype=torch.bfloat16, device="cuda"), ws)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 4
    assert M.moe_get_device_status(ws) == 0  # cleared by the read


# ---------------------------------------------------------------- weight preparation
def _tile_major(w, R, K):
    """The documented tile-major layout of a row-major [R, K] matrix."""
    return (w.reshape(R // 128, 128, K // 64, 64).permute(0, 2, 1, 3).reshape(-1))


@pytest.mark.parametrize("name", ["tiny_bf16_T64", "one_token", "ragged_pad1"])
def test_prepare_weights_layout(M, name):
    cfg = _cfg(name)
    c = M.config_from_shape(cfg)
    d = gen_device_inputs(cfg)
    if cfg.I_shared:
        d.update(zip(("ws1", "ws3", "ws2"), synth.gen_shared_weights(cfg, "cuda")))
    p = M.prepare_weights(c, weights_dict(d))
    torch.cuda.synchronize()
    E, H, I = cfg.E, cfg.H, cfg.I
    bf = lambda t: t.view(torch.bfloat16)  # prepared buffers are raw bytes
    assert torch.equal(bf(p["w1"]), _tile_major(d["w1"].reshape(E * I, H), E * I, H))
    assert torch.equal(bf(p["w3"]), _tile_major(d["w3"].reshape(E * I, H), E * I, H))
    assert torch.equal(bf(p["w2"]), _tile_major(d["w2"].reshape(E * H, I), E * H, I))
    if cfg.I_shared:
        Is = cfg.I_shared
        assert torch.equal(bf(p["ws1"]), _tile_major(d["ws1"], Is, H))
        assert torch.equal(bf(p["ws2"]), _tile_major(d["ws2"], H, Is))
    # preparing one expert range at a time gives the same buffers
    q = {k: torch.zeros_like(v) for k, v in p.items()}
    dst = M.binding.weights_struct(q)
    for e0 in range(0, E, 3):
        n = min(3, E - e0)
        M.moe_prepare_weights(c, 0, e0, n, d["w1"][e0:e0 + n].contiguous(),
                              d["w3"][e0:e0 + n].contiguous(), d["w2"][e0:e0 + n].contiguous(),
                              dst)
    torch.cuda.synchronize()
    for k in ("w1", "w3", "w2"):
        assert torch.equal(q[k], p[k])
