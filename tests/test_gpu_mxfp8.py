"""MXFP8 path against the oracle, through the C ABI: the quantizer (codes and
scales bit-exact), weight preparation, the code/scale permute, the
block-scaled grouped MLP and the whole layer (TransformerEngine PR
"DeepSeekV3Layer", Performance, MXFP8 rows: e4m3 elements, e8m0 scale per 32)."""

import numpy as np
import pytest
import torch

import synth
from moe_testlib import f64, near_ties, rel_frob, weights_dict
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

MX = {
    "tiny_mx": synth.get_config("tiny_bf16_T64").scaled(name="tiny_mx_T64", dtype="mxfp8",
                                                       pad_multiple=128, I_shared=128),
    "ragged_mx": synth.MoEShape(name="ragged_mx", T=300, H=384, I=256, E=8, n_group=2,
                                topk_group=1, top_k=2, rsf=1.0, I_shared=0, dtype="mxfp8",
                                pad_multiple=64, router_std=0.05),
    "hot_mx": synth.MoEShape(name="hot_mx", T=700, H=256, I=256, E=4, n_group=2, topk_group=2,
                             top_k=2, rsf=2.5, I_shared=128, dtype="mxfp8", pad_multiple=128,
                             router_std=0.02),
}


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available()
    import mixture_experts_layer_grouped_b200 as M
    M.lib()
    return M


def sf_plain(buf, rows, KB):
    """Scale bytes of the documented MMA layout, as a [rows, KB] array."""
    b = buf.cpu().numpy() if hasattr(buf, "cpu") else np.asarray(buf)
    r = np.arange(rows)[:, None]
    kb = np.arange(KB)[None, :]
    off = ((r >> 7) * (KB >> 2) + (kb >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3)
    return b[off]


def tile_major_plain(buf, rows, cols):
    """Row-major view of a tile-major byte buffer (128 rows x 128 bytes per tile)."""
    t = buf.cpu().numpy().reshape(rows // 128, cols // 128, 128, 128)
    return t.transpose(0, 2, 1, 3).reshape(rows, cols)


def _quant(M, x):
    rows, cols = x.shape
    codes = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(M.scale_bytes(rows, cols), dtype=torch.uint8, device="cuda")
    M.moe_quantize("mxfp8", x, codes, scales)
    return codes, scales


def test_quantize_bit_exact(M):
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    x = torch.randn(300, 512, generator=g, device="cuda") * 3
    x[0] = 0.0                      # all-zero blocks
    x[1, :32] = 1e4                 # saturation after scaling? no: amax sets the scale
    x[2, 5] = 500.0                 # one large element, the rest scaled down
    x[3] = torch.randn(512, generator=g, device="cuda") * 1e-30  # tiny values
    x = x.to(torch.bfloat16)
    codes, scales = _quant(M, x)
    torch.cuda.synchronize()
    rc, rs = O.mxfp8_quantize(f64(x))
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(sf_plain(scales, 300, 512 // 32), rs)


@pytest.mark.parametrize("name", ["tiny_mx", "ragged_mx"])
def test_prepare_weights_mxfp8(M, name):
    cfg = MX[name]
    c = M.config_from_shape(cfg)
    d = synth.gen_all(cfg, "cuda")
    if cfg.I_shared:
        d.update(zip(("ws1", "ws3", "ws2"), synth.gen_shared_weights(cfg, "cuda")))
    p = M.prepare_weights(c, weights_dict(d))
    torch.cuda.synchronize()
    E, H, I = cfg.E, cfg.H, cfg.I
    for key, R, K in (("w1", E * I, H), ("w3", E * I, H), ("w2", E * H, I)):
        rc, rs = O.mxfp8_quantize(f64(d[key]).reshape(R, K))
        assert np.array_equal(tile_major_plain(p[key], R, K), rc), key
        assert np.array_equal(sf_plain(p[key + "_scales"], R, K // 32), rs), key
    if cfg.I_shared:
        rc, rs = O.mxfp8_quantize(f64(d["ws2"]))
        assert np.array_equal(tile_major_plain(p["ws2"], H, cfg.I_shared), rc)
        assert np.array_equal(sf_plain(p["ws2_scales"], H, cfg.I_shared // 32), rs)


def _routing(cfg):
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    logits = torch.randn(cfg.T, cfg.E, generator=g, device="cuda")
    _, bias = synth.gen_router(cfg, "cuda")
    return O.route(f64(logits), f64(bias), cfg.n_group, cfg.topk_group, cfg.top_k, cfg.rsf)


# permute-only shapes for the other gather forms: 14 and 17 code vectors per lane
MX_WIDE = {
    "wide_mx": synth.MoEShape(name="wide_mx", T=96, H=7168, I=128, E=16, n_group=4, topk_group=2,
                              top_k=4, rsf=2.5, I_shared=0, dtype="mxfp8", pad_multiple=64,
                              router_std=0.02),
    "wider_mx": synth.MoEShape(name="wider_mx", T=96, H=8448, I=128, E=16, n_group=4,
                               topk_group=2, top_k=4, rsf=2.5, I_shared=0, dtype="mxfp8",
                               pad_multiple=64, router_std=0.02),
}


@pytest.mark.parametrize("name", list(MX) + list(MX_WIDE))
def test_permute_mxfp8(M, name):
    cfg = MX[name] if name in MX else MX_WIDE[name]
    c = M.config_from_shape(cfg)
    r = _routing(cfg)
    m = O.permute_maps(r["idx"], cfg.E, cfg.pad_multiple)
    x = synth.gen_x(cfg, "cuda")
    xc, xs = _quant(M, x)
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes)
    i32 = dict(dtype=torch.int32, device="cuda")
    rows = torch.full((r_cap, cfg.H), 7, dtype=torch.uint8, device="cuda")
    rs = torch.full((M.scale_bytes(r_cap, cfg.H),), 9, dtype=torch.uint8, device="cuda")
    counts, offsets = torch.empty(cfg.E, **i32), torch.empty(cfg.E + 1, **i32)
    row_token, token_row = torch.empty(r_cap, **i32), torch.empty(cfg.T * cfg.top_k, **i32)
    M.moe_permute(c, torch.from_numpy(r["idx"]).cuda(), xc, counts, offsets, row_token,
                  token_row, rows, ws, src_scales=xs, dst_scales=rs)
    torch.cuda.synchronize()
    n = int(m["offsets"][-1])
    assert np.array_equal(offsets.cpu().numpy(), m["offsets"])
    assert np.array_equal(rows[:n].cpu().numpy(), O.gather_rows(xc.cpu().numpy(), m["row_token"]))
    xs_plain = sf_plain(xs, cfg.T, cfg.H // 32)
    ref_s = O.gather_rows(xs_plain, m["row_token"])
    assert np.array_equal(sf_plain(rs, n, cfg.H // 32), ref_s)


def _run_mlp(M, cfg, d, r, gather=False):
    """Quantize x, permute with the oracle's maps, grouped MLP on the GPU.
    gather=True: only the scales are permuted and fc1 gathers code rows from x."""
    c = M.config_from_shape(cfg)
    m = O.permute_maps(r["idx"], cfg.E, cfg.pad_multiple)
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes)
    xc, xs = _quant(M, d["x"])
    i32 = dict(dtype=torch.int32, device="cuda")
    rows = torch.zeros(r_cap, cfg.H, dtype=torch.uint8, device="cuda")
    rs = torch.zeros(M.scale_bytes(r_cap, cfg.H), dtype=torch.uint8, device="cuda")
    counts, offsets = torch.empty(cfg.E, **i32), torch.empty(cfg.E + 1, **i32)
    row_token, token_row = torch.empty(r_cap, **i32), torch.empty(cfg.T * cfg.top_k, **i32)
    M.moe_permute(c, torch.from_numpy(r["idx"]).cuda(), xc, counts, offsets, row_token,
                  token_row, None if gather else rows, ws, src_scales=xs, dst_scales=rs)
    p = M.prepare_weights(c, weights_dict(d))
    out_rows = torch.zeros(r_cap, cfg.H, dtype=torch.bfloat16, device="cuda")
    shared_out = (torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
                  if cfg.I_shared else None)
    M.moe_grouped_mlp(c, p, None if gather else rows, counts, offsets, out_rows, ws, x=xc,
                      shared_out=shared_out, row_scales=rs, x_scales=xs,
                      row_token=row_token if gather else None)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    return m, out_rows, shared_out


@pytest.mark.parametrize("gather", [False, True], ids=["rows", "gather"])
@pytest.mark.parametrize("name", list(MX))
def test_grouped_mlp_mxfp8(M, name, gather):
    cfg = MX[name]
    d = synth.gen_all(cfg, "cuda")
    if cfg.I_shared:
        d.update(zip(("ws1", "ws3", "ws2"), synth.gen_shared_weights(cfg, "cuda")))
    h = {k: f64(v) for k, v in d.items()}
    r = _routing(cfg)
    m, out_rows, shared_out = _run_mlp(M, cfg, d, r, gather)
    xq = O.quantize_dequantize(h["x"], "mxfp8")
    xr = O.gather_rows(xq, m["row_token"])
    got = f64(out_rows)
    for e in range(cfg.E):
        lo, cnt = int(m["offsets"][e]), int(m["counts"][e])
        if cnt == 0:
            continue
        _, o = O.expert_forward(xr[lo:lo + cnt], h["w1"][e], h["w3"][e], h["w2"][e], "mxfp8")
        assert rel_frob(got[lo:lo + cnt], o) < 2e-2, e
    if cfg.I_shared:
        _, so = O.expert_forward(xq, h["ws1"], h["ws3"], h["ws2"], "mxfp8")
        assert rel_frob(f64(shared_out), so) < 2e-2


@pytest.mark.parametrize("name", list(MX))
def test_gathered_rows_give_the_same_bits_mxfp8(M, name):
    """fc1 reading its rows from x through row_token computes exactly what it
    computes on the permuted copy (same data, same MMA order)."""
    cfg = MX[name]
    d = synth.gen_all(cfg, "cuda")
    if cfg.I_shared:
        d.update(zip(("ws1", "ws3", "ws2"), synth.gen_shared_weights(cfg, "cuda")))
    r = _routing(cfg)
    _, a, _ = _run_mlp(M, cfg, d, r, False)
    _, b, _ = _run_mlp(M, cfg, d, r, True)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name", list(MX))
def test_forward_mxfp8_end_to_end(M, name):
    cfg = MX[name]
    c = M.config_from_shape(cfg)
    d = synth.gen_all(cfg, "cuda")
    if cfg.I_shared:
        d.update(zip(("ws1", "ws3", "ws2"), synth.gen_shared_weights(cfg, "cuda")))
    h = {k: f64(v) for k, v in d.items()}
    layer = M.MoELayer(c, weights_dict(d), d["w_router"], d["bias"])
    y = layer.forward(d["x"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    sh = (h["ws1"], h["ws3"], h["ws2"]) if cfg.I_shared else None
    ref = O.forward(cfg, h["x"], h["w_router"], h["bias"], h["w1"], h["w3"], h["w2"], shared=sh)
    keep = ~near_ties(ref["route"])
    assert rel_frob(f64(y)[keep], ref["y"][keep]) < 2e-2
