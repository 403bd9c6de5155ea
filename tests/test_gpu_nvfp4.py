"""NVFP4 W4A4 path against the oracle, through the C ABI: the quantizer
(global scale, packed e2m1 codes and ue4m3 block scales bit-exact), weight
preparation (per-expert global scales), the permute, the block-scaled grouped
MLP (h re-quantized with a per-expert global scale) and the whole layer
(sglang PR "Mistral Large 3 NVFP4 TRTLLM MoE support", Modifications).  The
full-size DeepSeek-V4 NVFP4 layers are in test_gpu_fullsize.py."""

import numpy as np
import pytest
import torch

import synth
from moe_testlib import f64, near_ties, rel_frob, weights_dict
from oracle import moe_oracle as O
from test_gpu_mxfp8 import sf_plain

pytestmark = pytest.mark.gpu

NV = {
    "tiny_nv": synth.MoEShape(name="tiny_nv", T=64, H=256, I=256, E=16, n_group=4, topk_group=2,
                              top_k=4, rsf=2.5, I_shared=256, dtype="nvfp4", pad_multiple=128,
                              router_std=0.02),
    "ragged_nv": synth.MoEShape(name="ragged_nv", T=300, H=512, I=256, E=8, n_group=2,
                                topk_group=1, top_k=2, rsf=1.0, I_shared=0, dtype="nvfp4",
                                pad_multiple=64, router_std=0.05),
    # about 500 rows per expert: every expert spans three 192-token tiles, the
    # last one ragged, as the heavy experts of the 8192-token prefill do
    "hot_nv": synth.MoEShape(name="hot_nv", T=1000, H=512, I=256, E=4, n_group=2, topk_group=2,
                             top_k=2, rsf=2.5, I_shared=256, dtype="nvfp4", pad_multiple=64,
                             router_std=0.02),
}


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available()
    import mixture_experts_layer_grouped_b200 as M
    M.lib()
    return M


def unpack_e2m1(packed, rows, cols):
    """Packed bytes (element 2i in the low nibble) -> one code per element."""
    b = packed.cpu().numpy().reshape(rows, cols // 2)
    out = np.empty((rows, cols), dtype=np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def tile_major_plain(buf, rows, row_bytes):
    t = buf.cpu().numpy().reshape(rows // 128, row_bytes // 128, 128, 128)
    return t.transpose(0, 2, 1, 3).reshape(rows, row_bytes)


def _quant(M, x):
    rows, cols = x.shape
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(M.scale_bytes(rows, cols, "nvfp4"), dtype=torch.uint8, device="cuda")
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    M.moe_quantize("nvfp4", x, codes, scales, global_scale=g)
    return codes, scales, g


def test_quantize_bit_exact(M):
    gen = torch.Generator(device="cuda")
    gen.manual_seed(9)
    x = torch.randn(260, 512, generator=gen, device="cuda") * 2
    x[0] = 0.0
    x[1, :16] = torch.tensor([6.0, 2.5, -0.75, 1.25] * 4)
    x[2] *= 1e-6                    # blocks far below the tensor amax: zero block scales
    x = x.to(torch.bfloat16)
    codes, scales, g = _quant(M, x)
    torch.cuda.synchronize()
    xh = f64(x)
    gref = O.nvfp4_global_scale(np.abs(xh).max())
    assert g.item() == float(gref)
    rc, rs = O.nvfp4_quantize(xh, gref)
    assert np.array_equal(unpack_e2m1(codes, 260, 512), rc)
    assert np.array_equal(sf_plain(scales, 260, 512 // 16), rs)


@pytest.mark.parametrize("name", list(NV))
def test_prepare_weights_nvfp4(M, name):
    cfg = NV[name]
    c = M.config_from_shape(cfg)
    d = synth.gen_all(cfg, "cuda")
    p = M.prepare_weights(c, weights_dict(d))
    torch.cuda.synchronize()
    E, H, I = cfg.E, cfg.H, cfg.I
    w1, w3, w2 = f64(d["w1"]), f64(d["w3"]), f64(d["w2"])
    g13 = p["w13_global"].cpu().numpy()
    g2 = p["w2_global"].cpu().numpy()
    c1 = unpack_e2m1(torch.from_numpy(tile_major_plain(p["w1"], E * I, H // 2)), E * I, H)
    c2 = unpack_e2m1(torch.from_numpy(tile_major_plain(p["w2"], E * H, I // 2)), E * H, I)
    s1 = sf_plain(p["w1_scales"], E * I, H // 16)
    s2 = sf_plain(p["w2_scales"], E * H, I // 16)
    for e in range(E):
        ga = O.nvfp4_global_scale(max(np.abs(w1[e]).max(), np.abs(w3[e]).max()))
        gb = O.nvfp4_global_scale(np.abs(w2[e]).max())
        assert g13[e] == float(ga) and g2[e] == float(gb), e
        rc, rs = O.nvfp4_quantize(w1[e], ga)
        assert np.array_equal(c1[e * I:(e + 1) * I], rc), e
        assert np.array_equal(s1[e * I:(e + 1) * I], rs), e
        rc, rs = O.nvfp4_quantize(w2[e], gb)
        assert np.array_equal(c2[e * H:(e + 1) * H], rc), e
        assert np.array_equal(s2[e * H:(e + 1) * H], rs), e


def _routing(cfg):
    g = torch.Generator(device="cuda")
    g.manual_seed(78)
    logits = torch.randn(cfg.T, cfg.E, generator=g, device="cuda")
    _, bias = synth.gen_router(cfg, "cuda")
    return O.route(f64(logits), f64(bias), cfg.n_group, cfg.topk_group, cfg.top_k, cfg.rsf)


# permute-only shapes for the other gather forms: 7 and 17 code vectors per lane
NV_WIDE = {
    "wide_nv": synth.MoEShape(name="wide_nv", T=96, H=7168, I=256, E=16, n_group=4, topk_group=2,
                              top_k=4, rsf=2.5, I_shared=0, dtype="nvfp4", pad_multiple=64,
                              router_std=0.02),
    "wider_nv": synth.MoEShape(name="wider_nv", T=96, H=16640, I=256, E=16, n_group=4,
                               topk_group=2, top_k=4, rsf=2.5, I_shared=0, dtype="nvfp4",
                               pad_multiple=64, router_std=0.02),
}


@pytest.mark.parametrize("name", list(NV) + list(NV_WIDE))
def test_permute_nvfp4(M, name):
    cfg = NV[name] if name in NV else NV_WIDE[name]
    c = M.config_from_shape(cfg)
    r = _routing(cfg)
    m = O.permute_maps(r["idx"], cfg.E, cfg.pad_multiple)
    xc, xs, _ = _quant(M, synth.gen_x(cfg, "cuda"))
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes)
    i32 = dict(dtype=torch.int32, device="cuda")
    rows = torch.full((r_cap, cfg.H // 2), 7, dtype=torch.uint8, device="cuda")
    rs = torch.full((M.scale_bytes(r_cap, cfg.H, "nvfp4"),), 9, dtype=torch.uint8, device="cuda")
    counts, offsets = torch.empty(cfg.E, **i32), torch.empty(cfg.E + 1, **i32)
    row_token, token_row = torch.empty(r_cap, **i32), torch.empty(cfg.T * cfg.top_k, **i32)
    M.moe_permute(c, torch.from_numpy(r["idx"]).cuda(), xc, counts, offsets, row_token,
                  token_row, rows, ws, src_scales=xs, dst_scales=rs)
    torch.cuda.synchronize()
    n = int(m["offsets"][-1])
    assert np.array_equal(rows[:n].cpu().numpy(), O.gather_rows(xc.cpu().numpy(), m["row_token"]))
    ref_s = O.gather_rows(sf_plain(xs, cfg.T, cfg.H // 16), m["row_token"])
    assert np.array_equal(sf_plain(rs, n, cfg.H // 16), ref_s)


@pytest.mark.parametrize("gather", [False, True], ids=["rows", "gather"])
@pytest.mark.parametrize("name", list(NV))
def test_grouped_mlp_nvfp4(M, name, gather):
    """gather=True: only the scales are permuted and fc1 gathers code rows from x."""
    cfg = NV[name]
    c = M.config_from_shape(cfg)
    d = synth.gen_all(cfg, "cuda")
    h = {k: f64(v) for k, v in d.items()}
    r = _routing(cfg)
    m = O.permute_maps(r["idx"], cfg.E, cfg.pad_multiple)
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes)
    xc, xs, xg = _quant(M, d["x"])
    i32 = dict(dtype=torch.int32, device="cuda")
    rows = torch.zeros(r_cap, cfg.H // 2, dtype=torch.uint8, device="cuda")
    rs = torch.zeros(M.scale_bytes(r_cap, cfg.H, "nvfp4"), dtype=torch.uint8, device="cuda")
    counts, offsets = torch.empty(cfg.E, **i32), torch.empty(cfg.E + 1, **i32)
    row_token, token_row = torch.empty(r_cap, **i32), torch.empty(cfg.T * cfg.top_k, **i32)
    M.moe_permute(c, torch.from_numpy(r["idx"]).cuda(), xc, counts, offsets, row_token,
                  token_row, None if gather else rows, ws, src_scales=xs, dst_scales=rs)
    p = M.prepare_weights(c, weights_dict(d))
    out_rows = torch.zeros(r_cap, cfg.H, dtype=torch.bfloat16, device="cuda")
    shared_out = (torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
                  if cfg.I_shared else None)
    M.moe_grouped_mlp(c, p, None if gather else rows, counts, offsets, out_rows, ws, x=xc,
                      shared_out=shared_out, row_scales=rs, x_scales=xs, x_global=xg,
                      row_token=row_token if gather else None)
    torch.cuda.synchronize()
    assert M.moe_get_device_status(ws) == 0
    gx = O.nvfp4_global_scale(np.abs(h["x"]).max())
    xq = O.quantize_dequantize(h["x"], "nvfp4", gx)
    xr = O.gather_rows(xq, m["row_token"])
    got = f64(out_rows)
    for e in range(cfg.E):
        lo, cnt = int(m["offsets"][e]), int(m["counts"][e])
        if cnt == 0:
            continue
        _, o = O.expert_forward(xr[lo:lo + cnt], h["w1"][e], h["w3"][e], h["w2"][e], "nvfp4")
        assert rel_frob(got[lo:lo + cnt], o) < 2e-2, e
    if cfg.I_shared:
        sh = synth.gen_shared_weights(cfg, "cuda")
        _, so = O.expert_forward(xq, *[f64(t) for t in sh], "nvfp4")
        assert rel_frob(f64(shared_out), so) < 2e-2


@pytest.mark.parametrize("name", list(NV))
def test_forward_nvfp4_end_to_end(M, name):
    cfg = NV[name]
    c = M.config_from_shape(cfg)
    d = synth.gen_all(cfg, "cuda")
    h = {k: f64(v) for k, v in d.items()}
    layer = M.MoELayer(c, weights_dict(d), d["w_router"], d["bias"])
    y = layer.forward(d["x"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    sh = (h["ws1"], h["ws3"], h["ws2"]) if cfg.I_shared else None
    ref = O.forward(cfg, h["x"], h["w_router"], h["bias"], h["w1"], h["w3"], h["w2"], shared=sh)
    keep = ~near_ties(ref["route"])
    assert rel_frob(f64(y)[keep], ref["y"][keep]) < 2e-2
