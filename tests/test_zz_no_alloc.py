"""moe_permute_noalloc: the permute for callers that cannot allocate.

Some callers of this library cannot allocate device memory: a plugin inside an
inference engine that owns every device allocation and hands the plugin only
its input and output buffers, or code that must not call cudaMalloc because it
can synchronize the whole device.  moe_permute_noalloc serves them: its
histogram scratch is a fixed array compiled into the library instead of a
caller-provided workspace.  These tests check, through the C ABI, that it
returns exactly what moe_permute returns and what the oracle's maps and
gather give (the permute's outputs are integer maps and copied rows, so the
tolerance is bit-exact), on two calls in a row with different routings so
that stale scratch contents from the first call would show in the second, and
that what it does not serve (shapes too large for the built-in scratch, block
scales, block-scaled types) is refused before anything is launched.

This file is collected last so that a run stopping at its first failure has
already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

import synth
from oracle import moe_oracle as O


def _outputs(cfg, r_cap):
    i32 = dict(dtype=torch.int32, device="cuda")
    return dict(counts=torch.full((cfg.E,), -7, **i32),
                offsets=torch.full((cfg.E + 1,), -7, **i32),
                row_token=torch.full((r_cap,), -7, **i32),
                token_row=torch.full((cfg.T * cfg.top_k,), -7, **i32),
                rows=torch.full((r_cap, cfg.H), 3.0, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["mid_bf16_shared_T2048", "dsv4_bf16_T4096"])
def test_permute_noalloc_matches_permute_on_two_calls(name):
    import mixture_experts_layer_grouped_b200 as M
    cfg = synth.get_config(name)
    c = M.config_from_shape(cfg)
    nbytes, r_cap = M.moe_workspace_size(c)
    ws = M.binding.new_workspace(nbytes)
    x = synth.gen_x(cfg, "cuda")
    for call in range(2):
        g = torch.Generator(device="cuda")
        g.manual_seed(100 + call)
        # a different routing on each call: k distinct experts per token
        scores = torch.rand(cfg.T, cfg.E, generator=g, device="cuda")
        idx = scores.topk(cfg.top_k, dim=1).indices.to(torch.int32).contiguous()
        ref = _outputs(cfg, r_cap)
        M.moe_permute(c, idx, x, ref["counts"], ref["offsets"], ref["row_token"],
                      ref["token_row"], ref["rows"], ws)
        got = _outputs(cfg, r_cap)
        M.moe_permute_noalloc(c, idx, x, got["counts"], got["offsets"], got["row_token"],
                              got["token_row"], got["rows"])
        torch.cuda.synchronize()
        n = int(ref["offsets"][-1].item())
        for k in ("counts", "offsets", "row_token", "token_row"):
            assert torch.equal(got[k], ref[k]), (call, k)
        assert torch.equal(got["rows"][:n].view(torch.int16), ref["rows"][:n].view(torch.int16))
        assert M.moe_get_device_status(ws) == 0
        # and both are the oracle's maps and rows
        m = O.permute_maps(idx.cpu().numpy(), cfg.E, cfg.pad_multiple)
        assert np.array_equal(got["counts"].cpu().numpy(), m["counts"])
        assert np.array_equal(got["offsets"].cpu().numpy(), m["offsets"])
        rt = got["row_token"].cpu().numpy()
        assert np.array_equal(rt[:n], m["row_token"]) and np.all(rt[n:] == -1)
        assert np.array_equal(got["token_row"].cpu().numpy(), m["token_row"])
        ref_rows = O.gather_rows(x.cpu().view(torch.int16).numpy(), m["row_token"])
        assert np.array_equal(got["rows"][:n].cpu().view(torch.int16).numpy(), ref_rows)


def test_permute_noalloc_refuses_shapes_beyond_its_scratch():
    import mixture_experts_layer_grouped_b200 as M
    s = synth.MoEShape(name="too_big", T=65536, H=256, I=128, E=1024, n_group=8, topk_group=1,
                       top_k=8, rsf=1.0, I_shared=0, dtype="bf16", pad_multiple=8,
                       router_std=0.02)
    c = M.config_from_shape(s)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the size check fails first
    code = M.lib().moe_permute_noalloc(ctypes.byref(c), fake, fake, None, fake, fake, fake, fake,
                                       fake, None, None)
    assert code == 3  # MOE_ERR_WORKSPACE


def test_permute_noalloc_refuses_scales_and_block_scaled_types():
    import mixture_experts_layer_grouped_b200 as M
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the argument checks fail first
    s = synth.get_config("tiny_bf16_T64")
    c = M.config_from_shape(s)
    args = [fake] * 7
    # src_scales or dst_scales given: bf16 rows carry no scales
    assert M.lib().moe_permute_noalloc(ctypes.byref(c), fake, fake, fake, *args[:4], fake, None,
                                       None) == 1
    assert M.lib().moe_permute_noalloc(ctypes.byref(c), fake, fake, None, *args[:4], fake, fake,
                                       None) == 1
    # dst_rows is required
    assert M.lib().moe_permute_noalloc(ctypes.byref(c), fake, fake, None, *args[:4], None, None,
                                       None) == 1
    for dt in ("mxfp8", "nvfp4"):
        cq = M.config_from_shape(s.scaled(dtype=dt, pad_multiple=64, H=256, I=256))
        assert M.lib().moe_permute_noalloc(ctypes.byref(cq), fake, fake, fake, *args[:4], fake,
                                           fake, None) == 2  # MOE_ERR_UNSUPPORTED
