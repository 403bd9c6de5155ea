"""The C ABI on the host: the library loads, exports every function the header
declares, and rejects bad arguments before launching anything (no GPU needed:
every case below fails validation before the first CUDA call)."""

import ctypes
import os
import re
import subprocess

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def M():
    import mixture_experts_layer_grouped_b200 as M
    from mixture_experts_layer_grouped_b200 import build
    build.build()
    return M


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_five_steps():
    names = declared_functions()
    for f in ("moe_route", "moe_permute", "moe_grouped_mlp", "moe_combine", "moe_forward",
              "moe_workspace_size", "moe_status_string", "moe_get_device_status"):
        assert f in names


def test_library_exports_every_declared_function(M):
    lib = M.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", M.binding.LIB_PATH],
                         capture_output=True, text=True, check=True).stdout
    exported = set(l.split()[-1] for l in out.splitlines() if l.strip())
    assert set(declared_functions()) <= exported


def test_status_strings(M):
    lib = M.lib()
    for code in range(7):
        assert lib.moe_status_string(code)
    assert lib.moe_status_string(99) == b"unknown status"


def _cfg(M, **kw):
    s = synth.get_config("tiny_bf16_T64").scaled(**kw)
    return M.config_from_shape(s)


@pytest.mark.parametrize("kw,code", [
    (dict(T=0), 1), (dict(E=15), 2), (dict(H=200), 2), (dict(I=96), 2),
    (dict(n_group=5), 2), (dict(top_k=40), 2), (dict(topk_group=5), 2),
    (dict(pad_multiple=0), 1), (dict(I_shared=100), 2),
])
def test_workspace_size_rejects_bad_shapes(M, kw, code):
    c = _cfg(M, **kw)
    b, r = ctypes.c_size_t(), ctypes.c_int32()
    assert M.lib().moe_workspace_size(ctypes.byref(c), ctypes.byref(b), ctypes.byref(r)) == code


def test_workspace_size_and_rcap(M):
    s = synth.get_config("mid_bf16_shared_T2048")
    nbytes, r_cap = M.moe_workspace_size(M.config_from_shape(s))
    assert r_cap == s.r_cap == 2048 * 6 + 64 * 7
    assert nbytes >= r_cap * s.I * 2 + s.T * s.I_shared * 2
    assert M.moe_forward_workspace_size(M.config_from_shape(s)) > nbytes


def test_calls_reject_null_and_small_workspace(M):
    lib = M.lib()
    c = _cfg(M)
    nb, _ = M.moe_workspace_size(c)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    # null topk outputs
    assert lib.moe_route(ctypes.byref(c), fake, fake, fake, None, fake, None, None, fake, nb,
                         None) == 1
    # workspace too small
    assert lib.moe_route(ctypes.byref(c), fake, fake, fake, None, fake, fake, fake, fake, 16,
                         None) == 3
    # misaligned workspace
    assert lib.moe_permute(ctypes.byref(c), fake, fake, None, fake, fake, fake, fake, fake, None,
                           ctypes.c_void_p((1 << 20) + 8), nb, None) == 1
    w = M.MoEWeights()
    assert lib.moe_grouped_mlp(ctypes.byref(c), ctypes.byref(w), fake, None, fake, None, None,
                               fake, fake, None, fake, None, fake, nb, None) == 1
    # gathered rows (rows == NULL) need row_token
    wf = M.MoEWeights(w1=fake, w3=fake, w2=fake)
    assert lib.moe_grouped_mlp(ctypes.byref(c), ctypes.byref(wf), None, None, fake, None, None,
                               fake, fake, None, fake, None, fake, nb, None) == 1
    assert lib.moe_combine(ctypes.byref(c), None, fake, fake, None, fake, None) == 1
    assert lib.moe_forward(ctypes.byref(c), ctypes.byref(w), fake, fake, fake, fake, 0, fake, 16,
                           None) == 3


@pytest.mark.parametrize("name", sorted(synth.CONFIGS))
def test_every_workload_passes_validation(M, name):
    """Each workload the bench and the tests use is a shape the library accepts,
    with a workspace and prepared weights of the expected sizes."""
    s = synth.get_config(name)
    c = M.config_from_shape(s)
    nbytes, r_cap = M.moe_workspace_size(c)
    assert r_cap == s.r_cap and nbytes > 0
    assert M.moe_forward_workspace_size(c) > nbytes
    sizes = M.moe_prepared_weights_size(c)
    per = {"bf16": 2.0, "mxfp8": 1.0, "nvfp4": 0.5}[s.dtype]
    assert sizes["w13"] == int(s.E * s.I * s.H * per)
    assert sizes["w2"] == int(s.E * s.H * s.I * per)


def test_block_scaled_needs_64_row_padding(M):
    s = synth.get_config("dsv3_mxfp8_shared_T4096").scaled(pad_multiple=32)
    c = M.config_from_shape(s)
    sizes = M.binding.MoEWeightSizes()
    assert M.lib().moe_prepared_weights_size(ctypes.byref(c), ctypes.byref(sizes)) == 2
    s = s.scaled(pad_multiple=64)
    assert M.lib().moe_prepared_weights_size(ctypes.byref(M.config_from_shape(s)),
                                             ctypes.byref(sizes)) == 0


def test_backward_rejects_bad_arguments(M):
    """moe_backward validates on the host: bf16 only, the saved forward state
    and weight copies required, routed weight gradients only with 64-row
    segment pads, and a workspace of moe_backward_workspace_size bytes."""
    lib = M.lib()
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    s = synth.get_config("tiny_bf16_T64").scaled(pad_multiple=64)
    c = M.config_from_shape(s)
    nb = M.moe_backward_workspace_size(c)
    w = M.MoEWeights(w1=fake, w3=fake, w2=fake)
    bw = M.MoEBwdWeights(w2t=fake, w13t=fake, wdt=fake)
    sv = M.MoEFwdSaved(**{k: fake for k, _ in M.MoEFwdSaved._fields_})
    gr = M.MoEWeightGrads(dw1=fake)

    def call(cfg=c, bw=bw, sv=sv, gr=gr, ws=nb, dy=fake):
        return lib.moe_backward(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(bw),
                                ctypes.byref(sv), dy, fake, None, None,
                                ctypes.byref(gr) if gr is not None else None, fake, ws, None)

    assert call(ws=16) == 3
    assert call(dy=None) == 1
    assert call(bw=M.MoEBwdWeights(w2t=fake, w13t=fake)) == 1
    sv_missing = M.MoEFwdSaved(**{k: fake for k, _ in M.MoEFwdSaved._fields_ if k != "logits"})
    assert call(sv=sv_missing) == 1
    # shared-expert gradients of a layer without one
    assert call(gr=M.MoEWeightGrads(dws1=fake)) == 1
    # routed weight gradients need segment pads of a multiple of 64 rows
    c8 = M.config_from_shape(s.scaled(pad_multiple=8))
    nb8 = M.moe_backward_workspace_size(c8)
    assert call(cfg=c8, ws=nb8) == 2
    # block-scaled layers have no backward
    cq = M.config_from_shape(synth.get_config("dsv3_mxfp8_shared_T4096"))
    assert call(cfg=cq) == 2
    n = ctypes.c_size_t()
    assert lib.moe_backward_workspace_size(ctypes.byref(cq), ctypes.byref(n)) == 2


def test_backward_weight_sizes(M):
    s = synth.get_config("mid_bf16_shared_T2048")
    sz = M.moe_backward_weights_size(M.config_from_shape(s))
    assert sz["w2t"] == s.E * s.I * s.H * 2
    assert sz["w13t"] == s.E * s.H * 2 * s.I * 2
    assert sz["ws2t"] == s.I_shared * s.H * 2
    assert sz["wdt"] == s.H * (2 * s.I_shared + 64) * 2  # E = 64 columns of W_r^T


def test_binding_rejects_host_tensors_for_the_backward(M):
    """The binding's marshalling checks device, dtype and layout before any C
    call: host tensors are refused with a ValueError."""
    import torch
    s = synth.get_config("tiny_bf16_T64").scaled(pad_multiple=64)
    c = M.config_from_shape(s)
    x = torch.zeros(s.T, s.H, dtype=torch.bfloat16)
    saved = {k: x for k in ("x", "rows", "out_rows")}
    saved.update({k: torch.zeros(4, dtype=torch.int32) for k in
                  ("topk_idx", "counts", "offsets", "row_token", "token_row")})
    saved.update(logits=torch.zeros(4), topk_w=torch.zeros(4))
    with pytest.raises(ValueError):
        M.moe_backward(c, M.MoEWeights(), M.MoEBwdWeights(), saved, x, x,
                       torch.zeros(16, dtype=torch.uint8))
