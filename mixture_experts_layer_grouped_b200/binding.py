"""ctypes binding of libmoe_b200.so (argument marshalling only).

Each ``moe_*`` function takes torch tensors, checks device/dtype/contiguity,
and passes raw pointers, sizes and the current CUDA stream to the C function of
the same name.  Nothing here computes any part of the layer.
"""

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

DTYPES = {"bf16": 0, "mxfp8": 1, "nvfp4": 2}

STATUS = {
    0: "ok", 1: "invalid argument", 2: "unsupported shape or dtype",
    3: "workspace too small", 4: "expert index out of range (device)",
    5: "bounded wait timed out (device)", 6: "CUDA error",
}


class MoEError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({code})")


class MoEConfig(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
        ("E", ctypes.c_int32), ("n_group", ctypes.c_int32),
        ("topk_group", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("I_shared", ctypes.c_int32), ("routed_scaling_factor", ctypes.c_float),
        ("dtype", ctypes.c_int32), ("pad_multiple", ctypes.c_int32),
    ]


_WEIGHT_FIELDS = [
    "w1", "w3", "w2", "w1_scales", "w3_scales", "w2_scales", "w13_global", "w2_global",
    "ws1", "ws3", "ws2", "ws1_scales", "ws3_scales", "ws2_scales", "ws13_global", "ws2_global",
]


class MoEWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _WEIGHT_FIELDS]


class MoEWeightSizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("w13", "w2", "ws13", "ws2", "w13_scales", "w2_scales", "ws13_scales",
                 "ws2_scales", "w_globals", "ws_globals")]


class MoEBwdWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w2t", "w13t", "ws2t", "wdt")]


class MoEBwdWeightSizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("w2t", "w13t", "ws2t", "wdt")]


_SAVED_FIELDS = ("x", "rows", "logits", "topk_idx", "topk_w", "counts", "offsets",
                 "row_token", "token_row", "out_rows")


class MoEFwdSaved(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _SAVED_FIELDS]


_GRAD_FIELDS = ("dw1", "dw3", "dw2", "dws1", "dws3", "dws2", "dw_router")


class MoEWeightGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _GRAD_FIELDS] + [("accumulate", ctypes.c_int32)]


def config_from_shape(s, T=None) -> MoEConfig:
    """MoEConfig from any object with the layer's shape attributes."""
    return MoEConfig(
        T=s.T if T is None else T, H=s.H, I=s.I, E=s.E, n_group=s.n_group,
        topk_group=s.topk_group, top_k=s.top_k, I_shared=s.I_shared,
        routed_scaling_factor=s.rsf, dtype=DTYPES[s.dtype], pad_multiple=s.pad_multiple)


_lib = None
_VP = ctypes.c_void_p
_CFG = ctypes.POINTER(MoEConfig)


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m mixture_experts_layer_grouped_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "moe_workspace_size": ([_CFG, ctypes.POINTER(ctypes.c_size_t),
                                    ctypes.POINTER(ctypes.c_int32)], ctypes.c_int),
            "moe_forward_workspace_size": ([_CFG, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
            "moe_route": ([_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP],
                          ctypes.c_int),
            "moe_permute": ([_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                             ctypes.c_size_t, _VP], ctypes.c_int),
            "moe_permute_noalloc": ([_CFG, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP],
                                    ctypes.c_int),
            "moe_grouped_mlp": ([_CFG, ctypes.POINTER(MoEWeights), _VP, _VP, _VP, _VP, _VP,
                                 _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP],
                                ctypes.c_int),
            "moe_combine": ([_CFG, _VP, _VP, _VP, _VP, _VP, _VP], ctypes.c_int),
            "moe_forward": ([_CFG, ctypes.POINTER(MoEWeights), _VP, _VP, _VP, _VP,
                             ctypes.c_int32, _VP, ctypes.c_size_t, _VP], ctypes.c_int),
            "moe_get_device_status": ([_VP, ctypes.POINTER(ctypes.c_int32), _VP], ctypes.c_int),
            "moe_prepared_weights_size": ([_CFG, ctypes.POINTER(MoEWeightSizes)], ctypes.c_int),
            "moe_quantize": ([ctypes.c_int32, _VP, ctypes.c_int32, ctypes.c_int32, _VP, _VP, _VP,
                              _VP], ctypes.c_int),
            "moe_prepare_weights": ([_CFG, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _VP,
                                     _VP, _VP, ctypes.POINTER(MoEWeights), _VP], ctypes.c_int),
            "moe_backward_weights_size": ([_CFG, ctypes.POINTER(MoEBwdWeightSizes)],
                                          ctypes.c_int),
            "moe_prepare_backward_weights": ([_CFG, ctypes.c_int32, ctypes.c_int32,
                                              ctypes.c_int32, _VP, _VP, _VP, _VP,
                                              ctypes.POINTER(MoEBwdWeights), _VP], ctypes.c_int),
            "moe_backward_workspace_size": ([_CFG, ctypes.POINTER(ctypes.c_size_t)],
                                            ctypes.c_int),
            "moe_backward": ([_CFG, ctypes.POINTER(MoEWeights), ctypes.POINTER(MoEBwdWeights),
                              ctypes.POINTER(MoEFwdSaved), _VP, _VP, _VP, _VP,
                              ctypes.POINTER(MoEWeightGrads), _VP, ctypes.c_size_t, _VP],
                             ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def _p(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _cuda(t, dtype, name):
    if t is None:
        return None
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor, got "
                         f"{t.dtype} on {t.device} (contiguous={t.is_contiguous()})")
    return t


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, code):
    if code != 0:
        raise MoEError(fn, code)


def moe_workspace_size(cfg: MoEConfig):
    b, r = ctypes.c_size_t(), ctypes.c_int32()
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(b),
                                                          ctypes.byref(r)))
    return b.value, r.value


def moe_forward_workspace_size(cfg: MoEConfig):
    b = ctypes.c_size_t()
    _check("moe_forward_workspace_size",
           lib().moe_forward_workspace_size(ctypes.byref(cfg), ctypes.byref(b)))
    return b.value


def new_workspace(nbytes, device="cuda"):
    """A zeroed byte buffer (the status word must start at zero)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def moe_route(cfg, x, w_router, bias, topk_idx, topk_w, workspace, logits_in=None,
              logits_out=None, stream=None):
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    _check("moe_route", lib().moe_route(
        ctypes.byref(cfg), _p(_cuda(x, bf, "x")), _p(_cuda(w_router, bf, "w_router")),
        _p(_cuda(bias, f32, "bias")), _p(_cuda(logits_in, f32, "logits_in")),
        _p(_cuda(logits_out, f32, "logits_out")), _p(_cuda(topk_idx, i32, "topk_idx")),
        _p(_cuda(topk_w, f32, "topk_w")), _p(workspace), workspace.numel(), _stream(stream)))


def moe_permute(cfg, topk_idx, src_rows, counts, offsets, row_token, token_row, dst_rows,
                workspace, src_scales=None, dst_scales=None, stream=None):
    i32 = torch.int32
    _check("moe_permute", lib().moe_permute(
        ctypes.byref(cfg), _p(_cuda(topk_idx, i32, "topk_idx")), _p(src_rows), _p(src_scales),
        _p(_cuda(counts, i32, "counts")), _p(_cuda(offsets, i32, "offsets")),
        _p(_cuda(row_token, i32, "row_token")), _p(_cuda(token_row, i32, "token_row")),
        _p(dst_rows), _p(dst_scales), _p(workspace), workspace.numel(), _stream(stream)))


def moe_permute_noalloc(cfg, topk_idx, src_rows, counts, offsets, row_token, token_row,
                        dst_rows, src_scales=None, dst_scales=None, stream=None):
    """moe_permute without a workspace (scratch built into the library)."""
    i32 = torch.int32
    _check("moe_permute_noalloc", lib().moe_permute_noalloc(
        ctypes.byref(cfg), _p(_cuda(topk_idx, i32, "topk_idx")), _p(src_rows), _p(src_scales),
        _p(_cuda(counts, i32, "counts")), _p(_cuda(offsets, i32, "offsets")),
        _p(_cuda(row_token, i32, "row_token")), _p(_cuda(token_row, i32, "token_row")),
        _p(dst_rows), _p(dst_scales), _stream(stream)))


def weights_struct(w: dict) -> MoEWeights:
    return MoEWeights(**{k: (w[k].data_ptr() if w.get(k) is not None else None)
                         for k in _WEIGHT_FIELDS})


def moe_prepared_weights_size(cfg: MoEConfig) -> dict:
    v = MoEWeightSizes()
    _check("moe_prepared_weights_size", lib().moe_prepared_weights_size(ctypes.byref(cfg),
                                                                        ctypes.byref(v)))
    return {n: getattr(v, n) for n, _ in MoEWeightSizes._fields_}


def moe_quantize(dtype, x, codes, scales, global_scale=None, stream=None):
    """Block-scaled quantization of a bf16 [rows, cols] tensor (MXFP8)."""
    rows, cols = x.shape
    _check("moe_quantize", lib().moe_quantize(
        DTYPES[dtype] if isinstance(dtype, str) else dtype, _p(_cuda(x, torch.bfloat16, "x")),
        rows, cols, _p(codes), _p(scales), _p(global_scale), _stream(stream)))


def scale_bytes(rows, cols, dtype="mxfp8"):
    """Bytes of the MMA-layout scale buffer of a [rows, cols] block-scaled matrix."""
    return (rows + 127) // 128 * 128 * (cols // (32 if dtype == "mxfp8" else 16))


def moe_prepare_weights(cfg, which, e_begin, e_count, w1, w3, w2, dst, stream=None):
    """Re-lay bf16 row-major expert weights into the kernels' layout (dst)."""
    ws = dst if isinstance(dst, MoEWeights) else weights_struct(dst)
    bf = torch.bfloat16
    _check("moe_prepare_weights", lib().moe_prepare_weights(
        ctypes.byref(cfg), which, e_begin, e_count, _p(_cuda(w1, bf, "w1")),
        _p(_cuda(w3, bf, "w3")), _p(_cuda(w2, bf, "w2")), ctypes.byref(ws), _stream(stream)))


def allocate_prepared_weights(cfg, device="cuda") -> dict:
    """Empty device buffers for the prepared weights of a layer (sizes from
    moe_prepared_weights_size), keyed by the moe_weights field names; fill
    them with moe_prepare_weights, all experts at once or a range at a time."""
    sz = moe_prepared_weights_size(cfg)
    u8 = dict(dtype=torch.uint8, device=device)
    out = {"w1": torch.empty(sz["w13"], **u8), "w3": torch.empty(sz["w13"], **u8),
           "w2": torch.empty(sz["w2"], **u8)}
    if sz["w13_scales"]:
        out["w1_scales"] = torch.empty(sz["w13_scales"], **u8)
        out["w3_scales"] = torch.empty(sz["w13_scales"], **u8)
        out["w2_scales"] = torch.empty(sz["w2_scales"], **u8)
    if cfg.I_shared > 0:
        out["ws1"] = torch.empty(sz["ws13"], **u8)
        out["ws3"] = torch.empty(sz["ws13"], **u8)
        out["ws2"] = torch.empty(sz["ws2"], **u8)
        if sz["ws13_scales"]:
            out["ws1_scales"] = torch.empty(sz["ws13_scales"], **u8)
            out["ws3_scales"] = torch.empty(sz["ws13_scales"], **u8)
            out["ws2_scales"] = torch.empty(sz["ws2_scales"], **u8)
        if sz["ws_globals"]:
            out["ws13_global"] = torch.empty(1, dtype=torch.float32, device=device)
            out["ws2_global"] = torch.empty(1, dtype=torch.float32, device=device)
    if sz["w_globals"]:
        out["w13_global"] = torch.empty(cfg.E, dtype=torch.float32, device=device)
        out["w2_global"] = torch.empty(cfg.E, dtype=torch.float32, device=device)
    return out


def prepare_weights(cfg, raw: dict, stream=None) -> dict:
    """Allocate the prepared weight buffers (torch) and fill them from the
    row-major bf16 tensors in ``raw`` (keys w1, w3, w2 and, with a shared
    expert, ws1, ws3, ws2)."""
    out = allocate_prepared_weights(cfg, raw["w1"].device)
    dst = weights_struct(out)
    moe_prepare_weights(cfg, 0, 0, cfg.E, raw["w1"], raw["w3"], raw["w2"], dst, stream)
    if cfg.I_shared > 0:
        moe_prepare_weights(cfg, 1, 0, 1, raw["ws1"], raw["ws3"], raw["ws2"], dst, stream)
    return out


def moe_grouped_mlp(cfg, weights, rows, counts, offsets, out_rows, workspace, x=None,
                    shared_out=None, row_scales=None, x_scales=None, x_global=None,
                    row_token=None, stream=None):
    """rows=None: fc1 gathers each expert's rows from x through row_token."""
    ws = weights if isinstance(weights, MoEWeights) else weights_struct(weights)
    i32 = torch.int32
    _check("moe_grouped_mlp", lib().moe_grouped_mlp(
        ctypes.byref(cfg), ctypes.byref(ws), _p(rows), _p(row_scales), _p(x), _p(x_scales),
        _p(x_global), _p(_cuda(counts, i32, "counts")), _p(_cuda(offsets, i32, "offsets")),
        _p(_cuda(row_token, i32, "row_token")), _p(out_rows), _p(shared_out), _p(workspace),
        workspace.numel(), _stream(stream)))


def moe_combine(cfg, out_rows, token_row, topk_w, y, shared_out=None, stream=None):
    bf = torch.bfloat16
    _check("moe_combine", lib().moe_combine(
        ctypes.byref(cfg), _p(_cuda(out_rows, bf, "out_rows")),
        _p(_cuda(token_row, torch.int32, "token_row")), _p(_cuda(topk_w, torch.float32, "topk_w")),
        _p(_cuda(shared_out, bf, "shared_out")), _p(_cuda(y, bf, "y")), _stream(stream)))


def moe_forward(cfg, weights, w_router, bias, x, y, workspace, stream=None):
    """Whole layer.  If x and y are host tensors they are copied inside the call."""
    ws = weights if isinstance(weights, MoEWeights) else weights_struct(weights)
    on_host = not x.is_cuda
    if on_host != (not y.is_cuda):
        raise ValueError("x and y must both be host tensors or both device tensors")
    _check("moe_forward", lib().moe_forward(
        ctypes.byref(cfg), ctypes.byref(ws), _p(_cuda(w_router, torch.bfloat16, "w_router")),
        _p(_cuda(bias, torch.float32, "bias")), _p(x), _p(y), 1 if on_host else 0,
        _p(workspace), workspace.numel(), _stream(stream)))


def moe_get_device_status(workspace, stream=None) -> int:
    v = ctypes.c_int32()
    _check("moe_get_device_status",
           lib().moe_get_device_status(_p(workspace), ctypes.byref(v), _stream(stream)))
    return v.value


def moe_backward_weights_size(cfg: MoEConfig) -> dict:
    v = MoEBwdWeightSizes()
    _check("moe_backward_weights_size",
           lib().moe_backward_weights_size(ctypes.byref(cfg), ctypes.byref(v)))
    return {n: getattr(v, n) for n, _ in MoEBwdWeightSizes._fields_}


def moe_prepare_backward_weights(cfg, which, e_begin, e_count, w1, w3, w2, w_router, dst,
                                 stream=None):
    """Transposed tile-major weight copies for the backward (dst: a dict of
    uint8 buffers keyed w2t, w13t, ws2t, wdt, or an MoEBwdWeights)."""
    st = dst if isinstance(dst, MoEBwdWeights) else MoEBwdWeights(
        **{k: (dst[k].data_ptr() if dst.get(k) is not None else None)
           for k, _ in MoEBwdWeights._fields_})
    bf = torch.bfloat16
    _check("moe_prepare_backward_weights", lib().moe_prepare_backward_weights(
        ctypes.byref(cfg), which, e_begin, e_count, _p(_cuda(w1, bf, "w1")),
        _p(_cuda(w3, bf, "w3")), _p(_cuda(w2, bf, "w2")),
        _p(_cuda(w_router, bf, "w_router")), ctypes.byref(st), _stream(stream)))


def prepare_backward_weights(cfg, raw: dict, w_router, stream=None) -> dict:
    """Allocate and fill the backward's weight copies from the row-major bf16
    tensors in ``raw`` (keys w1, w3, w2 and, with a shared expert, ws1, ws3,
    ws2) and the router weight [E, H]."""
    sz = moe_backward_weights_size(cfg)
    dev = raw["w1"].device
    out = {k: (torch.empty(v, dtype=torch.uint8, device=dev) if v else None)
           for k, v in sz.items()}
    moe_prepare_backward_weights(cfg, 0, 0, cfg.E, raw["w1"], raw["w3"], raw["w2"], None, out,
                                 stream)
    moe_prepare_backward_weights(cfg, 1, 0, 1, raw.get("ws1"), raw.get("ws3"), raw.get("ws2"),
                                 w_router, out, stream)
    return out


def moe_backward_workspace_size(cfg: MoEConfig) -> int:
    n = ctypes.c_size_t()
    _check("moe_backward_workspace_size",
           lib().moe_backward_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def moe_backward(cfg, weights, bwd_weights, saved: dict, dy, dx, workspace, dlogits=None,
                 dgate=None, grads=None, accumulate=False, stream=None):
    """Gradients of the bf16 layer.  ``saved`` maps the moe_fwd_saved field
    names (x, rows, logits, topk_idx, topk_w, counts, offsets, row_token,
    token_row, out_rows) to the forward's tensors; ``grads`` (optional) maps
    dw1, dw3, dw2, dws1, dws3, dws2, dw_router to fp32 output tensors, which
    are overwritten, or added to with ``accumulate=True``."""
    ws = weights if isinstance(weights, MoEWeights) else weights_struct(weights)
    bw = bwd_weights if isinstance(bwd_weights, MoEBwdWeights) else MoEBwdWeights(
        **{k: (bwd_weights[k].data_ptr() if bwd_weights.get(k) is not None else None)
           for k, _ in MoEBwdWeights._fields_})
    types = {"x": torch.bfloat16, "rows": torch.bfloat16, "logits": torch.float32,
             "topk_idx": torch.int32, "topk_w": torch.float32, "counts": torch.int32,
             "offsets": torch.int32, "row_token": torch.int32, "token_row": torch.int32,
             "out_rows": torch.bfloat16}
    sv = MoEFwdSaved(**{k: _cuda(saved[k], types[k], k).data_ptr() for k in _SAVED_FIELDS})
    gr = None
    if grads is not None:
        gr = MoEWeightGrads(**{k: (_cuda(grads[k], torch.float32, k).data_ptr()
                                   if grads.get(k) is not None else None)
                               for k in _GRAD_FIELDS}, accumulate=1 if accumulate else 0)
    bf = torch.bfloat16
    _check("moe_backward", lib().moe_backward(
        ctypes.byref(cfg), ctypes.byref(ws), ctypes.byref(bw), ctypes.byref(sv),
        _p(_cuda(dy, bf, "dy")), _p(_cuda(dx, bf, "dx")),
        _p(_cuda(dlogits, torch.float32, "dlogits")), _p(_cuda(dgate, torch.float32, "dgate")),
        ctypes.byref(gr) if gr is not None else None, _p(workspace), workspace.numel(),
        _stream(stream)))


class MoELayer:
    """A layer with its weights resident on the device.

    ``weights`` maps the moe_weights field names (w1, w3, w2, ws1, ...) to
    row-major bf16 device tensors, which are prepared once into the kernels'
    layout (or to already prepared buffers with ``prepared=True``);
    ``forward(x)`` runs the whole layer through moe_forward.
    """

    def __init__(self, cfg: MoEConfig, weights: dict, w_router, bias, device="cuda",
                 prepared=False):
        self.cfg = cfg
        self.weights = dict(weights) if prepared else prepare_weights(cfg, weights)
        self._ws_struct = weights_struct(self.weights)
        self.w_router = w_router
        self.bias = bias
        self.workspace = new_workspace(moe_forward_workspace_size(cfg), device)

    def forward(self, x, out=None, stream=None):
        if out is None:
            out = torch.empty(self.cfg.T, self.cfg.H, dtype=torch.bfloat16, device=x.device,
                              pin_memory=not x.is_cuda)
        moe_forward(self.cfg, self._ws_struct, self.w_router, self.bias, x, out, self.workspace,
                    stream)
        return out

    def device_status(self) -> int:
        return moe_get_device_status(self.workspace)


class MoETrainLayer(MoELayer):
    """A bf16 layer that can also run its backward.

    ``forward(x)`` runs the step calls (route, permute, grouped MLP, combine)
    and keeps what the backward reads; ``backward(dy)`` then returns dx and,
    by default, every weight gradient (fp32, dict keyed like moe_weight_grads)
    plus dlogits and dgate.  ``weights`` are the row-major bf16 tensors (w1, w3,
    w2 and, with a shared expert, ws1, ws3, ws2): they are prepared for the
    forward and transposed for the backward once, here.  Routed weight
    gradients need cfg.pad_multiple % 64 == 0.  The forward keeps x by
    reference: it must not change before the backward that follows.
    """

    def __init__(self, cfg: MoEConfig, weights: dict, w_router, bias, device="cuda"):
        super().__init__(cfg, weights, w_router, bias, device)
        self.bwd_weights = prepare_backward_weights(cfg, weights, w_router)
        nbytes, r_cap = moe_workspace_size(cfg)
        self.step_ws = new_workspace(nbytes, device)
        self.bwd_ws = new_workspace(moe_backward_workspace_size(cfg), device)
        T, H, E, k = cfg.T, cfg.H, cfg.E, cfg.top_k
        i32 = dict(dtype=torch.int32, device=device)
        self.saved = {"logits": torch.empty(T, E, dtype=torch.float32, device=device),
                      "topk_idx": torch.empty(T, k, **i32),
                      "topk_w": torch.empty(T, k, dtype=torch.float32, device=device),
                      "counts": torch.empty(E, **i32), "offsets": torch.empty(E + 1, **i32),
                      "row_token": torch.empty(r_cap, **i32),
                      "token_row": torch.empty(T * k, **i32),
                      "rows": torch.empty(r_cap, H, dtype=torch.bfloat16, device=device),
                      "out_rows": torch.empty(r_cap, H, dtype=torch.bfloat16, device=device)}
        self.shared_out = (torch.empty(T, H, dtype=torch.bfloat16, device=device)
                           if cfg.I_shared > 0 else None)

    def forward(self, x, out=None, stream=None):
        c, sv = self.cfg, self.saved
        if out is None:
            out = torch.empty(c.T, c.H, dtype=torch.bfloat16, device=x.device)
        moe_route(c, x, self.w_router, self.bias, sv["topk_idx"], sv["topk_w"], self.step_ws,
                  logits_out=sv["logits"], stream=stream)
        moe_permute(c, sv["topk_idx"], x, sv["counts"], sv["offsets"], sv["row_token"],
                    sv["token_row"], sv["rows"], self.step_ws, stream=stream)
        moe_grouped_mlp(c, self._ws_struct, sv["rows"], sv["counts"], sv["offsets"],
                        sv["out_rows"], self.step_ws, x=x, shared_out=self.shared_out,
                        stream=stream)
        moe_combine(c, sv["out_rows"], sv["token_row"], sv["topk_w"], out,
                    shared_out=self.shared_out, stream=stream)
        sv["x"] = x
        return out

    def backward(self, dy, weight_grads=True, grads=None, accumulate=False, stream=None):
        """``grads``: fp32 tensors to write (or, with ``accumulate``, add) the
        weight gradients into, keyed like moe_weight_grads; allocated when
        not given."""
        c = self.cfg
        dev = dy.device
        f32 = dict(dtype=torch.float32, device=dev)
        dx = torch.empty(c.T, c.H, dtype=torch.bfloat16, device=dev)
        res = {"dx": dx, "dlogits": torch.empty(c.T, c.E, **f32),
               "dgate": torch.empty(c.T, c.top_k, **f32)}
        if grads is not None:
            res.update(grads)
        elif weight_grads:
            grads = {"dw1": torch.empty(c.E, c.I, c.H, **f32),
                     "dw3": torch.empty(c.E, c.I, c.H, **f32),
                     "dw2": torch.empty(c.E, c.H, c.I, **f32),
                     "dw_router": torch.empty(c.E, c.H, **f32)}
            if c.I_shared > 0:
                grads.update(dws1=torch.empty(c.I_shared, c.H, **f32),
                             dws3=torch.empty(c.I_shared, c.H, **f32),
                             dws2=torch.empty(c.H, c.I_shared, **f32))
            res.update(grads)
        moe_backward(c, self._ws_struct, self.bwd_weights, self.saved, dy, dx, self.bwd_ws,
                     dlogits=res["dlogits"], dgate=res["dgate"], grads=grads,
                     accumulate=accumulate, stream=stream)
        return res

    def device_status(self) -> int:
        return max(moe_get_device_status(self.step_ws), moe_get_device_status(self.bwd_ws))
