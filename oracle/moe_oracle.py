"""CPU oracle of the routed MoE layer (forward, and the bf16 backward) -- TEST
INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this module.  The library never calls it, and it shares no code with the CUDA
kernels: it is the plain, slow statement of what the layer computes, used to
check the kernels element by element.

Sources (page title, then the passage):

* TransformerEngine PR "DeepSeekV3Layer: full MoE transformer layer",
  Description, DeepSeekV3MoE bullet: a sigmoid router with an aux-loss-free bias
  and grouped top-k; experts as GroupedLinear -> ScaledSwiGLU -> GroupedLinear;
  an optional shared expert.
* same PR, Performance section, "NCCL EP local permute" row: staging into an
  expert-major layout with zero-filled padding, and its reduce (the combine).
* same PR, Performance section, "MXFP8 quantization" row: MXFP8 activations
  (e4m3 elements with an e8m0 scale per 32 along K).
* sglang PR "Mistral Large 3 NVFP4 TRTLLM MoE support", Modifications: W4A4
  NVFP4 (e2m1 elements, e4m3 scale per 16 along K, fp32 per-tensor global
  scale from amax).
* TransformerEngine PR "DeepSeekV3Layer", Performance section, "fused grouped
  MLP" row: the backward of the expert MLP (dGLU and the wgrad GEMMs); the
  backward here is the gradient of the same layer (dx, the router's dlogits,
  every weight gradient), written out by the chain rule.

quant_rows.c restates the two row quantizers in plain C (loaded through
native.py when gcc is available; the CPU tests check it against the numpy
functions here bit for bit), only so that full-size experts take well under a
second.

Arithmetic is fp64 on the values each stored tensor holds.  The storage
roundings that the layer defines are reproduced: bf16 storage of h, of the fc2
output rows and of y; the quantized codes of x, of the weights and of h.
Where the pages leave a step open, the reading taken is stated at the function.

Parity status: every function here is pinned by the CPU tests (brute force on
tiny inputs, closed forms, library cross-checks, invariants, a hand-worked
NVFP4 and MXFP8 expert that pins the quantized composition stage by stage, and
central finite differences of the forward for every backward function).
Quantization noise itself has no external truth to pin against; only the
code-level rules (round-to-nearest-even, saturation, scale selection and the
scope of each global scale) are pinned.
"""

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# ---------------------------------------------------------------------------
# bf16 storage
# ---------------------------------------------------------------------------

BF16_MAX = float.fromhex("0x1.fep127")


def from_bf16(t) -> np.ndarray:
    """bf16 tensor (torch) or raw uint16 bits (numpy) -> float64 values."""
    if type(t).__module__.startswith("torch"):
        import torch
        t = t.detach().cpu().contiguous().view(torch.int16).numpy()
    bits = np.asarray(t).view(np.uint16).astype(np.uint32) << 16
    return bits.view(np.float32).astype(np.float64)


def round_bf16(v) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even.

    bf16 has 8 significant bits; for |v| in [2^(e-1), 2^e) the spacing is
    2^(e-8).  Below the smallest normal (2^-126) the spacing stays 2^-133.
    """
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)
    e = np.maximum(e, -125)
    q = np.ldexp(np.rint(np.ldexp(v, 8 - e)), e - 8)
    q = np.where(np.abs(q) > BF16_MAX, np.copysign(np.inf, v), q)
    return q


def to_bf16_bits(v) -> np.ndarray:
    """float64 -> bf16 bit patterns (uint16), rounding to nearest even."""
    q = round_bf16(v).astype(np.float32)
    return (q.view(np.uint32) >> 16).astype(np.uint16)


# ---------------------------------------------------------------------------
# Router: sigmoid score, aux-loss-free bias, grouped top-k, normalised gates
# (TransformerEngine PR "DeepSeekV3Layer", Description, DeepSeekV3MoE bullet)
# ---------------------------------------------------------------------------

def router_logits(x, w_router) -> np.ndarray:
    """logits[t, e] = sum_h x[t, h] * W_r[e, h], exact products, fp64 sums."""
    return np.asarray(x, np.float64) @ np.asarray(w_router, np.float64).T


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-np.asarray(z, np.float64)))


def route(logits, bias, n_group, topk_group, top_k, rsf):
    """Grouped top-k selection and gates, per token.

    Readings where the pages give only the names:
      * score s = sigmoid(logit); selection key b = s + bias (the bias only
        steers selection: "aux-loss-free" balancing leaves the gate values
        alone), gates use the unbiased s;
      * groups are contiguous runs of E / n_group experts; a group's score is
        the sum of its two largest b (the DeepSeek-V3 rule the layer is named
        after);
      * the topk_group best groups are kept, every expert outside them is
        excluded (as -inf, since b can be negative);
      * ties, for groups and experts, go to the lower index; the k selected
        experts are listed by b descending;
      * gate_j = s_j / sum_j' s_j' * routed_scaling_factor.

    Returns a dict with idx [T, k] int32, w [T, k] float64 and the margins that
    decide near-ties: group_margin (g-th minus (g+1)-th group score) and
    expert_margin (k-th minus (k+1)-th eligible b), +inf where no competitor.
    """
    logits = np.asarray(logits, np.float64)
    T, E = logits.shape
    G, g, k = n_group, topk_group, top_k
    gs = E // G
    s = sigmoid(logits)
    b = s + np.asarray(bias, np.float64)[None, :]

    grouped = b.reshape(T, G, gs)
    top2 = np.sort(grouped, axis=2)[:, :, -2:] if gs >= 2 else grouped
    gscore = top2.sum(axis=2)                                   # [T, G]
    gorder = np.argsort(-gscore, axis=1, kind="stable")         # desc, ties -> low index
    keep = np.zeros((T, G), dtype=bool)
    np.put_along_axis(keep, gorder[:, :g], True, axis=1)
    gsorted = np.take_along_axis(gscore, gorder, axis=1)
    group_margin = (gsorted[:, g - 1] - gsorted[:, g]) if g < G else np.full(T, np.inf)

    masked = np.where(np.repeat(keep, gs, axis=1), b, -np.inf)
    eorder = np.argsort(-masked, axis=1, kind="stable")
    idx = eorder[:, :k]
    bsorted = np.take_along_axis(masked, eorder, axis=1)
    if k < E:
        nxt = bsorted[:, k]
        expert_margin = np.where(np.isfinite(nxt), bsorted[:, k - 1] - nxt, np.inf)
    else:
        expert_margin = np.full(T, np.inf)

    s_sel = np.take_along_axis(s, idx, axis=1)
    w = s_sel / s_sel.sum(axis=1, keepdims=True) * rsf
    return dict(idx=idx.astype(np.int32), w=w, s=s, b=b, group_score=gscore,
                group_margin=group_margin, expert_margin=expert_margin)


# ---------------------------------------------------------------------------
# Permute into padded expert-major order, and its inverse maps
# (TransformerEngine PR "DeepSeekV3Layer", Performance, "NCCL EP local permute")
# ---------------------------------------------------------------------------

def permute_maps(idx, E, pad_multiple):
    """Histogram, padded exclusive scan and the two row maps.

    Within an expert's segment rows are in ascending token order (a token
    picks an expert at most once).  Each segment is padded up to a multiple of
    ``pad_multiple`` rows; pad rows map to token -1 and hold zeros.

    Returns counts [E], offsets [E+1], row_token [offsets[E]] (-1 for pads) and
    token_row [T*k] (token_row[t*k + j] = row of (t, j)).
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    P = pad_multiple
    counts = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            counts[idx[t, j]] += 1
    padded = (counts + P - 1) // P * P
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + padded[e]
    row_token = np.full(int(offsets[E]), -1, dtype=np.int64)
    token_row = np.zeros(T * k, dtype=np.int64)
    fill = offsets[:E].copy()
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            r = fill[e]
            fill[e] += 1
            row_token[r] = t
            token_row[t * k + j] = r
    return dict(counts=counts, offsets=offsets, row_token=row_token, token_row=token_row)


def gather_rows(src, row_token):
    """dst[r] = src[row_token[r]], zero rows where row_token[r] == -1."""
    src = np.asarray(src)
    out = np.zeros((len(row_token),) + src.shape[1:], dtype=src.dtype)
    valid = row_token >= 0
    out[valid] = src[row_token[valid]]
    return out


# ---------------------------------------------------------------------------
# Element formats (OCP 8-bit floating point and microscaling formats)
# ---------------------------------------------------------------------------

def _e4m3_magnitudes():
    """Values of the non-negative E4M3 codes 0x00..0x7E (0x7F is NaN).

    Exponent bias 7, 3 mantissa bits, subnormals when the exponent field is 0.
    """
    vals = np.zeros(127)
    for c in range(127):
        ef, m = c >> 3, c & 7
        vals[c] = (m / 8.0) * 2.0 ** -6 if ef == 0 else (1.0 + m / 8.0) * 2.0 ** (ef - 7)
    return vals


E4M3_MAG = _e4m3_magnitudes()          # ascending in the code
E4M3_MAX = 448.0
E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MAX = 6.0


def decode_e4m3(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.int64)
    mag = E4M3_MAG[np.minimum(codes & 0x7F, 126)]
    mag = np.where((codes & 0x7F) == 0x7F, np.nan, mag)
    return np.where(codes & 0x80, -mag, mag)


def decode_e2m1(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.int64)
    mag = E2M1_MAG[codes & 7]
    return np.where(codes & 8, -mag, mag)


def decode_e8m0(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.int64)
    return np.where(codes == 255, np.nan, np.ldexp(1.0, codes - 127))


def _nearest_code(a, table):
    """Index of the table entry nearest to a (a within [0, table[-1]]),
    ties to the even index (the even mantissa)."""
    hi = np.clip(np.searchsorted(table, a, side="left"), 0, len(table) - 1)
    lo = np.maximum(hi - 1, 0)
    dlo = a - table[lo]
    dhi = table[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    return np.where(pick_hi, hi, lo)


def encode_e4m3(v) -> np.ndarray:
    """Round to nearest E4M3, ties to even, saturating to +-448."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E4M3_MAX)
    c = _nearest_code(a, E4M3_MAG).astype(np.uint8)
    return np.where(np.signbit(v), c | 0x80, c).astype(np.uint8)


def encode_e2m1(v) -> np.ndarray:
    """Round to nearest E2M1, ties to even, saturating to +-6 (one code per byte)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E2M1_MAX)
    c = _nearest_code(a, E2M1_MAG).astype(np.uint8)
    return np.where(np.signbit(v), c | 0x8, c).astype(np.uint8)


# ---------------------------------------------------------------------------
# MXFP8: e4m3 elements, one e8m0 scale per 32 consecutive K elements
# (TransformerEngine PR "DeepSeekV3Layer", Performance, MXFP8 rows)
# ---------------------------------------------------------------------------

MX_BLOCK = 32
E4M3_EMAX = 8   # exponent of the largest normal e4m3 value, 448 = 1.75 * 2^8


def mxfp8_quantize(v):
    """Quantize rows of bf16 values [R, K] to MXFP8 (K % 32 == 0).

    Scale rule of the OCP microscaling format: X = 2^(floor(log2 amax) - 8),
    with the e8m0 code clamped to [0, 254]; an all-zero block takes X = 1.
    Elements are v / X rounded to nearest-even e4m3, saturating at 448.
    Returns (codes uint8 [R, K], scale codes uint8 [R, K/32]).
    """
    v = np.asarray(v, dtype=np.float64)
    R, K = v.shape
    blocks = v.reshape(R, K // MX_BLOCK, MX_BLOCK)
    amax = np.abs(blocks).max(axis=2)
    _, e = np.frexp(amax)                    # amax = m * 2^e, m in [0.5, 1)
    xexp = (e - 1) - E4M3_EMAX               # floor(log2 amax) - emax
    scode = np.clip(xexp + 127, 0, 254)
    scode = np.where(amax == 0, 127, scode).astype(np.uint8)
    X = np.ldexp(1.0, scode.astype(np.int64) - 127)
    codes = encode_e4m3(blocks / X[:, :, None]).reshape(R, K)
    return codes, scode


def mxfp8_dequantize(codes, scodes):
    R, K = codes.shape
    vals = decode_e4m3(codes).reshape(R, K // MX_BLOCK, MX_BLOCK)
    return (vals * decode_e8m0(scodes)[:, :, None]).reshape(R, K)


# ---------------------------------------------------------------------------
# NVFP4: e2m1 elements, one e4m3 scale per 16 K elements, fp32 global scale
# (sglang PR "Mistral Large 3 NVFP4 TRTLLM MoE support", Modifications: W4A4)
# ---------------------------------------------------------------------------

NV_BLOCK = 16
_F32 = np.float32


def nvfp4_global_scale(amax) -> np.float32:
    """Global encode scale g = (448 * 6) / amax in fp32, or 1 when amax == 0.

    448 * 6 maps the largest block (amax) onto the largest e4m3 block scale
    times the largest e2m1 element.
    """
    amax = _F32(amax)
    if amax == 0:
        return _F32(1.0)
    return _F32(_F32(2688.0) / amax)


def nvfp4_quantize(v, g):
    """Quantize rows of bf16 values [R, K] to NVFP4 (K % 16 == 0).

    Per 16-element block, each step one IEEE fp32 operation in this order:
      t = (amax16 / 6) * g;  sb = e4m3(t) rounded to nearest-even, saturating;
      if sb == 0 the block's elements are all zero codes;
      else r = g / dec(sb) and q_i = e2m1(v_i * r), nearest-even, saturating.
    Returns (codes uint8 [R, K] one e2m1 code per byte, sb uint8 [R, K/16]).
    """
    g = _F32(g)
    v32 = np.asarray(v, dtype=np.float64).astype(_F32)
    R, K = v32.shape
    blocks = v32.reshape(R, K // NV_BLOCK, NV_BLOCK)
    amax = np.abs(blocks).max(axis=2).astype(_F32)
    t = (amax / _F32(6.0)).astype(_F32) * g
    sb = encode_e4m3(t.astype(_F32).astype(np.float64))
    dec_sb = decode_e4m3(sb).astype(_F32)
    with np.errstate(divide="ignore", invalid="ignore", over="ignore"):
        r = (g / dec_sb).astype(_F32)
        scaled = (blocks * r[:, :, None]).astype(_F32)
        codes = encode_e2m1(scaled.astype(np.float64))
    codes = np.where((sb == 0)[:, :, None], np.uint8(0), codes).astype(np.uint8)
    return codes.reshape(R, K), sb.astype(np.uint8)


def nvfp4_dequantize(codes, sb, g):
    R, K = codes.shape
    vals = decode_e2m1(codes).reshape(R, K // NV_BLOCK, NV_BLOCK)
    return (vals * decode_e4m3(sb)[:, :, None] / np.float64(_F32(g))).reshape(R, K)


ROW_BLOCK = 128


def by_row_blocks(fn, v, rows=ROW_BLOCK):
    """fn applied to consecutive blocks of `rows` rows of v, results stacked.

    Every quantizer here is row-local once its global scale is fixed (its
    blocks of 16 or 32 elements run along a row), so applying it block by
    block gives exactly the result of one call on the whole matrix.  The blocks
    run on a thread pool (numpy releases the interpreter lock inside its array
    operations); that only keeps full-size layers within minutes on the host.
    """
    v = np.asarray(v, np.float64)
    if v.shape[0] <= rows:
        return fn(v)
    parts = [v[i:i + rows] for i in range(0, v.shape[0], rows)]
    with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        return np.concatenate(list(ex.map(fn, parts)), axis=0)


def _qdq_native(v, dtype, g):
    """The same quantize-dequantize through the C restatement in quant_rows.c
    (checked bit for bit against the numpy functions above), or None."""
    from . import native
    L = native.load()
    if L is None:
        return None
    import ctypes
    v = np.ascontiguousarray(v, dtype=np.float64)
    if v.ndim != 2:
        return None
    out = np.empty_like(v)
    dp = ctypes.POINTER(ctypes.c_double)
    if dtype == "mxfp8":
        L.oracle_mxfp8_qdq_rows(v.ctypes.data_as(dp), out.ctypes.data_as(dp), v.shape[0],
                                v.shape[1])
    else:
        L.oracle_nvfp4_qdq_rows(v.ctypes.data_as(dp), out.ctypes.data_as(dp), v.shape[0],
                                v.shape[1], float(g))
    return out


def quantize_dequantize(v, dtype, g=None, native=True):
    """The values a quantized tensor stands for, as the MMA consumes them.

    NVFP4: ``g`` is the tensor's global encode scale; when None it is set from
    the amax of ``v`` itself (``v`` is then the whole tensor).  ``native``
    allows the C restatement of the row quantizers (same results)."""
    if dtype == "bf16":
        return np.asarray(v, np.float64)
    if dtype == "nvfp4" and g is None:
        g = nvfp4_global_scale(np.abs(np.asarray(v, np.float64)).max())
    if native and dtype in ("mxfp8", "nvfp4"):
        out = _qdq_native(v, dtype, g)
        if out is not None:
            return out
    if dtype == "mxfp8":
        return by_row_blocks(lambda b: mxfp8_dequantize(*mxfp8_quantize(b)), v)
    if dtype == "nvfp4":
        return by_row_blocks(lambda b: nvfp4_dequantize(*nvfp4_quantize(b, g), g), v)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# Expert MLP: GroupedLinear (fc1, W1 and W3) -> SwiGLU -> GroupedLinear (fc2)
# (TransformerEngine PR "DeepSeekV3Layer", Description, DeepSeekV3MoE bullet)
# ---------------------------------------------------------------------------

def silu(a):
    a = np.asarray(a, np.float64)
    return a / (1.0 + np.exp(-a))


def swiglu(a, u):
    """silu(gate) * up.  "ScaledSwiGLU" carries no further scale here: the gate
    weights are applied in the combine, and W1 is the gate, W3 the up proj."""
    return silu(a) * np.asarray(u, np.float64)


def _store(v, rounding):
    """The value a bf16 tensor stores (rounding=False: the exact value, for the
    smooth function the backward differentiates)."""
    return round_bf16(v) if rounding else np.asarray(v, np.float64)


def expert_fc1(X, W1, W3, rounding=True):
    """h = bf16(silu(X W1^T) * (X W3^T)) for one expert's rows X [m, H]."""
    a = X @ W1.T
    u = X @ W3.T
    return _store(swiglu(a, u), rounding)


def expert_fc2(h, W2, rounding=True):
    """o = bf16(h W2^T) for one expert's (possibly dequantized) h [m, I]."""
    return _store(h @ W2.T, rounding)


def combine(out_rows, token_row, w, shared_out=None, rounding=True):
    """y[t] = bf16(sum_j w[t, j] * out_rows[token_row[t*k + j]] (+ shared[t])).

    The gate-weighted scatter-add of the pages, written as a per-token sum in
    the order j = 0..k-1 of the selection.
    """
    w = np.asarray(w, np.float64)
    T, k = w.shape
    acc = np.zeros((T, out_rows.shape[1]), dtype=np.float64)
    tr = np.asarray(token_row).reshape(T, k)
    for j in range(k):
        acc += w[:, j:j + 1] * out_rows[tr[:, j]]
    if shared_out is not None:
        acc += shared_out
    return _store(acc, rounding)


# ---------------------------------------------------------------------------
# The whole layer
# ---------------------------------------------------------------------------

def prepare_expert_weights(W1, W3, W2, dtype):
    """An expert's weights as its GEMMs consume them: the bf16 values for
    bf16; for MXFP8 / NVFP4 the dequantized values of their codes.  W1 and W3
    are quantized as one stacked fc1 tensor (NVFP4: one global scale for both,
    from their joint amax), W2 on its own (its own global scale)."""
    if dtype == "bf16":
        return (np.asarray(W1, np.float64), np.asarray(W3, np.float64),
                np.asarray(W2, np.float64))
    I = W1.shape[0]
    w13 = quantize_dequantize(np.concatenate([W1, W3], axis=0), dtype)
    return w13[:I], w13[I:], quantize_dequantize(W2, dtype)


def expert_forward(X_deq, W1, W3, W2, dtype, h_global=None, prepared=False, rounding=True):
    """One expert on its rows: dequantized x rows in, bf16 fc2 rows out.

    W1/W3/W2 are the bf16 weight values, or (``prepared=True``) the output of
    prepare_expert_weights.  For MXFP8/NVFP4, h is rounded to bf16 and then
    quantized; its NVFP4 global scale is set from the amax over this expert's
    rows (each expert's fc2 input is its own tensor of the grouped GEMM),
    unless ``h_global`` is given.
    """
    w1, w3, w2 = (W1, W3, W2) if prepared else prepare_expert_weights(W1, W3, W2, dtype)
    h = expert_fc1(X_deq, w1, w3, rounding)
    if dtype == "nvfp4":
        g = nvfp4_global_scale(np.abs(h).max()) if h_global is None else h_global
        hq = quantize_dequantize(h, dtype, g)
    else:
        hq = quantize_dequantize(h, dtype)
    return h, expert_fc2(hq, w2, rounding)


def forward(cfg, x, w_router, bias, w1, w3, w2, shared=None, logits=None,
            experts=None, rounding=True):
    """Full layer forward on the host.

    ``x``, ``w_router`` and the weights are float64 arrays of the bf16 inputs;
    ``w1``/``w3``/``w2`` may be callables ``e -> array`` so that large
    workloads can hand over one expert at a time.  ``experts`` limits the
    expert math to a subset (rows of other experts stay zero); the routing,
    the maps and the quantized x cover all tokens.  ``rounding=False`` skips
    the bf16 storage of h, the fc2 rows and y (the smooth function the
    backward differentiates).
    """
    T, H = x.shape
    E = cfg.E
    get = (lambda W, e: W(e) if callable(W) else W[e])
    if logits is None:
        logits = router_logits(x, w_router)
    r = route(logits, bias, cfg.n_group, cfg.topk_group, cfg.top_k, cfg.rsf)
    m = permute_maps(r["idx"], E, cfg.pad_multiple)
    xq = quantize_dequantize(x, cfg.dtype) if cfg.dtype != "nvfp4" else None
    if cfg.dtype == "nvfp4":
        gx = nvfp4_global_scale(np.abs(x).max())
        xq = quantize_dequantize(x, "nvfp4", gx)
    rows = gather_rows(xq, m["row_token"])
    Rn = rows.shape[0]
    out_rows = np.zeros((Rn, H))
    h_rows = np.zeros((Rn, cfg.I))
    for e in (range(E) if experts is None else experts):
        lo, cnt = int(m["offsets"][e]), int(m["counts"][e])
        if cnt == 0:
            continue
        h, o = expert_forward(rows[lo:lo + cnt], get(w1, e), get(w3, e), get(w2, e), cfg.dtype,
                              rounding=rounding)
        h_rows[lo:lo + cnt] = h
        out_rows[lo:lo + cnt] = o
    shared_out = None
    if shared is not None:
        _, shared_out = expert_forward(xq, shared[0], shared[1], shared[2], cfg.dtype,
                                       rounding=rounding)
    y = combine(out_rows, m["token_row"], r["w"], shared_out, rounding)
    return dict(logits=logits, route=r, maps=m, xq=xq, rows=rows, h_rows=h_rows,
                out_rows=out_rows, shared_out=shared_out, y=y)


# ---------------------------------------------------------------------------
# Backward (input gradients) of the bf16 layer
# (TransformerEngine PR "DeepSeekV3Layer", Performance, "fused grouped MLP"
#  row: dGLU backward and the grouped GEMMs of the backward pass)
# ---------------------------------------------------------------------------

def expert_backward(X, W1, W3, W2, dO):
    """Input gradient of one expert on its rows.

    Forward: a = X W1^T, u = X W3^T, h = silu(a) u, O = h W2^T.  Given dO =
    dL/dO [m, H]:
      dh = dO W2;  da = dh * u * silu'(a);  du = dh * silu(a);
      dX = da W1 + du W3,
    with silu'(a) = sigma(a) (1 + a (1 - sigma(a))).  The bf16 storage of h
    and O has no derivative; it is read as the identity (the gradient of the
    smooth function, forward with rounding=False).  Returns dX and the
    intermediates.
    """
    X, W1, W3, W2, dO = (np.asarray(t, np.float64) for t in (X, W1, W3, W2, dO))
    a = X @ W1.T
    u = X @ W3.T
    sg = sigmoid(a)
    dh = dO @ W2
    da = dh * u * (sg * (1.0 + a * (1.0 - sg)))
    du = dh * (a * sg)
    return da @ W1 + du @ W3, dict(a=a, u=u, dh=dh, da=da, du=du)


def gate_backward(logits, idx, rsf, dgate):
    """d logits from d gates.  Gates: w_j = rsf * s_j / S over the selected
    experts (s = sigmoid(logit), S = sum of the selected s); the selection and
    the bias are piecewise constant, so only selected experts get a gradient:
      ds_j = rsf * (g_j / S - sum_i g_i s_i / S^2),  dlogit_j = ds_j s_j (1 - s_j)
    with g = dL/dw.  Returns [T, E]."""
    logits = np.asarray(logits, np.float64)
    s = sigmoid(logits)
    s_sel = np.take_along_axis(s, idx, axis=1)
    S = s_sel.sum(axis=1, keepdims=True)
    g = np.asarray(dgate, np.float64)
    ds = rsf * (g / S - (g * s_sel).sum(axis=1, keepdims=True) / S ** 2)
    dl = np.zeros_like(logits)
    np.put_along_axis(dl, idx, ds * s_sel * (1.0 - s_sel), axis=1)
    return dl


def expert_weight_grads(X, dO, mid, rounding=True):
    """Weight gradients of one expert from its rows X, dO and the
    intermediates of expert_backward: with h = silu(a) u as the forward
    stores it (bf16 when ``rounding``),
      dW1 = da^T X,  dW3 = du^T X,  dW2 = dO^T h."""
    X, dO = np.asarray(X, np.float64), np.asarray(dO, np.float64)
    h = _store(swiglu(mid["a"], mid["u"]), rounding)
    return mid["da"].T @ X, mid["du"].T @ X, dO.T @ h


def backward(cfg, x, w_router, bias, w1, w3, w2, dy, shared=None, logits=None, rounding=True,
             weight_grads=None):
    """Gradients of the bf16 layer for dL/dy = dy, with its intermediates.

    y[t] = sum_j w[t, j] O[row(t, j)] + shared(x[t]); the combine's backward
    gives dO[row(t, j)] = w[t, j] dy[t] and dgate[t, j] = <dy[t], O[row(t, j)]>
    (O as the forward stores it, bf16); each expert's rows give dX rows
    (expert_backward); dx[t] = sum_j dX[row(t, j)] + shared's dx[t] +
    (d logits W_r)[t] (gate_backward through the router GEMM).
    ``weight_grads``: None for none, True for every expert, or an iterable
    of expert ids; then dw1/dw3/dw2 map those experts to dW1_e, dW3_e, dW2_e
    (expert_weight_grads on the expert's rows), and dws1/dws3/dws2 (shared
    expert on x with dO = dy) and dw_router = dlogits^T x are added.
    ``w1``/``w3``/``w2`` may be callables e -> array, as in forward.
    ``rounding=False``: the O in dgate and the h in dW2 are the exact values
    (the gradient of forward with rounding=False).
    """
    if cfg.dtype != "bf16":
        raise ValueError("the backward is written for the bf16 layer")
    get = (lambda W, e: W(e) if callable(W) else W[e])
    f = forward(cfg, x, w_router, bias, w1, w3, w2, shared=shared, logits=logits,
                rounding=rounding)
    r, m = f["route"], f["maps"]
    dy = np.asarray(dy, np.float64)
    T, k = r["idx"].shape
    tr = np.asarray(m["token_row"]).reshape(T, k)
    dgate = np.einsum("th,tjh->tj", dy, f["out_rows"][tr])
    dO = np.zeros_like(f["out_rows"])
    for j in range(k):
        dO[tr[:, j]] = r["w"][:, j:j + 1] * dy
    if weight_grads is None:
        wg = set()
    elif weight_grads is True:
        wg = set(range(cfg.E))
    else:
        wg = set(int(e) for e in weight_grads)
    dw1, dw3, dw2 = {}, {}, {}
    dX_rows = np.zeros_like(f["rows"])
    for e in range(cfg.E):
        lo, cnt = int(m["offsets"][e]), int(m["counts"][e])
        if cnt == 0:
            if e in wg:
                dw1[e] = np.zeros((cfg.I, cfg.H))
                dw3[e] = np.zeros((cfg.I, cfg.H))
                dw2[e] = np.zeros((cfg.H, cfg.I))
            continue
        Xe, dOe = f["rows"][lo:lo + cnt], dO[lo:lo + cnt]
        dX_rows[lo:lo + cnt], mid = expert_backward(Xe, get(w1, e), get(w3, e), get(w2, e), dOe)
        if e in wg:
            dw1[e], dw3[e], dw2[e] = expert_weight_grads(Xe, dOe, mid, rounding)
    dx = np.zeros_like(np.asarray(x, np.float64))
    for j in range(k):
        dx += dX_rows[tr[:, j]]
    dx_shared = None
    out = {}
    if shared is not None:
        dx_shared, mid_s = expert_backward(x, shared[0], shared[1], shared[2], dy)
        dx += dx_shared
        if weight_grads is not None:
            out["dws1"], out["dws3"], out["dws2"] = expert_weight_grads(x, dy, mid_s, rounding)
    dl = gate_backward(f["logits"], r["idx"], cfg.rsf, dgate)
    dx += dl @ np.asarray(w_router, np.float64)
    if weight_grads is not None:
        out.update(dw1=dw1, dw3=dw3, dw2=dw2,
                   dw_router=dl.T @ np.asarray(x, np.float64))
    out.update(dx=dx, dlogits=dl, dgate=dgate, dO=dO, dX_rows=dX_rows, dx_shared=dx_shared,
               fwd=f)
    return out
