"""Throughput of the routed MoE layer forward on B200.

One step = one whole forward of the layer (router GEMM + grouped top-k,
quantize, permute, grouped fc1+SwiGLU / fc2, combine) over one batch of T
synthetic tokens, weights resident in HBM.  The default workload is the
largest single-GPU one: the DeepSeek-V4 routed-expert geometry in NVFP4 W4A4
at prefill size (T=8192, H=7168, I=3072, E=384, groups 8/4, top-6); --config
picks another.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  python bench.py --backward --config mid_bf16_shared_T2048   (the bf16 backward)

With N > 1 (torchrun) every rank runs an independent replica on its own batch
(tokens are independent, so the layer shards by batch with no exchange): weak
scaling, whole-job tokens/s = N*T*K / max-over-ranks time.

--impl reference times the CPU oracle (fp64) on a bounded token sample of the
same workload, on rank 0 only.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402
from synth.configs import BENCH_CONFIG  # noqa: E402

METRIC = "MoE layer fwd tokens/s at 1 B200; % of roofline (tensor peak or HBM GB/s)"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def _workload(cfg, l2_note):
    return {
        "workload": f"routed MoE layer forward, {cfg.name}",
        "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "n_group": cfg.n_group,
        "topk_group": cfg.topk_group, "top_k": cfg.top_k, "I_shared": cfg.I_shared,
        "routed_scaling_factor": cfg.rsf, "pad_multiple": cfg.pad_multiple,
        "global_batch": None, "seq_len": None, "l2": l2_note,
    }


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self):
        return time.time()

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0=0.0, t1=float("inf")):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, l in self.lines:
            if ts < t0 or ts > t1:
                continue
            parts = [x.strip() for x in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# Replicas: the layer shards by batch with no exchange.  Every rank holds the
# same weights and runs its own batch of T tokens (drawn with seed = rank); the
# job's time is the slowest rank's, and its throughput counts every rank's tokens.

def replica_config(cfg, rank):
    """The seeds a rank draws its token batch with (same shapes)."""
    return cfg.scaled(seed=rank) if rank else cfg


def replica_inputs(cfg, rank, device):
    """A rank's inputs: its own token batch, the job's router weights and bias
    (expert weights are drawn from `cfg` as well, in prepare_streaming)."""
    w_router, bias = synth.gen_router(cfg, device)
    return synth.gen_x(replica_config(cfg, rank), device), w_router, bias


def max_over_ranks(value, dist, device):
    """The largest of every rank's value (each rank passes its own)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank, n_ranks, ms_max):
    return n_ranks * tokens_per_rank / (ms_max * 1e-3)


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle
# ---------------------------------------------------------------------------

def _host_cores():
    """Threads the oracle uses: numpy's BLAS pool and the OpenMP pool of its C
    row quantizers, each as wide as the host."""
    n = os.cpu_count() or 1
    try:
        from threadpoolctl import threadpool_info
        b = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max([n] + b)
    except Exception:
        return n


def oracle_tokens(cfg, seconds, device):
    """Tokens in the oracle's sample so that one pass takes about `seconds` on
    the host: a one-token pass is timed first (its time goes mostly into
    preparing the weights of the experts the token touches, so a pass grows
    about linearly with the tokens until every expert is touched)."""
    _, t1, _ = time_oracle(cfg, 1, 1, 0, device)
    n = int(seconds / max(t1, 1e-6))
    if n >= 2 * cfg.E // max(1, cfg.top_k):   # every expert touched: only the GEMMs grow
        n = 128
    return max(1, min(128, cfg.T, n))


def oracle_sample(cfg, n_tokens, device):
    """The oracle's inputs: the first n_tokens tokens of the workload's batch
    (the GPU arm's draws), the router, and host copies of the bf16 weights of
    exactly the experts those tokens are routed to."""
    from oracle import moe_oracle as O
    xh = O.from_bf16(synth.gen_x(cfg, device)[:n_tokens])
    wr, bias = synth.gen_router(cfg, device)
    wrh, bh = O.from_bf16(wr), bias.cpu().numpy().astype(np.float64)
    r = O.route(O.router_logits(xh, wrh), bh, cfg.n_group, cfg.topk_group, cfg.top_k, cfg.rsf)
    experts = sorted(set(r["idx"].ravel().tolist()))
    W = {e: tuple(t.cpu() for t in synth.gen_expert_weights(cfg, e, device)) for e in experts}
    sh = synth.gen_shared_weights(cfg, device)
    sh = tuple(O.from_bf16(t) for t in sh) if sh is not None else None
    return xh, wrh, bh, W, sh


def time_oracle(cfg, n_tokens, steps, warmup, device):
    """The oracle's forward (as it stands: weights quantized inside, fp64
    arithmetic) on an n_tokens sample; returns (tokens/s, seconds per pass,
    experts touched)."""
    from oracle import moe_oracle as O
    xh, wrh, bh, W, sh = oracle_sample(cfg, n_tokens, device)
    scfg = cfg.scaled(T=n_tokens)
    w = [(lambda e, k=k: O.from_bf16(W[e][k])) for k in range(3)]

    def one():
        O.forward(scfg, xh, wrh, bh, w[0], w[1], w[2], shared=sh)

    for _ in range(warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(steps):
        one()
    dt = (time.perf_counter() - t0) / max(steps, 1)
    return n_tokens / dt, dt, len(W)


def time_oracle_backward(cfg, n_tokens, device):
    """The oracle's backward with every weight gradient (fp64, as it stands)
    on an n_tokens sample; returns (tokens/s, seconds per pass, experts
    touched)."""
    from oracle import moe_oracle as O
    xh, wrh, bh, W, sh = oracle_sample(cfg, n_tokens, device)
    dyh = O.from_bf16(synth.gen_dy(cfg, device)[:n_tokens])
    scfg = cfg.scaled(T=n_tokens)
    w = [(lambda e, k=k: O.from_bf16(W[e][k])) for k in range(3)]
    t0 = time.perf_counter()
    O.backward(scfg, xh, wrh, bh, w[0], w[1], w[2], dyh, shared=sh, weight_grads=sorted(W))
    dt = time.perf_counter() - t0
    return n_tokens / dt, dt, len(W)


def _oracle_note(cfg, n_tokens, n_experts):
    return (f"oracle forward (fp64; weights of the {n_experts} experts the sample touches "
            f"quantized inside each pass, as the oracle stands) on the first {n_tokens} tokens of "
            f"the {cfg.name} batch, per pass")


def run_reference(args, cfg):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    # the whole --steps K --warmup W run stays within a few minutes
    n = args.ref_tokens or oracle_tokens(cfg, 150.0 / max(1, args.steps + args.warmup), dev)
    tps, dt, ne = time_oracle(cfg, n, args.steps, args.warmup, dev)
    line = {
        "impl": "reference", "metric": METRIC, "value": tps, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": _workload(cfg, "host oracle; no GPU kernels"),
        "cpu_baseline": {"value": tps, "unit": "tokens/s", "cores": _host_cores(), "kind": "oracle",
                         "sample": _oracle_note(cfg, n, ne)},
        "e2e": {"value": tps, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

WEIGHT_BYTES = {"bf16": 2.0, "mxfp8": 1.0 + 1.0 / 32, "nvfp4": 0.5 + 1.0 / 16}  # per element
# Dense tensor peaks of the block-scaled types, TFLOP/s: library GEMMs at 8192^3
# timed on one B200 by `bench.py --tensor-peaks` (burst); bf16 comes from the
# driver's measurement (MEASURED_PEAKS.json).
TENSOR_PEAK = {"mxfp8": 2834.6, "nvfp4": 6217.2}
# DRAM bytes (read + written) of one grouped-MLP call's fc1 and fc2 launches per
# algorithmic weight byte, from ncu dram__bytes_read.sum + dram__bytes_write.sum
# captures, keyed by workload, each with the hash of the kernel source it was
# taken on (kernel_source_hash): a ratio is reported only while the kernels
# are unchanged since its capture.  Workloads too large to capture whole were
# captured on fewer experts with the same tokens per expert; the ratio carries
# over per touched expert.
TRAFFIC_RATIO = {
    "dsv4_nvfp4_prefill_T8192": (1.066, "32a54879bb76cd88"),
    "mid_bf16_shared_T2048": (1.191, "32a54879bb76cd88"),
    "dsv4_bf16_T4096": (1.032, "dcc545b0947a04af"),
    "dsv3_mxfp8_shared_T4096": (1.080, "dcc545b0947a04af"),
    "dsv4_mxfp8_T4096": (1.018, "dcc545b0947a04af"),
    "dsv4_nvfp4_decode_T128": (1.010, "dcc545b0947a04af"),
    "dsv4_nvfp4_serve_T1024": (1.010, "dcc545b0947a04af"),
}


def kernel_source_hash():
    """Hash of the grouped-GEMM kernel source (the files its code is in)."""
    import hashlib
    h = hashlib.sha256()
    for f in ("grouped_gemm.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "mixture_experts_layer_grouped_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def graph_kernel_names(graph):
    """Names of the kernel nodes of a captured CUDA graph (one per launch), or
    None when the driver bindings cannot list them."""
    try:
        from cuda.bindings import driver as drv
        raw = graph.raw_cuda_graph()
        g = raw if isinstance(raw, drv.CUgraph) else drv.CUgraph(int(raw))
        err, _, n = drv.cuGraphGetNodes(g, 0)
        err, nodes, n = drv.cuGraphGetNodes(g, n)
        names = []
        for nd in nodes[:n]:
            err, t = drv.cuGraphNodeGetType(nd)
            if t != drv.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
                continue
            err, prm = drv.cuGraphKernelNodeGetParams(nd)
            err, name = drv.cuFuncGetName(prm.func)
            names.append(name.decode() if isinstance(name, bytes) else str(name))
        return names
    except Exception:
        return None


def grouped_mlp_algorithmic(cfg, touched):
    """Bytes and FLOPs the grouped MLP call cannot avoid: every touched routed
    expert's and the shared expert's weights read once; 6*H*I per row."""
    wbytes = int(WEIGHT_BYTES[cfg.dtype] * 3 * cfg.H * (touched * cfg.I + cfg.I_shared))
    flops = 6 * cfg.H * (cfg.T * cfg.top_k * cfg.I + cfg.T * cfg.I_shared)
    return wbytes, flops


def layer_algorithmic(cfg, touched):
    """Whole-layer algorithmic bytes / FLOPs: weights touched + shared + router,
    x in and y out (bf16)."""
    wb, fl = grouped_mlp_algorithmic(cfg, touched)
    b = wb + 2 * cfg.E * cfg.H + 2 * 2 * cfg.T * cfg.H
    f = fl + 2 * cfg.T * cfg.H * cfg.E
    return b, f


def prepare_streaming(M, cfg, c, dev):
    """Prepared weights, drawn and converted one expert at a time."""
    p = M.allocate_prepared_weights(c, dev)
    dst = M.binding.weights_struct(p)
    for e in range(cfg.E):
        M.moe_prepare_weights(c, 0, e, 1, *synth.gen_expert_weights(cfg, e, dev), dst)
    if cfg.I_shared:
        M.moe_prepare_weights(c, 1, 0, 1, *synth.gen_shared_weights(cfg, dev), dst)
    torch.cuda.synchronize()
    return p


def tensor_peaks(device="cuda"):
    """Dense library GEMM throughput on this GPU, 8192^3, burst (50 timed calls after
    5 untimed): bf16 (torch matmul), MXFP8 and NVFP4 (torch._scaled_mm with block
    scales; the scale values do not change the work).  The denominators of the
    block-scaled tensor fractions."""
    M = N = K = 8192
    res = {}

    def timeit(fn, iters=50):
        for _ in range(5):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return 2 * M * N * K / (e0.elapsed_time(e1) / iters * 1e-3) / 1e12

    def pad(v, m):
        return (v + m - 1) // m * m

    u8 = dict(dtype=torch.uint8, device=device)
    x = torch.randn(M, K, device=device, dtype=torch.bfloat16)
    y = torch.randn(K, N, device=device, dtype=torch.bfloat16)
    res["bf16_tflops"] = timeit(lambda: x @ y)
    a8 = torch.randn(M, K, device=device).to(torch.float8_e4m3fn)
    b8 = torch.randn(N, K, device=device).to(torch.float8_e4m3fn).t()
    s8a = torch.full((pad(M, 128) * pad(K // 32, 4),), 127, **u8).view(torch.float8_e8m0fnu)
    s8b = torch.full((pad(N, 128) * pad(K // 32, 4),), 127, **u8).view(torch.float8_e8m0fnu)
    res["mxfp8_tflops"] = timeit(lambda: torch._scaled_mm(a8, b8, s8a, s8b,
                                                          out_dtype=torch.bfloat16))
    a4 = torch.randint(0, 255, (M, K // 2), **u8).view(torch.float4_e2m1fn_x2)
    b4 = torch.randint(0, 255, (N, K // 2), **u8).view(torch.float4_e2m1fn_x2).t()
    s4a = torch.full((pad(M, 128) * pad(K // 16, 4),), 56, **u8).view(torch.float8_e4m3fn)
    s4b = torch.full((pad(N, 128) * pad(K // 16, 4),), 56, **u8).view(torch.float8_e4m3fn)
    res["nvfp4_tflops"] = timeit(lambda: torch._scaled_mm(a4, b4, s4a, s4b,
                                                          out_dtype=torch.bfloat16))
    return res


def backward_algorithmic(cfg, touched):
    """Bytes and FLOPs the backward cannot avoid: the touched experts', the
    shared expert's and the router's bf16 weights read once; their fp32
    gradients written once; x, dy and the saved rows and fc2 outputs read,
    dx written.  FLOPs: dh, dX and the three weight gradients, 12*H*I per
    routed row (the recomputation of a and u, 4*H*I more, is not counted)."""
    R = cfg.T * cfg.top_k
    w_el = 3 * cfg.H * (touched * cfg.I + cfg.I_shared) + cfg.E * cfg.H
    b = 2 * w_el + 4 * w_el + 2 * (3 * cfg.T * cfg.H + 2 * R * cfg.H)
    f = 12 * cfg.H * (R * cfg.I + cfg.T * cfg.I_shared) + 4 * cfg.T * cfg.H * cfg.E
    return b, f


def run_backward(args, cfg):
    """The backward of the bf16 layer (moe_backward: dx, router and weight
    gradients), one call per step, captured in a CUDA graph."""
    import mixture_experts_layer_grouped_b200 as M
    if cfg.dtype != "bf16":
        raise SystemExit("--backward: the backward is built for the bf16 layer")
    if cfg.pad_multiple % 64:
        cfg = cfg.scaled(pad_multiple=64)  # routed weight gradients read 64-row steps
    ws_n, rank, local = _dist()
    if ws_n > 1:
        raise SystemExit("--backward runs on one GPU")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    c = M.config_from_shape(cfg)
    x, w_r, bias = replica_inputs(cfg, rank, dev)
    prepared = prepare_streaming(M, cfg, c, dev)
    sz = M.moe_backward_weights_size(c)
    bw = {k: (torch.empty(v, dtype=torch.uint8, device=dev) if v else None)
          for k, v in sz.items()}
    for e in range(cfg.E):
        M.moe_prepare_backward_weights(c, 0, e, 1, *synth.gen_expert_weights(cfg, e, dev), None,
                                       bw)
    sh = synth.gen_shared_weights(cfg, dev) or (None, None, None)
    M.moe_prepare_backward_weights(c, 1, 0, 1, *sh, w_r, bw)
    # the forward's saved state, through the step calls
    nbytes, r_cap = M.moe_workspace_size(c)
    wsf = M.binding.new_workspace(nbytes, dev)
    i32 = dict(dtype=torch.int32, device=dev)
    T, H, E, I, Is, k = cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k
    sv = {"x": x, "logits": torch.empty(T, E, dtype=torch.float32, device=dev),
          "topk_idx": torch.empty(T, k, **i32),
          "topk_w": torch.empty(T, k, dtype=torch.float32, device=dev),
          "counts": torch.empty(E, **i32), "offsets": torch.empty(E + 1, **i32),
          "row_token": torch.empty(r_cap, **i32), "token_row": torch.empty(T * k, **i32),
          "rows": torch.empty(r_cap, H, dtype=torch.bfloat16, device=dev),
          "out_rows": torch.empty(r_cap, H, dtype=torch.bfloat16, device=dev)}
    M.moe_route(c, x, w_r, bias, sv["topk_idx"], sv["topk_w"], wsf, logits_out=sv["logits"])
    M.moe_permute(c, sv["topk_idx"], x, sv["counts"], sv["offsets"], sv["row_token"],
                  sv["token_row"], sv["rows"], wsf)
    shared_out = torch.empty(T, H, dtype=torch.bfloat16, device=dev) if Is else None
    M.moe_grouped_mlp(c, prepared, sv["rows"], sv["counts"], sv["offsets"], sv["out_rows"], wsf,
                      x=x, shared_out=shared_out)
    dy = synth.gen_dy(cfg, dev)
    dx = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    dlogits = torch.empty(T, E, dtype=torch.float32, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    grads = {"dw1": torch.empty(E, I, H, **f32), "dw3": torch.empty(E, I, H, **f32),
             "dw2": torch.empty(E, H, I, **f32), "dw_router": torch.empty(E, H, **f32)}
    if Is:
        grads.update(dws1=torch.empty(Is, H, **f32), dws3=torch.empty(Is, H, **f32),
                     dws2=torch.empty(H, Is, **f32))
    wsb = M.binding.new_workspace(M.moe_backward_workspace_size(c), dev)
    stream = torch.cuda.current_stream()

    def call(with_grads):
        M.moe_backward(c, prepared, bw, sv, dy, dx, wsb, dlogits=dlogits,
                       grads=grads if with_grads else None)

    def timed(with_grads):
        for _ in range(args.warmup):
            torch.cuda.nvtx.range_push("moe_backward")
            call(with_grads)
            torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(graph):
            call(with_grads)
        graph.instantiate()
        names = graph_kernel_names(graph)
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize()
        if M.moe_get_device_status(wsb) != 0:
            raise RuntimeError("device status set in the backward")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / args.steps, names

    clk = ClockSampler(local).__enter__()
    t_soak = time.time()
    ms_dgrad, _ = timed(False)
    ms, names = timed(True)
    t_end = time.time()
    clk.__exit__(None, None, None)
    touched = int((sv["counts"] > 0).sum().item())
    hbm, tf_burst, tf_sus, peak_kind = _peaks()
    b, f = backward_algorithmic(cfg, touched)
    gbs = b / (ms * 1e-3) / 1e9
    tfs = f / (ms * 1e-3) / 1e12
    roof_ms = max(b / (hbm * 1e9), f / (tf_burst * 1e12)) * 1e3
    # the weight-gradient kernel alone, by difference: the fp32 gradients
    # written and its operands read once per expert
    w_el = 3 * H * (touched * I + Is) + E * H
    # operands per routed row: [da | du] (2I) and X (H), dO (H) and h (I); per
    # token: the shared expert's (3 I_s + 2H when present) and the router's
    # bf16 dlogits (E) and x (H)
    wg_bytes = 4 * w_el + 2 * (T * k * (3 * I + 2 * H) + T * ((3 * Is + 2 * H if Is else 0) + E + H))
    wg_ms = ms - ms_dgrad
    clocks = clk.summary(t_soak, t_end)
    cpu = None
    if not args.no_cpu_baseline:
        n = args.ref_tokens
        if not n:  # about 15 s of host work: a one-token pass sizes the sample
            _, t1, _ = time_oracle_backward(cfg, 1, dev)
            n = max(1, min(32, int(15.0 / max(t1, 1e-6))))
        tps, dt, ne = time_oracle_backward(cfg, n, dev)
        cpu = {"value": tps, "unit": "tokens/s", "cores": _host_cores(), "kind": "oracle",
               "sample": f"oracle backward (fp64, every weight gradient of the {ne} experts "
                         f"the sample touches) on the first {n} tokens of the {cfg.name} "
                         f"batch, one pass of {dt:.1f} s"}
    line = {
        "metric": "MoE layer bwd (dgrad + wgrad) tokens/s at 1 B200",
        "value": T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 (fp32 accumulation, fp32 weight gradients)",
        "data": "synthetic (seeded normal inputs, dy and random-init weights of the workload)",
        "config": dict(_workload(cfg, "inputs larger than L2: %.0f MB of bf16 weights read and "
                                 "%.0f MB of fp32 gradients written per step"
                                 % (2 * w_el / 1e6, 4 * w_el / 1e6)),
                       workload=f"routed MoE layer backward, {cfg.name}",
                       launch="CUDA graph of one moe_backward call", parallelism="replicas1"),
        "roofline": {"bound": "hbm" if b / (hbm * 1e9) >= f / (tf_burst * 1e12) else "tensor",
                     "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": roof_ms / ms,
                     "kernel": "the whole moe_backward call (its roofline time = max of "
                               "algorithmic bytes / HBM and FLOPs / bf16 peak)",
                     "algorithmic_bytes": b, "flops": f, "tensor_tflops": tfs,
                     "roofline_ms": roof_ms, "traffic": None,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, bf16_tflops)"},
        "wgrad": {"ms": wg_ms, "bytes": wg_bytes, "gbs": wg_bytes / (wg_ms * 1e-3) / 1e9,
                  "frac": wg_bytes / (wg_ms * 1e-3) / 1e9 / hbm,
                  "how": "moe_backward with weight gradients minus without"},
        "dgrad_ms": ms_dgrad,
        "cpu_baseline": cpu,
        "gpu_launches": len(names) * args.steps if names is not None else None,
        "gpu_launches_per_step": names,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples": clocks["samples"]},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, cfg):
    import mixture_experts_layer_grouped_b200 as M
    ws_n, rank, local = _dist()
    torch.cuda.set_device(local)
    dist = None
    if ws_n > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    c = M.config_from_shape(cfg)
    d = dict(zip(("x", "w_router", "bias"), replica_inputs(cfg, rank, dev)))
    layer = M.MoELayer(c, prepare_streaming(M, cfg, c, dev), d["w_router"], d["bias"],
                       prepared=True)
    x, y = d["x"], torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    clk = ClockSampler(local).__enter__()
    # warm-up (eager; an NVTX range per forward lets a profiler pick out the
    # kernels of one call), then capture one forward into a CUDA graph
    for _ in range(args.warmup):
        torch.cuda.nvtx.range_push("moe_forward")
        layer.forward(x, out=y)
        torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(graph):
        layer.forward(x, out=y)
    graph.instantiate()
    launches = graph_kernel_names(graph)  # the library's kernels in one forward
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    status = layer.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after warm-up")

    # untimed soak so the clock sampler sees the GPU under this load
    t_soak = time.time()
    while time.time() - t_soak < args.soak_s:
        for _ in range(20):
            graph.replay()
        torch.cuda.synchronize()

    # ---- timed region: device-resident inputs, graph replay
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    t_timed_end = time.time()
    clk.__exit__(None, None, None)
    ms = ev0.elapsed_time(ev1) / args.steps
    barrier()
    ms_max = max_over_ranks(ms, dist, dev)
    value = job_tokens_per_s(cfg.T, ws_n, ms_max)

    # ---- e2e: host (pinned) x and y through the same C call, which copies x
    # in and y out on its stream.  Two calls are in flight, on two streams with
    # a workspace each, so one call's copies overlap the other's kernels (the
    # way a serving loop feeds the layer); every step still moves its own x in
    # and y out.  The one-stream figure (copies never overlapped) is reported
    # beside it.
    layers = [layer, M.MoELayer(c, layer.weights, d["w_router"], d["bias"], prepared=True)]
    streams = [torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    x_h = [x.cpu().pin_memory() for _ in range(2)]
    y_h = [torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]

    def e2e_loop(n, two):
        for i in range(n):
            j = i % 2 if two else 0
            layers[j].forward(x_h[j], out=y_h[j], stream=streams[j])

    def e2e_timed(two):
        e2e_loop(args.warmup, two)
        barrier()
        ev0.record(stream)
        for st in streams:
            st.wait_event(ev0)
        e2e_loop(args.steps, two)
        for st in streams:
            stream.wait_stream(st)
        ev1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(ev0.elapsed_time(ev1) / args.steps, dist, dev)

    e2e_ms_serial = e2e_timed(False)
    e2e_ms = e2e_timed(True)
    for lay in layers:
        if lay.device_status() != 0:
            raise RuntimeError("device status set in the end-to-end loop")
    e2e_value = job_tokens_per_s(cfg.T, ws_n, e2e_ms)

    # ---- roofline of the dominant call (grouped MLP: fc1+SwiGLU and fc2)
    nbytes, r_cap = M.moe_workspace_size(c)
    wsp = M.binding.new_workspace(nbytes, dev)
    i32 = dict(dtype=torch.int32, device=dev)
    logits = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev)
    idx = torch.empty(cfg.T, cfg.top_k, **i32)
    tw = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device=dev)
    counts, offsets = torch.empty(cfg.E, **i32), torch.empty(cfg.E + 1, **i32)
    row_token, token_row = torch.empty(r_cap, **i32), torch.empty(cfg.T * cfg.top_k, **i32)
    mx = cfg.dtype != "bf16"  # block-scaled: quantize x, permute codes and scales
    rb = {"bf16": 2 * cfg.H, "mxfp8": cfg.H, "nvfp4": cfg.H // 2}[cfg.dtype]
    rows = torch.empty(r_cap, rb, dtype=torch.uint8, device=dev)
    xc = xs = rows_sf = xg = None
    if mx:
        xc = torch.empty(cfg.T, rb, dtype=torch.uint8, device=dev)
        xs = torch.zeros(M.scale_bytes(cfg.T, cfg.H, cfg.dtype), dtype=torch.uint8, device=dev)
        rows_sf = torch.zeros(M.scale_bytes(r_cap, cfg.H, cfg.dtype), dtype=torch.uint8,
                              device=dev)
        xg = torch.empty(1, dtype=torch.float32, device=dev)
    out_rows = torch.empty(r_cap, cfg.H, dtype=torch.bfloat16, device=dev)
    shared_out = (torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device=dev)
                  if cfg.I_shared else None)
    steps_ms = {"route": [], "quantize": [], "permute": [], "grouped_mlp": [], "combine": []}
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for it in range(args.warmup + args.steps):
        torch.cuda.nvtx.range_push("moe_step")
        evs[0].record(stream)
        M.moe_route(c, x, d["w_router"], d["bias"], idx, tw, wsp, logits_out=logits)
        evs[1].record(stream)
        if mx:
            M.moe_quantize(cfg.dtype, x, xc, xs, global_scale=xg)
        evs[2].record(stream)
        M.moe_permute(c, idx, xc if mx else x, counts, offsets, row_token, token_row, rows, wsp,
                      src_scales=xs, dst_scales=rows_sf)
        evs[3].record(stream)
        M.moe_grouped_mlp(c, layer.weights, rows, counts, offsets, out_rows, wsp,
                          x=xc if mx else x, shared_out=shared_out, row_scales=rows_sf,
                          x_scales=xs, x_global=xg)
        evs[4].record(stream)
        M.moe_combine(c, out_rows, token_row, tw, y, shared_out=shared_out)
        evs[5].record(stream)
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        if it >= args.warmup:
            for i, k in enumerate(steps_ms):
                steps_ms[k].append(evs[i].elapsed_time(evs[i + 1]))
    touched = int((counts > 0).sum().item())
    mlp_ms = statistics.mean(steps_ms["grouped_mlp"])
    wbytes, flops = grouped_mlp_algorithmic(cfg, touched)
    hbm, tf_burst, tf_sus, peak_kind = _peaks()
    # a contraction takes the peak of its own dtype
    tf_dtype = TENSOR_PEAK.get(cfg.dtype, tf_burst)
    achieved_gbs = wbytes / (mlp_ms * 1e-3) / 1e9
    lb, lf = layer_algorithmic(cfg, touched)
    roof_ms = max(lb / (hbm * 1e9), lf / (tf_dtype * 1e12)) * 1e3

    if dist is not None:
        dist.barrier()
        del graph
        dist.destroy_process_group()
    if rank != 0:
        return

    cpu = None
    if ws_n == 1 and not args.no_cpu_baseline:
        n = args.ref_tokens or oracle_tokens(cfg, 20.0, dev)
        tps, _, ne = time_oracle(cfg, n, 1, 0, dev)
        cpu = {"value": tps, "unit": "tokens/s", "cores": _host_cores(), "kind": "oracle",
               "sample": _oracle_note(cfg, n, ne) + ", one pass"}
    src_hash = kernel_source_hash()
    tr = TRAFFIC_RATIO.get(cfg.name)
    traffic = tr[0] * wbytes if tr is not None and tr[1] == src_hash else None
    clocks = clk.summary(t_soak, t_timed_end)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": {"bf16": "bf16", "mxfp8": "e4m3+e8m0 (mxfp8), fp32 acc",
                  "nvfp4": "e2m1+ue4m3+fp32 global (nvfp4), fp32 acc"}[cfg.dtype],
        "data": "synthetic (seeded normal inputs and random-init weights of the workload)",
        "config": dict(_workload(cfg, "inputs larger than L2: %.0f MB of expert weights per step"
                                 % (WEIGHT_BYTES[cfg.dtype] * 3 * cfg.H * cfg.I * cfg.E / 1e6)),
                       launch="CUDA graph of the one-call forward", parallelism=f"replicas{ws_n}"),
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm, "unit": "GB/s",
                     "frac": achieved_gbs / hbm,
                     "traffic": traffic,
                     "traffic_source": ("estimate, not counted in this run: the ratio of "
                                        "ncu dram__bytes_read.sum + dram__bytes_write.sum of "
                                        "the fc1 and fc2 launches to their algorithmic weight "
                                        f"bytes, captured on kernel source {src_hash}, x this "
                                        "call's algorithmic bytes" if traffic is not None else
                                        f"no ncu capture of kernel source {src_hash}"),
                     "kernel": "moe_grouped_mlp (fc1+SwiGLU and fc2 tcgen05 kernels)",
                     "algorithmic_bytes_per_launch": wbytes, "ms_per_launch": mlp_ms,
                     "tensor_tflops": flops / (mlp_ms * 1e-3) / 1e12,
                     "tensor_frac": flops / (mlp_ms * 1e-3) / 1e12 / tf_dtype,
                     "tensor_peak_tflops": tf_dtype,
                     "peak_source": (f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs; tensor: " +
                                     ("bf16_tflops" if cfg.dtype == "bf16" else
                                      f"{cfg.dtype} library GEMM measured by bench.py "
                                      "--tensor-peaks") + ")")},
        "layer_roofline": {"ms": roof_ms, "frac": roof_ms / ms_max,
                           "bytes": lb, "flops": lf, "experts_touched": touched},
        "step_ms": {k: statistics.mean(v) for k, v in steps_ms.items()},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": cfg.T * cfg.H * 2, "d2h_bytes_per_step": cfg.T * cfg.H * 2,
                "mode": "moe_forward on pinned host x / y (copies inside the call), two calls in "
                        "flight on two streams",
                "one_stream_value": job_tokens_per_s(cfg.T, ws_n, e2e_ms_serial)},
        "gpu_launches": (len(launches) * args.steps if launches is not None else None),
        "gpu_launches_per_step": launches,
        "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                   "reasons": clocks["reasons"], "samples": clocks["samples"]},
        "gemm_pairs": os.environ.get("MOE_GEMM_PAIRS", "1") != "0",
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=BENCH_CONFIG, choices=sorted(synth.CONFIGS))
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="tokens in the oracle's sample (0: sized to a time budget)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--experts", type=int, default=0,
                    help="profiling only: scale the workload to this many experts, keeping "
                         "the rows per expert (T scales with E)")
    ap.add_argument("--tokens", type=int, default=0,
                    help="profiling only: run this many tokens (with --experts, keeps the "
                         "token-side kernels at full size while the weights stay small)")
    ap.add_argument("--tensor-peaks", action="store_true",
                    help="measure the dense bf16 / MXFP8 / NVFP4 library GEMM throughput")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward of the bf16 layer (moe_backward) instead")
    ap.add_argument("--soak-s", type=float, default=1.5,
                    help="untimed graph replays before the timed region (clock sampling)")
    args = ap.parse_args()
    cfg = synth.get_config(args.config)
    if args.experts:
        t = args.tokens or max(1, round(cfg.T * args.experts / cfg.E))
        cfg = cfg.scaled(E=args.experts, T=t, name=f"{cfg.name}_E{args.experts}_T{t}")
    elif args.tokens:
        cfg = cfg.scaled(T=args.tokens, name=f"{cfg.name}_T{args.tokens}")
    if args.tensor_peaks:
        print(json.dumps(tensor_peaks()), flush=True)
    elif args.backward:
        run_backward(args, cfg)
    elif args.impl == "reference":
        run_reference(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
