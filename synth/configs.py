"""Workload shapes of the routed MoE layer forward.

The workloads are the routed-MoE shapes the method is exercised on:

* a tiny bf16 layer (T=64, H=256, I=128, E=16, groups 4/2, top-4);
* a mid-size bf16 layer with a shared expert and a skewed router
  (T=2048, H=2048, I=1024, E=64, groups 8/4, top-6, shared I=1024);
* the DeepSeek-V4 routed-expert geometry 4096/2048/top-6/E=256 in bf16
  (aiconfigurator issue "DeepSeek-V4 support on trtllm", per-op status table,
  moe row);
* DeepSeek-V3 dims with MXFP8 and a shared expert (TransformerEngine PR
  "DeepSeekV3Layer", Performance section: DeepSeek-V3 dims, top-k 8, MXFP8);
* the DeepSeek-V4 geometry 7168/3072/top-6/E=384 in NVFP4 W4A4 (sglang PR
  "Mistral Large 3 NVFP4 TRTLLM MoE support", Modifications: W4A4 NVFP4), at a
  decode size (T=128) and a prefill size (T=8192);
* and for serving, the same geometry at a batch between those (T=1024, NVFP4)
  and in MXFP8 (T=4096).

``pad_multiple`` is the row multiple each expert segment is padded to in the
expert-major layout: 64 for the block-scaled paths (whose scale chunks the
GEMM addresses in 64-row steps), 8 for bf16.
"""

from dataclasses import dataclass, field, asdict


@dataclass(frozen=True)
class MoEShape:
    name: str
    T: int
    H: int
    I: int
    E: int
    n_group: int
    topk_group: int
    top_k: int
    rsf: float
    I_shared: int
    dtype: str  # "bf16" | "mxfp8" | "nvfp4"
    pad_multiple: int
    router_std: float  # std of W_r entries; <= 0 means 1/sqrt(H)
    skew_experts: int = 0  # number of experts whose router rows are scaled
    skew_factor: float = 1.0
    bias_range: float = 0.1
    seed: int = 0

    @property
    def R(self) -> int:
        return self.T * self.top_k

    @property
    def r_cap(self) -> int:
        """Upper bound on the padded expert-major row count."""
        P = self.pad_multiple
        r = self.T * self.top_k + self.E * (P - 1)
        return (r + P - 1) // P * P

    def scaled(self, **kw) -> "MoEShape":
        d = asdict(self)
        d.update(kw)
        return MoEShape(**d)


CONFIGS = {
    "tiny_bf16_T64": MoEShape(
        name="tiny_bf16_T64", T=64, H=256, I=128, E=16, n_group=4, topk_group=2,
        top_k=4, rsf=2.5, I_shared=0, dtype="bf16", pad_multiple=8, router_std=0.02),
    "mid_bf16_shared_T2048": MoEShape(
        name="mid_bf16_shared_T2048", T=2048, H=2048, I=1024, E=64, n_group=8,
        topk_group=4, top_k=6, rsf=2.5, I_shared=1024, dtype="bf16", pad_multiple=8,
        router_std=0.02, skew_experts=8, skew_factor=3.0),
    "dsv4_bf16_T4096": MoEShape(
        name="dsv4_bf16_T4096", T=4096, H=4096, I=2048, E=256, n_group=8,
        topk_group=4, top_k=6, rsf=2.5, I_shared=0, dtype="bf16", pad_multiple=8,
        router_std=-1.0),
    "dsv3_mxfp8_shared_T4096": MoEShape(
        name="dsv3_mxfp8_shared_T4096", T=4096, H=7168, I=2048, E=256, n_group=8,
        topk_group=4, top_k=8, rsf=2.5, I_shared=2048, dtype="mxfp8",
        pad_multiple=64, router_std=-1.0),
    "dsv4_nvfp4_decode_T128": MoEShape(
        name="dsv4_nvfp4_decode_T128", T=128, H=7168, I=3072, E=384, n_group=8,
        topk_group=4, top_k=6, rsf=2.5, I_shared=0, dtype="nvfp4",
        pad_multiple=64, router_std=-1.0),
    "dsv4_nvfp4_prefill_T8192": MoEShape(
        name="dsv4_nvfp4_prefill_T8192", T=8192, H=7168, I=3072, E=384, n_group=8,
        topk_group=4, top_k=6, rsf=2.5, I_shared=0, dtype="nvfp4",
        pad_multiple=64, router_std=-1.0),
    # serving sizes of the same geometry: a batch between the decode and
    # prefill sizes (16 routed rows per expert on average), and the MXFP8 form
    "dsv4_nvfp4_serve_T1024": MoEShape(
        name="dsv4_nvfp4_serve_T1024", T=1024, H=7168, I=3072, E=384, n_group=8,
        topk_group=4, top_k=6, rsf=2.5, I_shared=0, dtype="nvfp4",
        pad_multiple=64, router_std=-1.0),
    "dsv4_mxfp8_T4096": MoEShape(
        name="dsv4_mxfp8_T4096", T=4096, H=7168, I=3072, E=384, n_group=8,
        topk_group=4, top_k=6, rsf=2.5, I_shared=0, dtype="mxfp8",
        pad_multiple=64, router_std=-1.0),
}

# The workload the throughput benchmark times by default: the largest one that
# fits one GPU (DeepSeek-V4 geometry, NVFP4 W4A4, prefill batch of 8192 tokens).
BENCH_CONFIG = "dsv4_nvfp4_prefill_T8192"


def get_config(name: str) -> MoEShape:
    return CONFIGS[name]
