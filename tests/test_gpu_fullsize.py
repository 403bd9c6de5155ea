"""Every workload at its full size through the C ABI, against the oracle
(TransformerEngine PR "DeepSeekV3Layer", Description, DeepSeekV3MoE bullet;
sglang PR "Mistral Large 3 NVFP4 TRTLLM MoE support", Modifications: W4A4
NVFP4; aiconfigurator issue "DeepSeek-V4 support on trtllm", moe row).

Each layer runs whole on the GPU through the step calls, with the weights
prepared one expert at a time; the one-call forward must give the same bits.
The oracle then checks, from its own fp64 router logits:
  * the routing of every token (indices bit-exact, gates within 1e-6 * rsf);
  * whole experts -- the most loaded one and seven seeded others -- their
    row maps and every fc2 output row (relative Frobenius per expert);
  * 32 tokens end to end (picked so that they share experts, which bounds the
    oracle's per-expert work), relative Frobenius over the sample.
Tolerances: 1e-2 for bf16, 2e-2 for MXFP8 / NVFP4.
"""

import pytest
import torch

import synth
from moe_testlib import check_full_size, prepare_streaming, run_layer_steps

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = ["mid_bf16_shared_T2048", "dsv4_bf16_T4096", "dsv3_mxfp8_shared_T4096",
        "dsv4_mxfp8_T4096", "dsv4_nvfp4_decode_T128", "dsv4_nvfp4_serve_T1024",
        "dsv4_nvfp4_prefill_T8192"]


@pytest.fixture(scope="module")
def M():
    assert torch.cuda.is_available()
    import mixture_experts_layer_grouped_b200 as M
    M.lib()
    return M


@pytest.mark.parametrize("name", FULL)
def test_full_size_layer(M, name):
    cfg = synth.get_config(name)
    x = synth.gen_x(cfg, "cuda")
    w_r, bias = synth.gen_router(cfg, "cuda")
    p = prepare_streaming(M, cfg)
    gpu = run_layer_steps(M, cfg, x, w_r, bias, p)
    assert gpu["status"] == 0
    layer = M.MoELayer(M.config_from_shape(cfg), p, w_r, bias, prepared=True)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    assert torch.equal(y.view(torch.int16), gpu["y"].view(torch.int16))
    del layer, y
    stats = check_full_size(cfg, x, w_r, bias, gpu)
    print(name, stats)
