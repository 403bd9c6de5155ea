"""Helper for the GPU tests: one forward of a named workload on its seeded
inputs, output saved with torch.save.  Run as a separate process so that
launch-time switches read from the environment (MOE_FC2_EARLY,
MOE_DYNAMIC_TILES, ...) take effect:  python tests/forward_once.py <workload> <out.pt>"""

import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import synth  # noqa: E402
from moe_testlib import weights_dict  # noqa: E402
import test_gpu_mxfp8  # noqa: E402
import test_gpu_nvfp4  # noqa: E402
import test_gpu_parity  # noqa: E402


def shape(name):
    if name in test_gpu_parity.EDGE:
        return test_gpu_parity.EDGE[name]
    if name in test_gpu_mxfp8.MX:
        return test_gpu_mxfp8.MX[name]
    if name in test_gpu_nvfp4.NV:
        return test_gpu_nvfp4.NV[name]
    return synth.get_config(name)


def main():
    import mixture_experts_layer_grouped_b200 as M
    cfg = shape(sys.argv[1])
    d = synth.gen_all(cfg, "cuda")
    layer = M.MoELayer(M.config_from_shape(cfg), weights_dict(d), d["w_router"], d["bias"])
    y = layer.forward(d["x"])
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    torch.save(y.cpu(), sys.argv[2])


if __name__ == "__main__":
    main()
