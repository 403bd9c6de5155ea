"""Helper for the GPU failure-path test: a forward whose fc2 chunk waits can
never be satisfied (MOE_TEST_FC2_NEVER_READY=1 for that call only), then a
normal forward in the same process.  Prints the two device status codes and
whether the second output equals a fresh reference run's:
python tests/timeout_once.py <workload>"""

import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import synth  # noqa: E402
from moe_testlib import weights_dict  # noqa: E402


def main():
    import mixture_experts_layer_grouped_b200 as M
    cfg = synth.get_config(sys.argv[1])
    d = synth.gen_all(cfg, "cuda")
    layer = M.MoELayer(M.config_from_shape(cfg), weights_dict(d), d["w_router"], d["bias"])
    y_ref = layer.forward(d["x"]).clone()
    torch.cuda.synchronize()
    s0 = layer.device_status()
    os.environ["MOE_TEST_FC2_NEVER_READY"] = "1"
    layer.forward(d["x"])
    torch.cuda.synchronize()
    s1 = layer.device_status()
    del os.environ["MOE_TEST_FC2_NEVER_READY"]
    y = layer.forward(d["x"])
    torch.cuda.synchronize()
    s2 = layer.device_status()
    same = bool(torch.equal(y.view(torch.int16), y_ref.view(torch.int16)))
    print(f"status {s0} {s1} {s2} same {int(same)}")


if __name__ == "__main__":
    main()
