"""Seeded synthetic inputs for the routed MoE layer forward.

This package holds workload shapes and random-number draws only.  It contains
none of the layer's arithmetic, so that both the CUDA library and the CPU oracle
can consume the same bytes without sharing any code of the method.
"""

from .configs import CONFIGS, MoEShape, get_config  # noqa: F401
from .inputs import (  # noqa: F401
    gen_x,
    gen_dy,
    gen_router,
    gen_expert_weights,
    gen_shared_weights,
    gen_all,
)
