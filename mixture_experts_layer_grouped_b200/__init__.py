"""Routed Mixture-of-Experts layer on one B200 (sm_100a): the forward, and the
backward of the bf16 layer.

A thin ctypes binding over ``libmoe_b200.so``: the functions below marshal
torch tensors into device pointers and call the C ABI of include/moe_b200.h
with the same names.  Every step runs in the library's CUDA kernels; there is
no fallback path, and importing the binding fails loudly when the library has
not been built.
"""

from .binding import (  # noqa: F401
    MoEConfig,
    MoEWeights,
    MoEError,
    config_from_shape,
    lib,
    moe_workspace_size,
    moe_forward_workspace_size,
    moe_route,
    moe_permute,
    moe_permute_noalloc,
    moe_grouped_mlp,
    moe_combine,
    moe_forward,
    moe_get_device_status,
    moe_prepared_weights_size,
    moe_prepare_weights,
    moe_quantize,
    scale_bytes,
    prepare_weights,
    allocate_prepared_weights,
    MoELayer,
    MoETrainLayer,
    MoEBwdWeights,
    MoEFwdSaved,
    MoEWeightGrads,
    moe_backward_weights_size,
    moe_prepare_backward_weights,
    prepare_backward_weights,
    moe_backward_workspace_size,
    moe_backward,
)
