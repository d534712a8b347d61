"""Routing-weighted SiTU-GLU for NVIDIA B200 (sm_100a).

    T_g = beta * tanh(G / beta) * sigmoid(G)
    T_u = linear_beta * tanh(U / linear_beta)     (U when linear_beta is None)
    Y   = T_g * T_u * routing_weight

over gate_up[..., 2I] = [G | U], with the fused analytic backward.  The work
runs in the hand-written CUDA kernels of libsitu_glu.so behind the C ABI in
include/situ_glu.h; this package only marshals torch tensors into it.
"""
from . import abi, distributed
from .host_pipeline import HostPipeline
from .abi import NativeLibraryError, SituError
from .functional import (
    DEFAULT_BETA,
    apply_attn_res,
    attn_res_core,
    DEFAULT_LINEAR_BETA,
    WeightedSiTUFunction,
    situ_glu_bwd,
    situ_glu_bwd_mxfp8,
    situ_glu_fc1_fwd,
    situ_glu_fc2_dgrad_bwd,
    situ_glu_fwd,
    situ_glu_fwd_mxfp8,
    situ_glu_fwd_nvfp4,
    situ_glu_bwd_nvfp4,
    situlu,
    weighted_situ,
)

__all__ = [
    "abi",
    "distributed",
    "HostPipeline",
    "NativeLibraryError",
    "SituError",
    "DEFAULT_BETA",
    "DEFAULT_LINEAR_BETA",
    "apply_attn_res",
    "attn_res_core",
    "WeightedSiTUFunction",
    "situ_glu_fwd",
    "situ_glu_bwd",
    "situ_glu_fwd_mxfp8",
    "situ_glu_bwd_mxfp8",
    "situ_glu_fwd_nvfp4",
    "situ_glu_bwd_nvfp4",
    "situ_glu_fc1_fwd",
    "situ_glu_fc2_dgrad_bwd",
    "situlu",
    "weighted_situ",
]
