"""Padding-free MoE layer on B200 (sm_100a): C-ABI library + thin Python binding.

``padding_free_moe_b200._lib`` mirrors the C entry points of ``include/pfmoe.h``
one to one; ``padding_free_moe_b200.layer.PFTMoELayer`` owns the device buffers
of one layer and calls them in order (forward, backward, RBD plan).
"""
from ._lib import (  # noqa: F401
    PFMOE_BF16, PFMOE_F32, PFMoEError, TILE_ROWS, dtype_code, lib, moe_abi_version, moe_backward,
    moe_backward_workspace_size, moe_combine, moe_dispatch, moe_expert_ffn, moe_last_error, moe_profile_enable,
    moe_profile_read, moe_profile_reset, moe_route, moe_route_workspace_size, pft_build, pft_build_workspace_size, rbd_plan,
    rbd_plan_workspace_size,
)

__version__ = "0.1.0"
