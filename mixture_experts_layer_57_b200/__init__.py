"""Single-GPU Mixture-of-Experts FFN layer forward pass for B200 (sm_100a).

router (fp32 logits, softmax, top-k, load-balance statistics) -> capacity-limited first-come
dispatch into an expert-major packed buffer -> per-expert two-layer GeLU FFN on tcgen05 tensor
cores -> gate-weighted combine with the residual and the optional PR-MoE dense MLP branch.

The computation lives in ``libmoe.so`` (C ABI, ``include/moe.h``); :mod:`.moe` is its ctypes
binding. Build with ``python -m mixture_experts_layer_57_b200.build``.
"""
from . import moe  # noqa: F401
from .moe import (MoEError, moe_capacity, moe_combine, moe_dispatch, moe_expert_ffn,  # noqa: F401
                  moe_get_device_error, moe_layer_forward, moe_layer_workspace_bytes,
                  moe_packed_rows_max, moe_router_topk, moe_workspace_reset, layer_args)
