"""B200 (sm_100a) MoE FFN layer: the dots.llm1 fine-grained MoE hot path.

The compute lives in ``libmoe.so`` (hand-written CUDA, C ABI declared in
``include/moe.h``).  This package only marshals arguments to it
(``grouped_gemm_fp32_b200._lib``) and sequences the calls of one layer over
caller-owned torch buffers (``grouped_gemm_fp32_b200.layer``).  There is no
CPU or PyTorch fallback: without the built library every call raises.
"""
from ._lib import (MOE_GEMM1, MOE_GEMM2, MoeDims, MoeError, grouped_gemm_bwd_dw,  # noqa: F401
                   grouped_gemm_bwd_dw1_gather, grouped_gemm_bwd_dx, grouped_gemm_fwd,
                   grouped_gemm_fwd_gather, grouped_gemm_set_groups, lib_path,
                   load, moe_bias_update, moe_combine, moe_combine_bwd, moe_combine_f32,
                   moe_combine_split,
                   moe_gate_topk, moe_get_device_status, moe_last_cuda_error, moe_permute_align,
                   moe_permute_align_static, moe_router_bwd, moe_router_bwd_seqbal,
                   moe_rows_routed, moe_rows_total, moe_seq_balance_loss, moe_status_string,
                   moe_workspace_size, MOE_EP_MAX_WORLD, MOE_EP_WAIT_DX, MOE_EP_WAIT_Y,
                   MoeEpPeers, grouped_gemm_bwd_dx_ep, grouped_gemm_fwd_ep, moe_ep_combine_bwd,
                   moe_ep_dispatch, moe_ep_plan, moe_ep_wait, moe_ep_workspace_size,
                   moe_ep_zero_pads)
