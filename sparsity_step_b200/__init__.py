"""B200-native (sm_100a) Sparse-BitNet BitLinear path.

The functions below are thin bindings of the C ABI in include/bitlinear.h; the
library libbitlinear.so is loaded on first use and its absence is an error.
"""
from .bitlinear import (  # noqa: F401
    BL_GRADW_DEQUANT_X,
    BL_OUT_BF16,
    BL_OUT_F32,
    bitlinear_abi_version,
    bitlinear_act_quant,
    bitlinear_bwd,
    bitlinear_bwd_workspace_size,
    bitlinear_device_status,
    bitlinear_fwd,
    bitlinear_fwd_grouped,
    bitlinear_grad_x_i8,
    bitlinear_grad_x_i8_workspace_size,
    bitlinear_mask_threshold_hist,
    bitlinear_quant_mask,
    bitlinear_quant_mask_noalloc,
    bitlinear_quant_mask_status,
    bitlinear_quant_mask_workspace_size,
    bitlinear_sgd_quant_mask,
    bitlinear_grad_w_grouped,
    sp_meta_shape,
)
