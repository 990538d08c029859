"""BitLinear W1.58A8 forward (BitNet b1.58) for B200 (sm_100a).

The computation lives in ``libbitlinear.so`` (hand-written CUDA behind the C ABI
of ``include/bitlinear.h``); this package is its Python binding, the
tensor-parallel FFN orchestration over torch.distributed in ``tp``, and the
seeded synthetic input generators in ``synth``.
"""
from .binding import (  # noqa: F401
    BL_BF16, BL_FP32, BL_GEMV_AUTO, BL_GEMV_LUT, BL_GEMV_STREAM, BL_GEMV_TENSOR, BL_OK, BL_OP_FFN, BL_OP_FORWARD, BL_OP_PACK,
    BL_OP_VALIDATE, LIB_PATH, SIGNATURES, STATUS_NAMES, BitLinearError, ffn, forward, forward_ex, forward_rowwise,
    gemv_kernel, get_device_error, lib, pack_weights, pack_weights_rowwise, quant_act, set_gemv_kernel,
    validate_packed, workspace_bytes, BL_OP_FFN_TP_UP, BL_OP_FFN_TP_DOWN, absmean_sum, pack_weights_global,
    ffn_tp_up, ffn_tp_down, ffn_tp_finish,
)
