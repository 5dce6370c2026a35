"""rotated_bit_dit_b200: the rotated low-bit quantized linear layer on B200 (sm_100a).

The compute runs in librbd.so (hand-written CUDA for sm_100a behind a C ABI,
include/rbd.h); this package is the ctypes binding plus a small layer object.
Importing the package does not load the library; the first call does, and it
raises if the library cannot be loaded (there is no CPU fallback).
"""
from ._binding import (  # noqa: F401
    CODES_E4M3,
    CODES_INT8,
    EXPORTED,
    Epilogue,
    QCfg,
    RbdError,
    load,
    make_epilogue,
    rbd_check,
    rbd_debug_timeout_probe,
    rbd_lowrank_fused,
    rbd_lowrank_down,
    rbd_pack_weights_int4,
    rbd_pack_weights_int8,
    rbd_rot_quant_act,
    rbd_norm_rot_quant_act,
    rbd_status_string,
    rbd_version,
    rbd_w4a4_linear,
    rbd_w8a8_linear,
    rbd_nvfp4_scale_bytes,
    rbd_nvfp4_quant,
    rbd_nvfp4_quant_noalloc,
    rbd_nvfp4_linear,
    rbd_kv4_encode,
    rbd_kv4_decode,
    rbd_qk_norm_rope,
    rbd_rope_tables,
    rbd_attn_workspace_bytes,
    rbd_attn_quant,
    rbd_attn_int8,
    rbd_svdquant_fit,
)
from .attention import attention_operands, int8_attention  # noqa: F401
from .kvcache import Int4KVCache  # noqa: F401
from .layer import RotatedLowBitLinear  # noqa: F401
