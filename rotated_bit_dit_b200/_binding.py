"""ctypes binding of librbd.so: the same entry points as include/rbd.h.

Argument marshalling only.  Every computation runs in the library's CUDA
kernels; there is no Python or CPU fallback.  Tensors must be CUDA tensors on
the current device (others are refused before any launch); the current torch
stream is used unless `stream` is given.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

RBD_OK = 0
STATUS_NAMES = {0: "RBD_OK", 1: "RBD_ERR_INVALID_ARG", 2: "RBD_ERR_UNSUPPORTED", 3: "RBD_ERR_ALIGNMENT",
                4: "RBD_ERR_CUDA", 5: "RBD_ERR_DEVICE_TIMEOUT"}

EXPORTED = ("rbd_rot_quant_act", "rbd_norm_rot_quant_act", "rbd_lowrank_fused", "rbd_lowrank_down", "rbd_pack_weights_int4", "rbd_pack_weights_int8",
            "rbd_w4a4_linear", "rbd_w8a8_linear", "rbd_nvfp4_scale_bytes", "rbd_nvfp4_quant",
            "rbd_nvfp4_quant_noalloc", "rbd_nvfp4_linear", "rbd_kv4_encode", "rbd_kv4_decode", "rbd_qk_norm_rope", "rbd_rope_tables", "rbd_attn_workspace_bytes", "rbd_attn_quant", "rbd_attn_int8",
            "rbd_svdquant_workspace_bytes", "rbd_svdquant_fit",
            "rbd_check", "rbd_debug_timeout_probe", "rbd_status_string", "rbd_version")


class RbdError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


CODES_INT8 = 0   # activation code stored as a two's-complement int8
CODES_E4M3 = 1   # activation code stored as the E4M3 byte of the same value (4-bit codes)


class QCfg(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("rot_group", ctypes.c_int32), ("scale_group", ctypes.c_int32),
                ("code_format", ctypes.c_int32)]


class Epilogue(ctypes.Structure):
    _fields_ = [("bias", ctypes.c_void_p), ("ld", ctypes.c_void_p), ("l2t", ctypes.c_void_p),
                ("r", ctypes.c_int32), ("gate_mode", ctypes.c_int32), ("gate_col0", ctypes.c_int64),
                ("gate_col1", ctypes.c_int64), ("gate", ctypes.c_void_p), ("residual", ctypes.c_void_p),
                ("ldr", ctypes.c_int64), ("acc_debug", ctypes.c_void_p)]


_LIB = None


def lib_path() -> str:
    return _build.LIB_PATH


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load librbd.so (building it first when absent).  Raises if it cannot be loaded."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = lib_path()
    if not os.path.exists(path):
        if not build_if_missing:
            raise RuntimeError(f"librbd.so not built: {path}")
        _build.build()
    lib = ctypes.CDLL(path)
    i64, i32, vp = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
    sigs = {
        "rbd_rot_quant_act": [vp, i64, i64, i64, QCfg, vp, vp, vp],
        "rbd_norm_rot_quant_act": [vp, i64, i64, i64, vp, vp, vp, ctypes.c_float, QCfg, vp, vp, vp],
        "rbd_lowrank_fused": [vp, i64, i64, i64, QCfg, vp, vp, vp, i32, vp, vp],
        "rbd_lowrank_down": [vp, i64, i64, i64, vp, i32, vp, vp],
        "rbd_pack_weights_int4": [vp, i64, i64, QCfg, vp, vp, vp],
        "rbd_pack_weights_int8": [vp, i64, i64, QCfg, vp, vp, vp],
        "rbd_w4a4_linear": [vp, vp, vp, vp, i64, i64, i64, QCfg, ctypes.POINTER(Epilogue), vp, i64, vp],
        "rbd_w8a8_linear": [vp, vp, vp, vp, i64, i64, i64, QCfg, ctypes.POINTER(Epilogue), vp, i64, vp],
        "rbd_nvfp4_quant": [vp, i64, i64, i64, i32, vp, vp, vp, vp, vp],
        "rbd_nvfp4_quant_noalloc": [vp, i64, i64, i64, i32, vp, vp, vp, vp],
        "rbd_nvfp4_linear": [vp, vp, vp, vp, vp, vp, i64, i64, i64, ctypes.POINTER(Epilogue), vp, i64, vp],
        "rbd_kv4_encode": [vp, i64, i64, i64, i32, vp, vp, i64, i64, vp],
        "rbd_kv4_decode": [vp, vp, i64, i64, i64, i64, i32, vp, i64, vp],
        "rbd_qk_norm_rope": [vp, i64, i64, i64, vp, vp, vp, ctypes.c_float, vp, i64, vp],
        "rbd_rope_tables": [vp, i64, ctypes.c_double, vp, vp, vp],
        "rbd_attn_quant": [vp, i64, vp, i64, vp, i64, i64, i64, i64, vp, vp, vp, vp, vp, i64, vp, vp],
        "rbd_attn_int8": [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, i64, vp],
        "rbd_svdquant_fit": [vp, i64, i64, QCfg, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "rbd_check": [vp],
        "rbd_debug_timeout_probe": [i64, vp],
    }
    for name, args in sigs.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.rbd_nvfp4_scale_bytes.argtypes = [i64, i64]
    lib.rbd_nvfp4_scale_bytes.restype = i64
    lib.rbd_attn_workspace_bytes.argtypes = [i64, i64]
    lib.rbd_attn_workspace_bytes.restype = i64
    lib.rbd_svdquant_workspace_bytes.argtypes = [i64, i64, i32, i32, QCfg]
    lib.rbd_svdquant_workspace_bytes.restype = i64
    lib.rbd_status_string.argtypes = [ctypes.c_int]
    lib.rbd_status_string.restype = ctypes.c_char_p
    lib.rbd_version.argtypes = []
    lib.rbd_version.restype = ctypes.c_char_p
    _LIB = lib
    return lib


def _ptr(t: Optional[torch.Tensor]):
    """Device address of t.  Every kernel launches on the current device, so a tensor that
    lives on another device is refused here, before any launch (its address would be
    dereferenced by the wrong GPU)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    cur = torch.cuda.current_device()
    if t.device.index is not None and t.device.index != cur:
        raise ValueError(f"tensor on {t.device} while cuda:{cur} is current; "
                         f"call under torch.cuda.device({t.device})")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ok(status: int, where: str):
    if status != RBD_OK:
        raise RbdError(status, where)


def _qcfg(bits: int, rot_group: int, scale_group: int, code_format: int = CODES_INT8) -> QCfg:
    return QCfg(bits, rot_group, scale_group, code_format)


def _rowstride(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D row-major tensor")
    return t.stride(0)


# ---------------------------------------------------------------- entry points
def rbd_rot_quant_act(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, bits: int = 4,
                      rot_group: int = 256, scale_group: int = 0, stream=None, code_format: int = CODES_INT8) -> None:
    """x bf16 [M, K] -> codes [M, K] (one byte each, in code_format), scales float32 [M] or [M, K/64]."""
    M, K = x.shape
    _ok(load().rbd_rot_quant_act(_ptr(x), M, K, _rowstride(x), _qcfg(bits, rot_group, scale_group, code_format),
                                 _ptr(codes), _ptr(scales), _stream(stream)), "rbd_rot_quant_act")


def rbd_norm_rot_quant_act(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                           gamma: Optional[torch.Tensor] = None, shift: Optional[torch.Tensor] = None,
                           scale: Optional[torch.Tensor] = None, eps: float = 1e-6, bits: int = 4,
                           rot_group: int = 256, scale_group: int = 0, stream=None,
                           code_format: int = CODES_INT8) -> None:
    """RMSNorm (optional gamma) and modulation x*(1 + scale) + shift, then rbd_rot_quant_act.
    gamma, shift, scale: bf16 [K] or None."""
    M, K = x.shape
    for name, v in (("gamma", gamma), ("shift", shift), ("scale", scale)):
        if v is not None and (v.numel() != K or not v.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous bf16 vector of length K")
    _ok(load().rbd_norm_rot_quant_act(_ptr(x), M, K, _rowstride(x), _ptr(gamma), _ptr(shift), _ptr(scale),
                                      float(eps), _qcfg(bits, rot_group, scale_group, code_format), _ptr(codes),
                                      _ptr(scales), _stream(stream)), "rbd_norm_rot_quant_act")


def rbd_lowrank_fused(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, l1t: torch.Tensor,
                      ld: torch.Tensor, bits: int = 4, rot_group: int = 256, scale_group: int = 0,
                      stream=None, code_format: int = CODES_INT8) -> None:
    """rbd_rot_quant_act plus ld = X @ L1 (l1t = L1^T bf16 [r, K], ld bf16 [M, r])."""
    M, K = x.shape
    r = l1t.shape[0]
    if _rowstride(l1t) != K:
        raise ValueError("l1t must be a contiguous [r, K] tensor")
    _ok(load().rbd_lowrank_fused(_ptr(x), M, K, _rowstride(x), _qcfg(bits, rot_group, scale_group, code_format),
                                 _ptr(codes), _ptr(scales), _ptr(l1t), r, _ptr(ld), _stream(stream)),
        "rbd_lowrank_fused")


def rbd_lowrank_down(x: torch.Tensor, l1t: torch.Tensor, ld: torch.Tensor, stream=None) -> None:
    """ld = X @ L1 alone (l1t = L1^T bf16 [r, K], ld bf16 [M, r])."""
    M, K = x.shape
    r = l1t.shape[0]
    if _rowstride(l1t) != K:
        raise ValueError("l1t must be a contiguous [r, K] tensor")
    _ok(load().rbd_lowrank_down(_ptr(x), M, K, _rowstride(x), _ptr(l1t), r, _ptr(ld), _stream(stream)),
        "rbd_lowrank_down")


def rbd_pack_weights_int4(w: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, rot_group: int = 256,
                          scale_group: int = 0, stream=None) -> None:
    """w bf16 [N, K] -> packed uint8 [N, K/2], scales float32 [N] or [N, K/64]."""
    N, K = w.shape
    _ok(load().rbd_pack_weights_int4(_ptr(w), N, K, _qcfg(4, rot_group, scale_group), _ptr(packed),
                                     _ptr(scales), _stream(stream)), "rbd_pack_weights_int4")


def rbd_pack_weights_int8(w: torch.Tensor, w8: torch.Tensor, scales: torch.Tensor, rot_group: int = 256,
                          scale_group: int = 0, stream=None) -> None:
    """w bf16 [N, K] -> w8 int8 [N, K], scales float32 [N] or [N, K/64]."""
    N, K = w.shape
    _ok(load().rbd_pack_weights_int8(_ptr(w), N, K, _qcfg(8, rot_group, scale_group), _ptr(w8),
                                     _ptr(scales), _stream(stream)), "rbd_pack_weights_int8")


def make_epilogue(bias=None, ld=None, l2t=None, gate_mode: int = 0, gate_cols=(0, 0), gate=None,
                  residual=None, acc_debug=None) -> Epilogue:
    e = Epilogue()
    e.bias = _ptr(bias)
    e.ld = _ptr(ld)
    e.l2t = _ptr(l2t)
    e.r = 0 if ld is None else int(ld.shape[1])
    e.gate_mode = gate_mode
    e.gate_col0, e.gate_col1 = int(gate_cols[0]), int(gate_cols[1])
    e.gate = _ptr(gate)
    e.residual = _ptr(residual)
    e.ldr = 0 if residual is None else _rowstride(residual)
    e.acc_debug = _ptr(acc_debug)
    return e


def _linear(fn, where, codes, sx, w, sw, y, bits, rot_group, scale_group, epi, stream, code_format=CODES_INT8):
    M, K = codes.shape
    N = y.shape[1]
    e = epi if epi is not None else Epilogue()
    _ok(fn(_ptr(codes), _ptr(sx), _ptr(w), _ptr(sw), M, N, K, _qcfg(bits, rot_group, scale_group, code_format),
           ctypes.byref(e), _ptr(y), _rowstride(y), _stream(stream)), where)


def rbd_w4a4_linear(codes: torch.Tensor, sx: torch.Tensor, w_packed: torch.Tensor, sw: torch.Tensor,
                    y: torch.Tensor, scale_group: int = 0, epi: Optional[Epilogue] = None,
                    rot_group: int = 256, stream=None, code_format: int = CODES_INT8) -> None:
    """y bf16 [M, N] = epilogue(dequant(codes @ unpack(w_packed)^T)); codes in code_format (E4M3
    codes take the FP8 tensor-core path, group-64 scales only)."""
    _linear(load().rbd_w4a4_linear, "rbd_w4a4_linear", codes, sx, w_packed, sw, y, 4, rot_group,
            scale_group, epi, stream, code_format)


def rbd_w8a8_linear(codes: torch.Tensor, sx: torch.Tensor, w8: torch.Tensor, sw: torch.Tensor,
                    y: torch.Tensor, scale_group: int = 0, epi: Optional[Epilogue] = None,
                    rot_group: int = 256, stream=None) -> None:
    """y bf16 [M, N] = epilogue(dequant(codes @ w8^T))."""
    _linear(load().rbd_w8a8_linear, "rbd_w8a8_linear", codes, sx, w8, sw, y, 8, rot_group,
            scale_group, epi, stream)


def rbd_nvfp4_scale_bytes(rows: int, K: int) -> int:
    """Bytes of a tile-interleaved E4M3 block-scale buffer for `rows` rows of length K."""
    return int(load().rbd_nvfp4_scale_bytes(rows, K))


def rbd_nvfp4_quant(x: torch.Tensor, codes: torch.Tensor, block_scales: torch.Tensor, tensor_scale: torch.Tensor,
                    work: torch.Tensor, rot_group: int = 256, stream=None) -> None:
    """x bf16 [M, K] -> codes uint8 [M, K/2] (E2M1 pairs), block_scales uint8 (tile-interleaved E4M3,
    rbd_nvfp4_scale_bytes(M, K)), tensor_scale float32 [1]; work: 4 bytes of device scratch."""
    M, K = x.shape
    _ok(load().rbd_nvfp4_quant(_ptr(x), M, K, _rowstride(x), rot_group, _ptr(codes), _ptr(block_scales),
                               _ptr(tensor_scale), _ptr(work), _stream(stream)), "rbd_nvfp4_quant")


def rbd_nvfp4_quant_noalloc(x: torch.Tensor, codes: torch.Tensor, block_scales: torch.Tensor,
                            tensor_scale: torch.Tensor, rot_group: int = 256, stream=None) -> None:
    """rbd_nvfp4_quant with its scratch word in library-owned device memory (no scratch argument)."""
    M, K = x.shape
    _ok(load().rbd_nvfp4_quant_noalloc(_ptr(x), M, K, _rowstride(x), rot_group, _ptr(codes), _ptr(block_scales),
                                       _ptr(tensor_scale), _stream(stream)), "rbd_nvfp4_quant_noalloc")


def rbd_nvfp4_linear(xq, xbs, xgs, wq, wbs, wgs, y: torch.Tensor, epi: Optional[Epilogue] = None,
                     stream=None) -> None:
    """y bf16 [M, N] = epilogue(gs_x gs_w (Q_x . Q_w^T)) on the block-scaled FP4 tensor cores."""
    M, K2 = xq.shape
    N = y.shape[1]
    e = epi if epi is not None else Epilogue()
    _ok(load().rbd_nvfp4_linear(_ptr(xq), _ptr(xbs), _ptr(xgs), _ptr(wq), _ptr(wbs), _ptr(wgs), M, N, 2 * K2,
                                ctypes.byref(e), _ptr(y), _rowstride(y), _stream(stream)), "rbd_nvfp4_linear")


def rbd_check(stream=None) -> int:
    """Synchronise the stream and return the device status (0 = fine)."""
    return load().rbd_check(_stream(stream))


def rbd_debug_timeout_probe(timeout_ns: int, stream=None) -> None:
    _ok(load().rbd_debug_timeout_probe(int(timeout_ns), _stream(stream)), "rbd_debug_timeout_probe")


def rbd_status_string(status: int) -> str:
    return load().rbd_status_string(status).decode()


def rbd_version() -> str:
    return load().rbd_version().decode()


def rbd_kv4_encode(x: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor, groups_per_band: int = 1,
                   slot0: int = 0, stream=None) -> None:
    """x bf16 [T, H*128] (row stride may be larger) -> cache slots (slot0 + t) mod capacity of
    codes uint8 [capacity, H, 64] and scales float32 [capacity, H, 3*groups_per_band]."""
    T = x.shape[0]
    capacity, H = codes.shape[0], codes.shape[1]
    _ok(load().rbd_kv4_encode(_ptr(x), T, H, _rowstride(x), groups_per_band, _ptr(codes), _ptr(scales),
                              capacity, slot0, _stream(stream)), "rbd_kv4_encode")


def rbd_kv4_decode(codes: torch.Tensor, scales: torch.Tensor, y: torch.Tensor, groups_per_band: int = 1,
                   slot0: int = 0, stream=None) -> None:
    """Cache slots (slot0 + t) mod capacity, t < y.shape[0] -> y bf16 [T, H*128]."""
    T = y.shape[0]
    capacity, H = codes.shape[0], codes.shape[1]
    _ok(load().rbd_kv4_decode(_ptr(codes), _ptr(scales), capacity, slot0, T, H, groups_per_band, _ptr(y),
                              _rowstride(y), _stream(stream)), "rbd_kv4_decode")


def rbd_qk_norm_rope(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor, y: torch.Tensor,
                     gamma: Optional[torch.Tensor] = None, eps: float = 1e-6, stream=None) -> None:
    """x bf16 [T, H*128] (row stride may be larger) -> y bf16 [T, H*128] (y may be x): per-head
    RMSNorm times gamma (bf16 [128] or None), then the RoPE turn by cos / sin float32 [T, 64]."""
    T = x.shape[0]
    if x.shape[1] % 128 or y.shape[0] != T or y.shape[1] != x.shape[1]:
        raise ValueError("x and y must be [T, H*128]")
    if cos.shape != (T, 64) or sin.shape != (T, 64) or not (cos.is_contiguous() and sin.is_contiguous()):
        raise ValueError("cos and sin must be contiguous [T, 64]")
    _ok(load().rbd_qk_norm_rope(_ptr(x), T, x.shape[1] // 128, _rowstride(x), _ptr(gamma), _ptr(cos), _ptr(sin),
                                eps, _ptr(y), _rowstride(y), _stream(stream)), "rbd_qk_norm_rope")


def rbd_rope_tables(pos: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor, base: float = 10000.0,
                    stream=None) -> None:
    """pos int32 [T, 3] (time, height, width) -> cos, sin float32 [T, 64]."""
    T = pos.shape[0]
    if pos.dtype != torch.int32 or pos.shape != (T, 3) or not pos.is_contiguous():
        raise ValueError("pos must be contiguous int32 [T, 3]")
    if cos.shape != (T, 64) or sin.shape != (T, 64) or not (cos.is_contiguous() and sin.is_contiguous()):
        raise ValueError("cos and sin must be contiguous [T, 64]")
    _ok(load().rbd_rope_tables(_ptr(pos), T, base, _ptr(cos), _ptr(sin), _stream(stream)), "rbd_rope_tables")


def rbd_attn_workspace_bytes(Tk: int, H: int) -> int:
    """Bytes of device scratch rbd_attn_quant needs for Tk keys and H heads."""
    return int(load().rbd_attn_workspace_bytes(Tk, H))


def rbd_attn_quant(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, H: int, qc: torch.Tensor, sq: torch.Tensor,
                   kc: torch.Tensor, sk: torch.Tensor, vt: torch.Tensor, work: torch.Tensor, stream=None) -> None:
    """q bf16 [Tq, >=H*128], k / v bf16 [Tk, >=H*128] -> qc int8 [H, Tq, 128], sq float32 [H, Tq],
    kc int8 [H, Tk, 128], sk float32 [H, tkp], vt fp16 [H, 128, tkp] (tkp = sk.shape[1]);
    work: rbd_attn_workspace_bytes(Tk, H) bytes of device scratch."""
    Tq, Tk = q.shape[0], k.shape[0]
    tkp = sk.shape[1]
    if vt.shape[-1] != tkp:
        raise ValueError("sk and vt must share the padded key count")
    _ok(load().rbd_attn_quant(_ptr(q), _rowstride(q), _ptr(k), _rowstride(k), _ptr(v), _rowstride(v), Tq, Tk, H,
                              _ptr(qc), _ptr(sq), _ptr(kc), _ptr(sk), _ptr(vt), tkp, _ptr(work), _stream(stream)),
        "rbd_attn_quant")


def rbd_attn_int8(qc: torch.Tensor, sq: torch.Tensor, kc: torch.Tensor, sk: torch.Tensor, vt: torch.Tensor,
                  o: torch.Tensor, stream=None) -> None:
    """Attention on rbd_attn_quant's operands -> o bf16 [Tq, >=H*128]."""
    H, Tq = sq.shape
    Tk = kc.shape[1]
    _ok(load().rbd_attn_int8(_ptr(qc), _ptr(sq), _ptr(kc), _ptr(sk), _ptr(vt), Tq, Tk, H, sk.shape[1], _ptr(o),
                             _rowstride(o), _stream(stream)), "rbd_attn_int8")


def rbd_svdquant_fit(w: torch.Tensor, rank: int, omegas, bits: int = 4, rot_group: int = 256, scale_group: int = 0,
                     act_rms=None, stream=None):
    """The offline SVDQuant fit of a bf16 [N, K] CUDA weight.  omegas: float64 array-like
    [iters, K, rank + oversample] (the test matrices); act_rms: float64 [K] or None.
    Returns dict(q, scales (CUDA tensors of the kept iterate), l1 [K, rank], l2 [rank, N] (float64
    numpy), errs [iters] (float64 numpy), best).  Synchronous."""
    import numpy as np
    N, K = w.shape
    om = np.ascontiguousarray(omegas, dtype=np.float64)
    iters, k_, p = om.shape
    if k_ != K or p < rank:
        raise ValueError("omegas must be [iters, K, rank + oversample]")
    cfg = _qcfg(bits, rot_group, scale_group)
    nbytes = int(load().rbd_svdquant_workspace_bytes(N, K, rank, p - rank, cfg))
    if nbytes < 0:
        raise RbdError(2, "rbd_svdquant_workspace_bytes")
    dev = w.device
    work = torch.empty((nbytes,), dtype=torch.uint8, device=dev)
    q = torch.empty((N, K // 2) if bits == 4 else (N, K), dtype=torch.uint8 if bits == 4 else torch.int8, device=dev)
    scales = torch.empty((N, K // 64) if scale_group else (N,), dtype=torch.float32, device=dev)
    l1 = np.zeros((K, rank), np.float64)
    l2 = np.zeros((rank, N), np.float64)
    errs = np.zeros(iters, np.float64)
    best = ctypes.c_int32(-1)
    ar = None if act_rms is None else np.ascontiguousarray(act_rms, dtype=np.float64)
    dp = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)
    _ok(load().rbd_svdquant_fit(_ptr(w), N, K, cfg, rank, p - rank, iters, dp(om), dp(ar), _ptr(q), _ptr(scales),
                                dp(l1), dp(l2), dp(errs), ctypes.byref(best), _ptr(work), _stream(stream)),
        "rbd_svdquant_fit")
    return dict(q=q, scales=scales, l1=l1, l2=l2, errs=errs, best=int(best.value))
