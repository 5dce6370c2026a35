"""Shared helpers of the GPU parity tests: device upload of the seeded bf16
inputs and the output tolerance check."""
import numpy as np
import torch

from oracle import rbd_oracle as O


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def host_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(v, np.float64))
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    return np.ldexp(1.0, np.maximum(ex - 1, -126) - 7)


def check_output(gpu_bits: np.ndarray, ref64: np.ndarray, ref_bf16: np.ndarray, rel_tol: float = 1e-3,
                 abs_tol: float = 2e-2):
    """Output tolerance (bf16 output of a float64 reference):
      rel-L2(GPU - RNE_bf16(ref64)) <= rel_tol, and elementwise
      |GPU - ref64| <= max(abs_tol, one bf16 ulp of ref64).
    The plain rel-L2 against ref64 is reported too (bf16 rounding alone gives about 1.6e-3)."""
    g = O.bf16_to_f64(gpu_bits)
    rb = O.bf16_to_f64(ref_bf16)
    denom = max(np.linalg.norm(rb), 1e-30)
    rel = np.linalg.norm(g - rb) / denom
    err = np.abs(g - ref64)
    bound = np.maximum(abs_tol, bf16_ulp(ref64))
    worst = float((err / bound).max(initial=0.0))
    rel64 = np.linalg.norm(g - ref64) / max(np.linalg.norm(ref64), 1e-30)
    assert rel <= rel_tol, f"rel-L2 vs bf16 reference {rel:.3e} > {rel_tol}"
    assert worst <= 1.0, f"max |err|/bound {worst:.3f} (max err {err.max():.3e})"
    return dict(rel_bf16=rel, rel64=rel64, max_err=float(err.max(initial=0.0)), worst=worst)


def e4m3_bytes(codes: np.ndarray) -> np.ndarray:
    """The E4M3 bytes of integer codes, by torch's float8_e4m3fn conversion (exact for |code| <= 16):
    what the quantisers write with the E4M3 code format."""
    t = torch.from_numpy(np.asarray(codes, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()
