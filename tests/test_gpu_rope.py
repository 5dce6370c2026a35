"""GPU parity of the Q/K RMSNorm + RoPE step against the CPU oracle: the device's
rotary tables within one float32 ulp of the oracle's float64 angles, and the
normalised, turned heads within the output tolerance (each side uses its own
tables), over ragged shapes, with and without gamma and eps, strided rows, in
place, and degenerate heads (all zero, huge, tiny)."""
import numpy as np
import pytest
import torch

import rotated_bit_dit_b200 as R
from oracle import rbd_oracle as O
from rotated_bit_dit_b200 import inputs as I
from tests.helpers import check_output, dev_bf16, host_u16

pytestmark = pytest.mark.gpu


def positions(T: int, seed: int) -> np.ndarray:
    """A frame-major patch grid cut to T tokens, late frames included (times up to ~4000)."""
    grid = I.video_positions(8, 24, 32, t0=4000 - 8)[: T // 2]
    far = I.video_positions(T - len(grid), 1, 1, t0=seed)
    return np.ascontiguousarray(np.concatenate([grid, far])[:T])


def device_tables(pos: np.ndarray):
    T = pos.shape[0]
    cos = torch.empty((T, 64), dtype=torch.float32, device="cuda")
    sin = torch.empty((T, 64), dtype=torch.float32, device="cuda")
    R.rbd_rope_tables(torch.from_numpy(pos).cuda(), cos, sin)
    return cos, sin


def test_rope_tables_within_one_float32_ulp():
    pos = positions(700, 3)
    cos, sin = device_tables(pos)
    assert R.rbd_check() == 0
    rc, rs = O.rope_tables(pos)
    for got, ref in ((cos, rc), (sin, rs)):
        g = got.cpu().numpy().astype(np.float64)
        ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
        assert np.all(np.abs(g - ref) <= ulp), np.abs(g - ref).max()
    zero = device_tables(np.zeros((3, 3), np.int32))
    assert torch.all(zero[0] == 1) and torch.all(zero[1] == 0)


def run_case(T, H, with_gamma, eps, seed, x_scale=1.0, in_place=False, pad=0):
    xb = I.gaussian_bf16(seed, (T, H, 128), x_scale, 0.02, 25.0)
    gb = I.f32_to_bf16_bits((1.0 + 0.1 * I.normal(seed + 1, 128)).astype(np.float32)) if with_gamma else None
    pos = positions(T, seed)
    cos, sin = device_tables(pos)
    ld = H * 128 + pad
    full = np.zeros((T, ld), np.uint16)
    full[:, :H * 128] = xb.reshape(T, H * 128)
    xbuf = dev_bf16(full)
    x = xbuf[:, :H * 128]
    if in_place:
        y = x
    else:
        ybuf = torch.zeros((T, ld), dtype=torch.bfloat16, device="cuda")
        y = ybuf[:, :H * 128]
    g = dev_bf16(gb) if with_gamma else None
    R.rbd_qk_norm_rope(x, cos, sin, y, gamma=g, eps=eps)
    assert R.rbd_check() == 0
    rc, rs = O.rope_tables(pos)
    ref64 = O.qk_norm_rope_f64(xb, gb, rc, rs, eps)
    out = host_u16(xbuf if in_place else ybuf)
    got = out[:, :H * 128]
    stats = check_output(got, ref64.reshape(T, H * 128), O.f64_to_bf16(ref64).reshape(T, H * 128))
    assert not out[:, H * 128:].any()             # the stride padding is not written
    return got, ref64, stats


@pytest.mark.parametrize("T,H", [(1, 1), (7, 3), (360, 24), (64, 40)])
@pytest.mark.parametrize("with_gamma", [False, True])
@pytest.mark.parametrize("eps", [1e-6, 0.0])
def test_qk_norm_rope_parity(T, H, with_gamma, eps):
    run_case(T, H, with_gamma, eps, 1100 + T + H)


def test_qk_norm_rope_strided_and_in_place():
    run_case(33, 5, True, 1e-6, 1200, pad=64)
    run_case(33, 5, True, 1e-6, 1201, pad=64, in_place=True)


@pytest.mark.parametrize("x_scale,eps", [(1e30, 1e-6), (1e-30, 0.0), (1e-4, 1e-6)])
def test_qk_norm_rope_extreme_magnitudes(x_scale, eps):
    run_case(20, 3, True, eps, 1300, x_scale=x_scale)


def test_qk_norm_rope_zero_heads():
    T, H = 6, 2
    x = torch.zeros((T, H * 128), dtype=torch.bfloat16, device="cuda")
    cos, sin = device_tables(positions(T, 1))
    y = torch.full((T, H * 128), 7.0, dtype=torch.bfloat16, device="cuda")
    R.rbd_qk_norm_rope(x, cos, sin, y, eps=0.0)
    assert R.rbd_check() == 0
    assert torch.all(y.float() == 0)              # r = 0 on an all-zero head: zeros (of either sign)
