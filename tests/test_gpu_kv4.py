"""GPU parity of the INT4 KV-cache codec against the CPU oracle: codes and
scales bit for bit on encode, bf16 values bit for bit on decode (decode is fed
both the GPU's own cache and caches the oracle wrote), the ring addressing,
strided rows, degenerate heads and every grouping."""
import numpy as np
import pytest
import torch

import rotated_bit_dit_b200 as R
from oracle import rbd_oracle as O
from rotated_bit_dit_b200 import inputs as I
from tests.helpers import dev_bf16, host_u16

pytestmark = pytest.mark.gpu


def cache(capacity, H, n):
    codes = torch.zeros((capacity, H, 64), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((capacity, H, 3 * n), dtype=torch.float32, device="cuda")
    return codes, scales


@pytest.mark.parametrize("T,H", [(1, 1), (7, 3), (64, 40), (300, 8)])
@pytest.mark.parametrize("n", [1, 2, 4])
def test_kv4_encode_decode_bit_exact(T, H, n):
    xb = I.gaussian_bf16(700 + T + H, (T, H, 128), 1.0, 0.01, 30.0)
    codes, scales = cache(T, H, n)
    R.rbd_kv4_encode(dev_bf16(xb.reshape(T, H * 128)), codes, scales, n)
    assert R.rbd_check() == 0
    ref_p, ref_s = O.kv4_encode(xb, n)
    assert np.array_equal(codes.cpu().numpy(), ref_p)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    y = torch.empty((T, H * 128), dtype=torch.bfloat16, device="cuda")
    R.rbd_kv4_decode(codes, scales, y, n)
    assert R.rbd_check() == 0
    assert np.array_equal(host_u16(y).reshape(T, H, 128), O.kv4_decode(ref_p, ref_s, n))


@pytest.mark.parametrize("n", [1, 2, 4])
def test_kv4_decode_of_an_oracle_cache(n):
    T, H = 33, 5
    xb = I.gaussian_bf16(710 + n, (T, H, 128), 2.0, 0.02, 10.0)
    ref_p, ref_s = O.kv4_encode(xb, n)
    codes = torch.from_numpy(ref_p).cuda()
    scales = torch.from_numpy(ref_s).cuda()
    y = torch.empty((T, H * 128), dtype=torch.bfloat16, device="cuda")
    R.rbd_kv4_decode(codes, scales, y, n)
    assert R.rbd_check() == 0
    assert np.array_equal(host_u16(y).reshape(T, H, 128), O.kv4_decode(ref_p, ref_s, n))


def test_kv4_ring_addressing_and_strided_rows():
    capacity, H, n, T, slot0, ld = 16, 4, 2, 9, 12, 4 * 128 + 64
    full = I.gaussian_bf16(720, (T, ld), 1.0, 0.01, 20.0)
    x = dev_bf16(full)[:, :H * 128]
    codes, scales = cache(capacity, H, n)
    R.rbd_kv4_encode(x, codes, scales, n, slot0)
    assert R.rbd_check() == 0
    xb = np.ascontiguousarray(full[:, :H * 128]).reshape(T, H, 128)
    ref_p, ref_s = O.kv4_encode(xb, n)
    slots = [(slot0 + t) % capacity for t in range(T)]
    got_p, got_s = codes.cpu().numpy(), scales.cpu().numpy()
    assert np.array_equal(got_p[slots], ref_p) and np.array_equal(got_s[slots], ref_s)
    untouched = [s for s in range(capacity) if s not in slots]
    assert not got_p[untouched].any() and not got_s[untouched].any()
    yfull = torch.zeros((T, ld), dtype=torch.bfloat16, device="cuda")
    R.rbd_kv4_decode(codes, scales, yfull[:, :H * 128], n, slot0)
    assert R.rbd_check() == 0
    out = host_u16(yfull)
    assert np.array_equal(out[:, :H * 128].reshape(T, H, 128), O.kv4_decode(ref_p, ref_s, n))
    assert not out[:, H * 128:].any()          # the stride padding is not written


def test_kv4_degenerate_heads():
    x = np.zeros((4, 2, 128), np.float32)
    x[1, 0, :44] = 7.0                          # the worked example of the oracle pins
    x[1, 0, 44:86] = -3.5
    x[2, 1, :] = np.linspace(-3e30, 3e30, 128)  # huge magnitudes
    x[3, :, :] = np.linspace(-1e-30, 1e-30, 128)
    xb = I.f32_to_bf16_bits(x)
    for n in (1, 2, 4):
        codes, scales = cache(4, 2, n)
        R.rbd_kv4_encode(dev_bf16(xb.reshape(4, 256)), codes, scales, n)
        assert R.rbd_check() == 0
        ref_p, ref_s = O.kv4_encode(xb, n)
        assert np.array_equal(codes.cpu().numpy(), ref_p)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
