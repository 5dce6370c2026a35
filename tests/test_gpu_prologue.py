"""GPU parity of the prologue kernels against the CPU oracle (bit-exact codes and
scales), the offline weight packers, the low-rank down product, and the
device-side timeout path."""
import numpy as np
import pytest
import torch

import rotated_bit_dit_b200 as R
from oracle import rbd_oracle as O
from rotated_bit_dit_b200 import inputs as I
from tests.helpers import dev_bf16, e4m3_bytes

pytestmark = pytest.mark.gpu


def run_rot_quant(xb, bits, rot, sg):
    M, K = xb.shape
    x = dev_bf16(xb)
    codes = torch.empty((M, K), dtype=torch.int8, device="cuda")
    scales = torch.empty((M, K // 64) if sg else (M,), dtype=torch.float32, device="cuda")
    R.rbd_rot_quant_act(x, codes, scales, bits, rot, sg)
    assert R.rbd_check() == 0
    return codes.cpu().numpy(), scales.cpu().numpy()


@pytest.mark.parametrize("M,K", [(64, 256), (37, 768), (5, 3072), (3, 12288), (2, 16384), (1, 512)])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("rot", [256, 0])
@pytest.mark.parametrize("sg", [0, 64])
def test_rot_quant_bit_exact(M, K, bits, rot, sg):
    xb = I.gaussian_bf16(100 + K + M, (M, K), 1.0, 0.005, 30.0)
    codes, scales = run_rot_quant(xb, bits, rot, sg)
    ref_q, ref_s = O.rot_quant(xb, bits, rot, sg)
    assert np.array_equal(scales.view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(codes, ref_q)


@pytest.mark.parametrize("M,K", [(64, 256), (37, 768), (5, 3072), (2, 16384)])
@pytest.mark.parametrize("rot", [256, 0])
@pytest.mark.parametrize("sg", [0, 64])
def test_rot_quant_e4m3_codes_bit_exact(M, K, rot, sg):
    # the E4M3 code format holds the same INT4 codes, each as the E4M3 byte of its value
    xb = I.gaussian_bf16(150 + K + M, (M, K), 1.0, 0.005, 30.0)
    x = dev_bf16(xb)
    codes = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, K // 64) if sg else (M,), dtype=torch.float32, device="cuda")
    R.rbd_rot_quant_act(x, codes, scales, 4, rot, sg, code_format=R.CODES_E4M3)
    assert R.rbd_check() == 0
    ref_q, ref_s = O.rot_quant(xb, 4, rot, sg)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), e4m3_bytes(ref_q))


def test_rot_quant_degenerate_rows():
    # all-zero row, a row with one nonzero value, a row of equal values, huge and tiny magnitudes
    K = 512
    x = np.zeros((5, K), np.float32)
    x[1, 7] = -3.0
    x[2, :] = 0.5
    x[3, :] = np.linspace(-1e30, 1e30, K)
    x[4, :] = np.linspace(-1e-30, 1e-30, K)
    xb = I.f32_to_bf16_bits(x)
    for bits in (4, 8):
        for sg in (0, 64):
            codes, scales = run_rot_quant(xb, bits, 256, sg)
            ref_q, ref_s = O.rot_quant(xb, bits, 256, sg)
            assert np.array_equal(codes, ref_q) and np.array_equal(scales.view(np.uint32), ref_s.view(np.uint32))


def test_rot_quant_strided_input():
    M, K, ld = 9, 512, 768
    full = I.gaussian_bf16(7, (M, ld), 1.0, 0.01, 20.0)
    x = dev_bf16(full)[:, :K]
    codes = torch.empty((M, K), dtype=torch.int8, device="cuda")
    scales = torch.empty((M,), dtype=torch.float32, device="cuda")
    R.rbd_rot_quant_act(x, codes, scales, 4, 256, 0)
    ref_q, ref_s = O.rot_quant(np.ascontiguousarray(full[:, :K]), 4)
    assert np.array_equal(codes.cpu().numpy(), ref_q)
    assert np.array_equal(scales.cpu().numpy(), ref_s)


def test_rot_quant_full_w8a8_layer_input():
    cfg = I.CONFIGS["w8a8_ffdown"]
    xb = I.gaussian_bf16(0 + I.SEED_X, (cfg["M"], cfg["K"]), 1.0, 0.005, 30.0, outlier_seed=0)
    codes, scales = run_rot_quant(xb, 8, 256, 0)
    ref_q, ref_s = O.rot_quant(xb, 8, 256, 0)
    assert np.array_equal(scales, ref_s)
    assert np.array_equal(codes, ref_q)


@pytest.mark.parametrize("sg", [0, 64])
def test_pack_weights_int4_bit_exact(sg):
    N, K = 384, 3072
    wb = I.gaussian_bf16(11, (N, K), 0.02)
    w = dev_bf16(wb)
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((N, K // 64) if sg else (N,), dtype=torch.float32, device="cuda")
    R.rbd_pack_weights_int4(w, packed, scales, 256, sg)
    ref_p, ref_s = O.quantize_weights(wb, 4, 256, sg)
    assert np.array_equal(packed.cpu().numpy(), ref_p)
    assert np.array_equal(scales.cpu().numpy(), ref_s)


def test_pack_weights_int8_bit_exact():
    N, K = 256, 12288
    wb = I.gaussian_bf16(12, (N, K), 0.02)
    w = dev_bf16(wb)
    w8 = torch.empty((N, K), dtype=torch.int8, device="cuda")
    scales = torch.empty((N,), dtype=torch.float32, device="cuda")
    R.rbd_pack_weights_int8(w, w8, scales, 256, 0)
    ref_q, ref_s = O.quantize_weights(wb, 8, 256, 0)
    assert np.array_equal(w8.cpu().numpy(), ref_q)
    assert np.array_equal(scales.cpu().numpy(), ref_s)


@pytest.mark.parametrize("r", [16, 32, 64])
@pytest.mark.parametrize("M", [1, 45, 256])
def test_lowrank_fused(r, M):
    K = 3072
    xb = I.gaussian_bf16(13, (M, K), 1.0, 0.005, 30.0)
    l1b = I.gaussian_bf16(14, (K, r), 0.01)
    x, l1t = dev_bf16(xb), dev_bf16(np.ascontiguousarray(l1b.T))
    codes = torch.empty((M, K), dtype=torch.int8, device="cuda")
    scales = torch.empty((M, K // 64), dtype=torch.float32, device="cuda")
    ld = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    R.rbd_lowrank_fused(x, codes, scales, l1t, ld, 4, 256, 64)
    assert R.rbd_check() == 0
    ref_q, ref_s = O.rot_quant(xb, 4, 256, 64)
    assert np.array_equal(codes.cpu().numpy(), ref_q) and np.array_equal(scales.cpu().numpy(), ref_s)
    ref_ld = O.lowrank_down(xb, l1b)
    got = ld.float().cpu().numpy().astype(np.float64)
    # float32 accumulation, one bf16 rounding: within 2^-8 relative plus accumulation noise
    err = np.abs(got - ref_ld)
    assert np.all(err <= np.abs(ref_ld) * 2.0 ** -8 + 1e-4 * np.abs(ref_ld).max())


@pytest.mark.parametrize("M,K,bits,rot,r", [
    (3, 256, 4, 256, 32),      # one 256-block (no prefetch beyond the first)
    (17, 768, 8, 256, 16),     # ragged token tile, INT8 codes
    (33, 12288, 4, 0, 64),     # no rotation, long rows
    (16, 16384, 8, 0, 32),     # K at the supported maximum
    (200, 3072, 4, 256, 64),
])
def test_lowrank_fused_shapes(M, K, bits, rot, r):
    # group-scale prologue in one pass: codes and scales bit-exact, the down
    # product within the float32-accumulation bound
    xb = I.gaussian_bf16(16 + M + K, (M, K), 1.0, 0.005, 30.0)
    l1b = I.gaussian_bf16(17 + r, (K, r), 0.01)
    x, l1t = dev_bf16(xb), dev_bf16(np.ascontiguousarray(l1b.T))
    codes = torch.empty((M, K), dtype=torch.int8, device="cuda")
    scales = torch.empty((M, K // 64), dtype=torch.float32, device="cuda")
    ld = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    R.rbd_lowrank_fused(x, codes, scales, l1t, ld, bits, rot, 64)
    assert R.rbd_check() == 0
    ref_q, ref_s = O.rot_quant(xb, bits, rot, 64)
    assert np.array_equal(codes.cpu().numpy(), ref_q)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    ref_ld = O.lowrank_down(xb, l1b)
    err = np.abs(ld.float().cpu().numpy().astype(np.float64) - ref_ld)
    assert np.all(err <= np.abs(ref_ld) * 2.0 ** -8 + 1e-4 * np.abs(ref_ld).max())


@pytest.mark.parametrize("M,K,rot,r", [(3, 256, 256, 32), (200, 3072, 256, 32), (33, 12288, 0, 64)])
def test_lowrank_fused_e4m3_codes(M, K, rot, r):
    # the single-pass group-scale prologue writing E4M3 code bytes (the layout the FP8 GEMM reads)
    xb = I.gaussian_bf16(26 + M + K, (M, K), 1.0, 0.005, 30.0)
    l1b = I.gaussian_bf16(27 + r, (K, r), 0.01)
    x, l1t = dev_bf16(xb), dev_bf16(np.ascontiguousarray(l1b.T))
    codes = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, K // 64), dtype=torch.float32, device="cuda")
    ld = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    R.rbd_lowrank_fused(x, codes, scales, l1t, ld, 4, rot, 64, code_format=R.CODES_E4M3)
    assert R.rbd_check() == 0
    ref_q, ref_s = O.rot_quant(xb, 4, rot, 64)
    assert np.array_equal(codes.cpu().numpy(), e4m3_bytes(ref_q))
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    ref_ld = O.lowrank_down(xb, l1b)
    err = np.abs(ld.float().cpu().numpy().astype(np.float64) - ref_ld)
    assert np.all(err <= np.abs(ref_ld) * 2.0 ** -8 + 1e-4 * np.abs(ref_ld).max())


def test_lowrank_fused_strided_input_and_row_scales():
    # a row stride larger than K, and the row-scale configuration (two kernels)
    M, K, ldx, r = 21, 1024, 1536, 32
    full = I.gaussian_bf16(18, (M, ldx), 1.0, 0.01, 20.0)
    l1b = I.gaussian_bf16(19, (K, r), 0.01)
    x, l1t = dev_bf16(full)[:, :K], dev_bf16(np.ascontiguousarray(l1b.T))
    xb = np.ascontiguousarray(full[:, :K])
    for sg in (64, 0):
        codes = torch.empty((M, K), dtype=torch.int8, device="cuda")
        scales = torch.empty((M, K // 64) if sg else (M,), dtype=torch.float32, device="cuda")
        ld = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
        R.rbd_lowrank_fused(x, codes, scales, l1t, ld, 4, 256, sg)
        assert R.rbd_check() == 0
        ref_q, ref_s = O.rot_quant(xb, 4, 256, sg)
        assert np.array_equal(codes.cpu().numpy(), ref_q)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
        ref_ld = O.lowrank_down(xb, l1b)
        err = np.abs(ld.float().cpu().numpy().astype(np.float64) - ref_ld)
        assert np.all(err <= np.abs(ref_ld) * 2.0 ** -8 + 1e-4 * np.abs(ref_ld).max())


def test_device_timeout_is_reported_and_context_survives():
    R.rbd_debug_timeout_probe(50_000_000)          # 50 ms bound on a wait nobody satisfies
    assert R.rbd_check() == 5                       # RBD_ERR_DEVICE_TIMEOUT
    assert R.rbd_check() == 0                       # cleared
    xb = I.gaussian_bf16(15, (4, 256))
    codes, scales = run_rot_quant(xb, 4, 256, 0)
    ref_q, _ = O.rot_quant(xb, 4)
    assert np.array_equal(codes, ref_q)
