"""GPU parity of the normalising prologue (RMSNorm + modulation, then the
rotation and the dynamic quantiser) against the CPU oracle: codes and scales
bit for bit, for every rotation / scale-group / bit-width setting, optional
vectors, ragged and strided rows, degenerate rows and the full layer input."""
import numpy as np
import pytest
import torch

import rotated_bit_dit_b200 as R
from oracle import rbd_oracle as O
from rotated_bit_dit_b200 import inputs as I
from tests.helpers import dev_bf16, e4m3_bytes

pytestmark = pytest.mark.gpu


def vectors(K, seed, which="gss"):
    g = O.f64_to_bf16(1.0 + O.bf16_to_f64(I.gaussian_bf16(seed, (K,), 0.1))) if "g" in which else None
    sh = I.gaussian_bf16(seed + 1, (K,), 0.5) if "h" in which or which == "gss" else None
    sc = I.gaussian_bf16(seed + 2, (K,), 0.3) if "c" in which or which == "gss" else None
    return g, sh, sc


def run(x, gamma, shift, scale, eps, bits, rot, sg):
    M, K = x.shape
    codes = torch.empty((M, K), dtype=torch.int8, device="cuda")
    scales = torch.empty((M, K // 64) if sg else (M,), dtype=torch.float32, device="cuda")
    dv = lambda v: None if v is None else dev_bf16(v)
    R.rbd_norm_rot_quant_act(x, codes, scales, dv(gamma), dv(shift), dv(scale), eps, bits, rot, sg)
    assert R.rbd_check() == 0
    return codes.cpu().numpy(), scales.cpu().numpy()


def check(xb, gamma, shift, scale, eps, bits, rot, sg, x=None):
    codes, scales = run(dev_bf16(xb) if x is None else x, gamma, shift, scale, eps, bits, rot, sg)
    ref_q, ref_s = O.norm_rot_quant(xb, bits, rot, sg, gamma, shift, scale, eps)
    assert np.array_equal(scales.view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(codes, ref_q)


@pytest.mark.parametrize("M,K", [(64, 256), (37, 768), (5, 3072), (3, 12288), (2, 16384), (1, 512)])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("rot", [256, 0])
@pytest.mark.parametrize("sg", [0, 64])
def test_norm_rot_quant_bit_exact(M, K, bits, rot, sg):
    xb = I.gaussian_bf16(500 + K + M, (M, K), 1.0, 0.005, 30.0)
    g, sh, sc = vectors(K, 600 + K)
    check(xb, g, sh, sc, 1e-6, bits, rot, sg)


@pytest.mark.parametrize("which", ["", "g", "h", "c", "gh"])
def test_norm_optional_vectors(which):
    K = 1024
    xb = I.gaussian_bf16(40, (19, K), 1.0, 0.01, 20.0)
    g, sh, sc = vectors(K, 41, which if which else "none")
    check(xb, g, sh, sc, 1e-5, 4, 256, 64)


def test_norm_degenerate_rows():
    K = 512
    x = np.zeros((6, K), np.float32)
    x[1, 3] = -2.5                                   # one nonzero value
    x[2, :] = 0.75                                   # constant row
    x[3, :] = np.linspace(-3e30, 3e30, K)            # huge magnitudes
    x[4, :] = np.linspace(-1e-30, 1e-30, K)          # tiny magnitudes
    x[5, ::7] = 1e-3                                 # sparse row
    xb = I.f32_to_bf16_bits(x)
    g, sh, sc = vectors(K, 42)
    for eps in (0.0, 1e-6):                          # eps 0: the zero row gets r = 0, output = shift
        for sg in (0, 64):
            check(xb, g, sh, sc, eps, 4, 256, sg)
            check(xb, None, None, None, eps, 8, 256, sg)


def test_norm_strided_input():
    M, K, ld = 11, 768, 1024
    full = I.gaussian_bf16(43, (M, ld), 1.0, 0.01, 20.0)
    g, sh, sc = vectors(K, 44)
    xb = np.ascontiguousarray(full[:, :K])
    check(xb, g, sh, sc, 1e-6, 4, 256, 0, x=dev_bf16(full)[:, :K])


def test_norm_full_layer_input():
    # the grouped Q|K|V|gate layer's input, 4096 tokens x 3072, with group-64 INT4 codes
    cfg = I.CONFIGS["w4a4_qkvg"]
    xb = I.gaussian_bf16(I.SEED_X, (cfg["M"], cfg["K"]), 1.0, 0.005, 30.0, outlier_seed=0)
    g, sh, sc = vectors(cfg["K"], 45)
    check(xb, g, sh, sc, 1e-6, 4, 256, 64)


@pytest.mark.parametrize("sg", [0, 64])
def test_norm_rot_quant_e4m3_codes(sg):
    # the normalising prologue writing E4M3 code bytes: the same codes as the oracle, as E4M3 values
    M, K = 29, 3072
    xb = I.gaussian_bf16(700, (M, K), 1.0, 0.005, 30.0)
    g, sh, sc = vectors(K, 701)
    dv = lambda v: None if v is None else dev_bf16(v)
    codes = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, K // 64) if sg else (M,), dtype=torch.float32, device="cuda")
    R.rbd_norm_rot_quant_act(dev_bf16(xb), codes, scales, dv(g), dv(sh), dv(sc), 1e-6, 4, 256, sg,
                             code_format=R.CODES_E4M3)
    assert R.rbd_check() == 0
    ref_q, ref_s = O.norm_rot_quant(xb, 4, 256, sg, g, sh, sc, 1e-6)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ref_s.view(np.uint32))
    assert np.array_equal(codes.cpu().numpy(), e4m3_bytes(ref_q))
