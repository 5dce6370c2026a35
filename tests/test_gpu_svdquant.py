"""GPU parity of the offline SVDQuant fit (library path: float64 products on the device,
Householder QR and Jacobi SVD on the host) against the CPU oracle's svdquant_fit on the
same test matrices: the per-iterate objective, the kept iterate, its codes and scales bit
for bit (whenever the residual's bf16 rounding agrees, which float64 differences in the
last bits could only break at a rounding boundary), and the branch L1 L2."""
import numpy as np
import pytest
import torch

import rotated_bit_dit_b200 as R
from oracle import rbd_oracle as O
from rotated_bit_dit_b200 import inputs as I
from tests.helpers import dev_bf16

pytestmark = pytest.mark.gpu


def lowrank_plus_noise(seed, n, k, r=16, noise=0.005):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((n, r)) @ rng.standard_normal((r, k)) * 0.02 / np.sqrt(r) + noise * rng.standard_normal((n, k))
    return O.f64_to_bf16(w)


def omegas(seed, iters, k, p):
    return np.random.default_rng(seed).standard_normal((iters, k, p))


def codes_of(q, bits):
    return O.unpack_int4(q) if bits == 4 else q


@pytest.mark.parametrize("N,K,rank,bits,sg,act", [
    (384, 3072, 32, 4, 0, False),
    (256, 1024, 16, 4, 64, True),
    (128, 512, 8, 8, 0, True),
])
def test_svdquant_fit_matches_oracle(N, K, rank, bits, sg, act):
    wb = lowrank_plus_noise(2000 + N, N, K)
    om = omegas(2001, 3, K, rank + 8)
    act_rms = np.abs(np.random.default_rng(2002).standard_normal(K)) + 0.1 if act else None
    got = R.rbd_svdquant_fit(dev_bf16(wb), rank, om, bits, 256, sg, act_rms)
    assert R.rbd_check() == 0
    ref = O.svdquant_fit(wb, rank, bits, list(om), 256, sg, act_rms)
    # the objective of every iterate, and which one is kept
    assert np.allclose(got["errs"], ref["errs"], rtol=1e-9, atol=0)
    assert got["best"] == int(np.argmin(ref["errs"]))
    assert abs(got["errs"][got["best"]] - ref["err"]) <= 1e-9 * ref["err"]
    # the branch (its factors' signs per component are free; their product is not)
    lr_got, lr_ref = got["l1"] @ got["l2"], ref["l1"] @ ref["l2"]
    assert np.abs(lr_got - lr_ref).max() <= 1e-9 * np.abs(lr_ref).max()
    # codes and scales of the kept iterate
    qg = got["q"].cpu().numpy()
    assert np.array_equal(got["scales"].cpu().numpy().view(np.uint32), np.asarray(ref["scales"]).view(np.uint32))
    assert np.array_equal(codes_of(qg, bits), codes_of(np.asarray(ref["q"]), bits))


def test_svdquant_fit_beats_plain_quantisation():
    # the kept iterate is at least as good as the one-shot split and far better than quantising W alone
    N, K, rank = 256, 1024, 16
    wb = lowrank_plus_noise(2010, N, K, r=rank)
    got = R.rbd_svdquant_fit(dev_bf16(wb), rank, omegas(2011, 4, K, rank + 8), 4, 256, 0)
    assert got["errs"][got["best"]] <= got["errs"][0]
    q, s = O.quantize_weights(wb, 4, 256, 0)
    plain = np.linalg.norm(O.bf16_to_f64(wb) - O.dequantize_weights(q, s, 4, 256, 0))
    assert got["errs"][got["best"]] < 0.5 * plain
