"""The allocation-free NVFP4 quantiser entry point (library-owned scratch)
against the entry point that takes a caller scratch buffer: identical codes,
block scales and tensor scale, on two calls in a row with different inputs.
Collected last so it also runs after every other GPU test."""
import numpy as np
import pytest
import torch

import rotated_bit_dit_b200 as R
from rotated_bit_dit_b200 import inputs as I
from tests.helpers import dev_bf16

pytestmark = pytest.mark.gpu


def quant(xb, noalloc):
    M, K = xb.shape
    x = dev_bf16(xb)
    codes = torch.zeros((M, K // 2), dtype=torch.uint8, device="cuda")
    bs = torch.zeros((R.rbd_nvfp4_scale_bytes(M, K),), dtype=torch.uint8, device="cuda")
    gs = torch.zeros((1,), dtype=torch.float32, device="cuda")
    if noalloc:
        R.rbd_nvfp4_quant_noalloc(x, codes, bs, gs)
    else:
        work = torch.empty((1,), dtype=torch.int32, device="cuda")
        R.rbd_nvfp4_quant(x, codes, bs, gs, work)
    assert R.rbd_check() == 0
    return codes.cpu().numpy(), bs.cpu().numpy(), gs.cpu().numpy()


def test_noalloc_matches_caller_scratch_on_two_calls_in_a_row():
    # the second input has a much smaller amax: a scratch word left over from
    # the first call would give a wrong tensor scale
    inputs = [I.gaussian_bf16(500, (200, 3072), 1.0, 0.005, 30.0), I.gaussian_bf16(501, (77, 1024), 0.01)]
    for xb in inputs:
        ref = quant(xb, noalloc=False)
        got = quant(xb, noalloc=True)
        for a, b in zip(got, ref):
            assert np.array_equal(a.view(np.uint8), b.view(np.uint8))
