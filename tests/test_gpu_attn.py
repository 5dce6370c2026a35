"""GPU parity of the INT8 attention (SageAttention v1 scheme) against the CPU oracle:
the prepared operands bit for bit (key smoothing, INT8 codes and scales of Q and of the
smoothed K, fp16 transposed values), and the attention output within the stated output
tolerance at ragged query / key counts, several heads, and score ranges that move the
running row maximum across tiles."""
import numpy as np
import pytest
import torch

import rotated_bit_dit_b200 as R
from oracle import rbd_oracle as O
from rotated_bit_dit_b200 import inputs as I
from tests.helpers import check_output, dev_bf16, host_u16

pytestmark = pytest.mark.gpu


def heads(seed, T, H, std=1.0, frac=0.02, scale=20.0):
    return I.gaussian_bf16(seed, (T, H, 128), std, frac, scale)


def run(qb, kb, vb, H, ld_pad=0):
    Tq, Tk = qb.shape[0], kb.shape[0]
    def dev(a):
        full = np.zeros((a.shape[0], H * 128 + ld_pad), np.uint16)
        full[:, :H * 128] = a.reshape(a.shape[0], H * 128)
        return dev_bf16(full)[:, :H * 128] if ld_pad else dev_bf16(full)
    q, k, v = dev(qb), dev(kb), dev(vb)
    ops = R.attention_operands(q, k, v, H)
    o = torch.empty((Tq, H * 128), dtype=torch.bfloat16, device="cuda")
    R.rbd_attn_int8(*ops, o)
    assert R.rbd_check() == 0
    return ops, host_u16(o).reshape(Tq, H, 128)


@pytest.mark.parametrize("Tq,Tk,H", [(64, 77, 1), (130, 300, 2), (1, 1, 1), (256, 1024, 3)])
def test_operands_bit_exact(Tq, Tk, H):
    qb, kb, vb = heads(1100 + Tq, Tq, H), heads(1200 + Tk, Tk, H), heads(1300, Tk, H)
    (qc, sq, kc, sk, vt), _ = run(qb, kb, vb, H)
    rq, rsq = O.quantize_heads_int8(O.bf16_to_f64(qb).astype(np.float32))
    rk, rsk = O.quantize_heads_int8(O.smooth_keys(O.bf16_to_f64(kb).astype(np.float32)))
    assert np.array_equal(qc.cpu().numpy(), rq.transpose(1, 0, 2))
    assert np.array_equal(sq.cpu().numpy().view(np.uint32), rsq.T.view(np.uint32))
    assert np.array_equal(kc.cpu().numpy(), rk.transpose(1, 0, 2))
    assert np.array_equal(sk.cpu().numpy()[:, :Tk].view(np.uint32), rsk.T.copy().view(np.uint32))
    v16 = O.bf16_to_f64(vb).astype(np.float16)                     # [Tk, H, 128]
    got = vt.cpu().numpy()                                         # [H, 128, tkp]
    assert np.array_equal(got[:, :, :Tk].view(np.uint16), v16.transpose(1, 2, 0).view(np.uint16))
    assert not got[:, :, Tk:].view(np.uint16).any()


@pytest.mark.parametrize("Tq,Tk,H", [(128, 128, 1), (200, 333, 2), (1, 77, 3), (384, 1000, 2), (130, 2100, 1)])
def test_attention_matches_oracle(Tq, Tk, H):
    qb, kb, vb = heads(1400 + Tq, Tq, H), heads(1500 + Tk, Tk, H), heads(1600 + H, Tk, H)
    _, y = run(qb, kb, vb, H, ld_pad=64)
    ref64 = O.sage_attention(qb, kb, vb)
    check_output(y.reshape(Tq, -1), ref64.reshape(Tq, -1), O.f64_to_bf16(ref64).reshape(Tq, -1))


def test_attention_running_maximum_moves_across_tiles():
    # keys grow in magnitude along the sequence and queries point along them, so later key tiles hold
    # far larger scores than the first: the running maximum moves several times and O is rescaled.
    # (Much sharper inputs, a few keys carrying the weight, reach rel-L2 ~1e-3 from the fp16 rounding
    # of P alone, the scheme's own P.V precision; these keys keep about a hundred in play.)
    Tq, Tk, H = 128, 1024, 1
    rng = np.random.default_rng(5)
    d = rng.standard_normal(128)
    d /= np.linalg.norm(d)
    ramp = np.linspace(0.0, 6.0, Tk)[:, None]
    k = rng.standard_normal((Tk, 128)) * 1.0 + ramp * d[None, :] * 10
    q = rng.standard_normal((Tq, 128)) * 0.3 + d[None, :] * 3
    qb = I.f32_to_bf16_bits(q.astype(np.float32)).reshape(Tq, 1, 128)
    kb = I.f32_to_bf16_bits(k.astype(np.float32)).reshape(Tk, 1, 128)
    vb = heads(1700, Tk, H)
    _, y = run(qb, kb, vb, H)
    ref64 = O.sage_attention(qb, kb, vb)
    s = O.attention_scores(qb, kb)[0]
    # the running maximum (kept in base 2, moved only past 8) must move: > 12 bits between first and last tile
    assert (s[:, -128:].max(axis=1) - s[:, :128].max(axis=1)).min() > 12 * np.log(2)
    check_output(y.reshape(Tq, -1), ref64.reshape(Tq, -1), O.f64_to_bf16(ref64).reshape(Tq, -1))


def test_attention_deterministic_and_zero_query():
    Tq, Tk, H = 100, 500, 2
    qb, kb, vb = heads(1800, Tq, H), heads(1801, Tk, H), heads(1802, Tk, H)
    qb[3] = 0                                          # an all-zero query: uniform weights over the keys
    _, y1 = run(qb, kb, vb, H)
    _, y2 = run(qb, kb, vb, H)
    assert np.array_equal(y1, y2)
    ref64 = O.sage_attention(qb, kb, vb)
    check_output(y1.reshape(Tq, -1), ref64.reshape(Tq, -1), O.f64_to_bf16(ref64).reshape(Tq, -1))
    mean_v = O.bf16_to_f64(vb).astype(np.float16).astype(np.float64).mean(axis=0)
    assert np.allclose(ref64[3], mean_v, atol=1e-12)
