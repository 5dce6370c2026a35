"""GPU parity of the NVFP4 variant against the CPU oracle: the two-level FP4
quantiser bit for bit (E2M1 codes, E4M3 block scales in the tile-interleaved
layout, float32 tensor scale), and the block-scaled FP4 GEMM with its
epilogue within the stated output tolerance."""
import numpy as np
import pytest
import torch

import rotated_bit_dit_b200 as R
from oracle import rbd_oracle as O
from rotated_bit_dit_b200 import inputs as I
from tests.helpers import check_output, dev_bf16, host_u16

pytestmark = pytest.mark.gpu

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def e4m3_values(b: np.ndarray) -> np.ndarray:
    b = b.astype(np.int64)
    e, m = (b >> 3) & 15, b & 7
    return np.where(e > 0, (1 + m / 8.0) * np.exp2(e - 7.0), m * 2.0 ** -9)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    lo, hi = packed & 0xF, packed >> 4
    out = np.empty((packed.shape[0], packed.shape[1] * 2), np.float64)
    out[:, 0::2] = E2M1[lo]
    out[:, 1::2] = E2M1[hi]
    return out


def scales_from_tiles(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Tile-interleaved scale buffer -> [rows, K/16] bytes (the layout documented in rbd.h)."""
    r = np.arange(rows)[:, None]
    c = np.arange(K // 16)[None, :]
    off = (((r >> 7) * (K // 64) + (c >> 2)) * 32 + (r & 31)) * 16 + ((r & 127) >> 5) * 4 + (c & 3)
    return buf[off]


def gpu_quant(xb: np.ndarray, rot: int = 256):
    M, K = xb.shape
    x = dev_bf16(xb)
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    bs = torch.zeros((R.rbd_nvfp4_scale_bytes(M, K),), dtype=torch.uint8, device="cuda")
    gs = torch.empty((1,), dtype=torch.float32, device="cuda")
    work = torch.empty((1,), dtype=torch.int32, device="cuda")
    R.rbd_nvfp4_quant(x, codes, bs, gs, work, rot)
    assert R.rbd_check() == 0
    return codes, bs, gs


@pytest.mark.parametrize("M,K", [(64, 256), (37, 768), (130, 3072), (3, 12288)])
@pytest.mark.parametrize("rot", [256, 0])
def test_nvfp4_quant_bit_exact(M, K, rot):
    xb = I.gaussian_bf16(300 + M + K, (M, K), 1.0, 0.005, 30.0)
    codes, bs, gs = gpu_quant(xb, rot)
    ref_q, ref_bs, ref_gs = O.nvfp4_quantize(O.rotate(O.bf16_to_f64(xb), rot))
    assert gs.cpu().numpy().view(np.uint32)[0] == np.float32(ref_gs).view(np.uint32)
    got_q = unpack_codes(codes.cpu().numpy())
    assert np.array_equal(np.abs(got_q), np.abs(ref_q))
    nz = ref_q != 0
    assert np.array_equal(np.sign(got_q[nz]), np.sign(ref_q[nz]))
    got_bs = e4m3_values(scales_from_tiles(bs.cpu().numpy(), M, K))
    assert np.array_equal(got_bs, ref_bs)


def test_nvfp4_quant_zero_tensor():
    codes, bs, gs = gpu_quant(np.zeros((5, 512), np.uint16))
    assert gs.item() == 0.0
    assert not codes.cpu().numpy().any()
    assert not scales_from_tiles(bs.cpu().numpy(), 5, 512).any()


def run_linear(xb, wb, bias=None, gate_mode=0, gate_cols=(0, 0), gate=None, residual=None, l1=None, l2=None):
    M, K = xb.shape
    N = wb.shape[0]
    xq, xbs, xgs = gpu_quant(xb)
    wq, wbs, wgs = gpu_quant(wb)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dv = lambda a: None if a is None else dev_bf16(a)
    ld = l2t = None
    if l1 is not None:
        # the branch's first factor from the unrotated input, then L2 as the GEMM's second MMA
        r = l1.shape[1]
        ld = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
        R.rbd_lowrank_down(dev_bf16(xb), dev_bf16(np.ascontiguousarray(l1.T)), ld)
        l2t = dev_bf16(np.ascontiguousarray(l2.T))
    epi = R.make_epilogue(dv(bias), ld, l2t, gate_mode, gate_cols, dv(gate), dv(residual))
    R.rbd_nvfp4_linear(xq, xbs, xgs, wq, wbs, wgs, y, epi)
    assert R.rbd_check() == 0
    return host_u16(y)


def reference(xb, wb, **kw):
    y = O.nvfp4_linear(xb, wb)
    # the branch's first factor crosses the ABI as bf16 [M, r]; the oracle's own
    # value, rounded the same way, is what the GEMM receives
    ld = O.bf16_to_f64(O.f64_to_bf16(O.lowrank_down(xb, kw["l1"]))) if kw.get("l1") is not None else None
    y = O.epilogue(y, kw.get("bias"), ld, kw.get("l2"), kw.get("gate_mode", 0), kw.get("gate_cols", (0, 0)),
                   kw.get("gate"), kw.get("residual"))
    return y, O.f64_to_bf16(y)


CASES = {
    "plain": dict(),
    "bias": dict(bias=True),
    "sigmoid": dict(gate_mode=1),
    "gated_residual": dict(gate_mode=2),
    "rank16": dict(rank=16),
    "rank32": dict(rank=32),
    "rank64": dict(rank=64),
    "all": dict(bias=True, rank=32, gate_mode=1),
}


@pytest.mark.parametrize("case", list(CASES))
@pytest.mark.parametrize("M,N,K", [(64, 256, 256), (200, 384, 768), (333, 128, 1024)])
def test_nvfp4_linear_matches_oracle(case, M, N, K):
    xb = I.gaussian_bf16(400 + M, (M, K), 1.0, 0.005, 30.0)
    wb = I.gaussian_bf16(401 + N, (N, K), 0.02)
    kw = dict(CASES[case])
    if kw.get("gate_mode") == 1:
        kw["gate_cols"] = (N // 2, N)
    if kw.pop("bias", False):
        kw["bias"] = I.gaussian_bf16(402, (N,), 0.1)
    if kw.get("gate_mode") == 2:
        kw["gate"] = I.gaussian_bf16(403, (N,), 1.0)
        kw["residual"] = I.gaussian_bf16(404, (M, N), 1.0)
    rank = kw.pop("rank", 0)
    if rank:
        kw["l1"] = I.gaussian_bf16(405 + rank, (K, rank), 0.05)
        kw["l2"] = I.gaussian_bf16(406 + rank, (rank, N), 0.05)
    y = run_linear(xb, wb, **kw)
    ref64, ref_bf16 = reference(xb, wb, **kw)
    check_output(y, ref64, ref_bf16)


def test_nvfp4_linear_small_m_sweep_shape():
    # the small-M sweep's layer shape (K = N = 3072) at M = 1024, every row checked
    M, N, K = 1024, 3072, 3072
    xb = I.gaussian_bf16(410, (M, K), 1.0, 0.005, 30.0)
    wb = I.gaussian_bf16(411, (N, K), 0.02)
    y = run_linear(xb, wb)
    ref64, ref_bf16 = reference(xb, wb)
    stats = check_output(y, ref64, ref_bf16)
    assert stats["rel64"] < 5e-3


def test_nvfp4_linear_qkvg_shape_sampled_rows():
    # the Q|K|V|gate layer shape the NVFP4 sweep times (M = 4096, K = 3072, N = 12288, rank-32
    # branch, sigmoid on the last quarter), checked on sampled token rows.  The activation tensor
    # scale depends on every row, so both operands are quantised whole and only the product is
    # restricted to the sampled rows.
    cfg = I.CONFIGS["w4a4_qkvg"]
    t = I.make_layer_inputs(cfg, seed=0)
    M, N = cfg["M"], cfg["N"]
    kw = dict(l1=t["l1"], l2=t["l2"], gate_mode=1, gate_cols=cfg["gate_cols"])
    y = run_linear(t["x"], t["w"], **kw)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 40, replace=False)]))
    xq, xbs, xgs = O.nvfp4_quantize(O.rotate(O.bf16_to_f64(t["x"])))
    wq, wbs, wgs = O.nvfp4_quantize(O.rotate(O.bf16_to_f64(t["w"])))
    xd = xq[rows] * np.repeat(xbs[rows], 16, axis=1) * float(xgs)
    wd = wq * np.repeat(wbs, 16, axis=1) * float(wgs)
    ld = O.bf16_to_f64(O.f64_to_bf16(O.lowrank_down(t["x"][rows], t["l1"])))
    ref64 = O.epilogue(xd @ wd.T, None, ld, t["l2"], 1, cfg["gate_cols"])
    stats = check_output(y[rows], ref64, O.f64_to_bf16(ref64))
    assert stats["rel64"] < 5e-3


def test_nvfp4_linear_low_rank_branch_is_added():
    # the branch must change the output by exactly its own contribution (within tolerance):
    # the same layer with L2 = 0 gives the plain result
    M, N, K, r = 96, 256, 512, 32
    xb = I.gaussian_bf16(420, (M, K), 1.0, 0.005, 30.0)
    wb = I.gaussian_bf16(421, (N, K), 0.02)
    l1 = I.gaussian_bf16(422, (K, r), 0.05)
    zero = np.zeros((r, N), np.uint16)
    assert np.array_equal(run_linear(xb, wb, l1=l1, l2=zero), run_linear(xb, wb))
    l2 = I.gaussian_bf16(423, (r, N), 0.05)
    y = run_linear(xb, wb, l1=l1, l2=l2)
    ref64, ref_bf16 = reference(xb, wb, l1=l1, l2=l2)
    check_output(y, ref64, ref_bf16)


@pytest.mark.parametrize("r", [16, 32, 64])
@pytest.mark.parametrize("M,K", [(1, 3072), (45, 256), (300, 1024)])
def test_lowrank_down_alone(r, M, K):
    xb = I.gaussian_bf16(430 + M, (M, K), 1.0, 0.005, 30.0)
    l1b = I.gaussian_bf16(431 + r, (K, r), 0.01)
    ld = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    R.rbd_lowrank_down(dev_bf16(xb), dev_bf16(np.ascontiguousarray(l1b.T)), ld)
    assert R.rbd_check() == 0
    ref = O.lowrank_down(xb, l1b)
    err = np.abs(ld.float().cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= np.abs(ref) * 2.0 ** -8 + 1e-4 * np.abs(ref).max())
