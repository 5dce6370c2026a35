"""Pins of the CPU oracle against facts the mathematics fixes (no GPU).

Each test is chosen so that a plausible slip in the oracle (a wrong Hadamard
construction, a transposed operand, a dropped 1/16, a wrong tie rule, a lost
scale, a wrong nibble order, a sign error in the epilogue) fails at least one.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import rbd_oracle as O
from rotated_bit_dit_b200 import inputs as I

H = O.hadamard_regular_kron()


# --------------------------------------------------------------- Hadamard
def test_hadamard_entries_and_orthogonality():
    assert set(np.unique(H)) == {-1, 1}
    assert np.array_equal(H @ H.T, 256 * np.eye(256, dtype=np.int64))


def test_hadamard_symmetric_and_regular():
    assert np.array_equal(H, H.T)
    # regular: every row (and column) sums to sqrt(256) = 16
    assert np.all(H.sum(axis=1) == 16) and np.all(H.sum(axis=0) == 16)


def test_hadamard_two_constructions_agree():
    assert np.array_equal(H, O.hadamard_regular_digits())


def test_hadamard_order4_is_J_minus_2I():
    h4 = O.hadamard_regular_kron(4)
    assert np.array_equal(h4, np.array([[-1, 1, 1, 1], [1, -1, 1, 1], [1, 1, -1, 1], [1, 1, 1, -1]]))


def test_sylvester_is_a_different_reading():
    s = O.hadamard_sylvester()
    assert np.array_equal(s @ s.T, 256 * np.eye(256, dtype=np.int64))
    assert not np.array_equal(s, H)
    # Sylvester is not regular: its row sums are 256, 0, 0, ...
    assert s.sum(axis=1)[0] == 256 and s.sum(axis=1)[1] == 0


# --------------------------------------------------------------- rotation
def _rand_bf16(seed, shape, std=1.0, frac=0.0, scale=1.0):
    return O.bf16_to_f64(I.gaussian_bf16(seed, shape, std, frac, scale))


def test_rotation_constant_block_is_fixed_point():
    # regularity: R (c 1) = c 1 (each column of H sums to 16)
    for c in (1.0, -3.5, 0.015625):
        x = np.full((1, 256), c)
        assert np.array_equal(O.rotate(x), np.full((1, 256), c, dtype=np.float32))
    # the Sylvester reading maps a constant block to (16c, 0, 0, ...)
    s = O.hadamard_sylvester().astype(np.float64) / 16
    y = np.full((1, 256), 2.0) @ s
    assert y[0, 0] == 32.0 and np.all(y[0, 1:] == 0)


def test_rotation_unit_vector_is_a_column_over_16():
    for j in (0, 5, 255):
        x = np.zeros((1, 256))
        x[0, j] = 1.0
        y = O.rotate(x)[0]
        assert np.array_equal(y, (H[:, j] / 16.0).astype(np.float32))
        assert set(np.abs(y)) == {np.float32(1 / 16)}


def test_rotation_is_an_involution_in_float64():
    # R = R^T and R R^T = I, so rotating twice returns the input exactly
    x = _rand_bf16(11, (4, 512))
    r = O.rotation_matrix()
    xg = x.reshape(4, 2, 256)
    assert np.array_equal(np.matmul(np.matmul(xg, r), r), xg)


def test_rotation_groups_are_independent_blocks():
    x = _rand_bf16(12, (3, 768))
    y = O.rotate(x)
    for g in range(3):
        assert np.array_equal(y[:, 256 * g:256 * (g + 1)], O.rotate(x[:, 256 * g:256 * (g + 1)]))


def test_rotation_matches_exact_rationals():
    # brute force: exact rational sum, rounded once to float32
    x = _rand_bf16(13, (2, 256), 1.0, 0.05, 30.0)
    got = O.rotate(x)
    for r in range(2):
        assert np.array_equal(got[r], O.rotate_exact_fraction(x[r]))


def test_rotation_wide_exponent_span_uses_exact_path():
    # a group whose exponent span exceeds the float64 exactness bound
    x = np.zeros((1, 256))
    x[0, 0] = 2.0 ** 60
    x[0, 1] = 2.0 ** -40 * 1.5
    x[0, 2] = 3.0
    assert not O._group_span_ok(x.reshape(1, 1, 256)).all()
    assert np.array_equal(O.rotate(x)[0], O.rotate_exact_fraction(x[0]))


def test_rotation_preserves_products_before_quantisation():
    # X W^T = (X R)(W R)^T per block, float64, to 1e-12 relative
    x = _rand_bf16(14, (8, 512), 1.0, 0.01, 20.0)
    w = _rand_bf16(15, (16, 512), 0.02)
    r = O.rotation_matrix()
    xr = np.matmul(x.reshape(8, 2, 256), r).reshape(8, 512)
    wr = np.matmul(w.reshape(16, 2, 256), r).reshape(16, 512)
    ref = x @ w.T
    assert np.max(np.abs(xr @ wr.T - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_no_rotation_mode_is_identity():
    x = _rand_bf16(16, (2, 256))
    assert np.array_equal(O.rotate(x, 0), x.astype(np.float32))


# --------------------------------------------------------------- quantiser
@pytest.mark.parametrize("bits", [4, 8])
def test_quantiser_is_nearest_code_with_even_ties(bits):
    qmax = O.qmax_of(bits)
    xr = O.rotate(_rand_bf16(17, (16, 256), 1.0, 0.02, 20.0))
    q, s = O.quantize(xr, bits)
    codes = np.arange(-qmax - 1, qmax + 1)
    for m in range(xr.shape[0]):
        amax = np.float32(np.abs(xr[m]).max())
        inv = np.float32(np.float32(qmax) / amax)
        assert s[m] == np.float32(amax / np.float32(qmax))
        t = (xr[m] * inv).astype(np.float32).astype(np.float64)
        d = np.abs(t[:, None] - codes[None, :])
        best = d.min(axis=1, keepdims=True)
        cand = np.where(d == best, codes[None, :], 10 ** 6)
        # ties: prefer the even code
        even = np.where((cand % 2 == 0) & (cand != 10 ** 6), cand, 10 ** 6).min(axis=1)
        first = cand.min(axis=1)
        expect = np.where((d == best).sum(axis=1) > 1, even, first)
        assert np.array_equal(q[m].astype(np.int64), expect)


def test_quantiser_error_bound():
    for bits in (4, 8):
        xr = O.rotate(_rand_bf16(18, (32, 512), 1.0, 0.01, 30.0))
        q, s = O.quantize(xr, bits)
        err = np.abs(xr.astype(np.float64) - q.astype(np.float64) * s[:, None].astype(np.float64))
        assert np.all(err <= s[:, None] / 2 * (1 + 2.0 ** -20))


def test_quantiser_range_and_extremes():
    xr = O.rotate(_rand_bf16(19, (8, 256)))
    q, s = O.quantize(xr, 4)
    assert q.min() >= -7 and q.max() <= 7          # -8 is never produced by symmetric scaling
    amax_idx = np.abs(xr).argmax(axis=1)
    assert np.all(np.abs(q[np.arange(8), amax_idx]) == 7)


def test_quantiser_half_way_ties():
    # amax = 7 -> inv = 1: values k + 0.5 must go to the even neighbour
    xr = np.zeros((1, 256), dtype=np.float32)
    xr[0, :8] = [7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5]
    q, s = O.quantize(xr, 4)
    assert s[0] == 1.0
    assert list(q[0, :8]) == [7, 0, 2, 2, 0, -2, -2, 4]


def test_zero_row_and_zero_group():
    xr = np.zeros((2, 128), dtype=np.float32)
    xr[1, 64:] = 1.0
    q, s = O.quantize(xr, 4, scale_group=64)
    assert np.all(q[0] == 0) and np.all(s[0] == 0)
    assert s[1, 0] == 0 and np.all(q[1, :64] == 0)
    assert s[1, 1] == np.float32(1 / np.float32(7)) and np.all(q[1, 64:] == 7)


def test_group_scales_equal_row_scale_when_groups_share_amax():
    xr = np.tile(np.linspace(-1, 1, 64, dtype=np.float32), (3, 4))
    q_row, s_row = O.quantize(xr, 4)
    q_g, s_g = O.quantize(xr, 4, scale_group=64)
    assert np.array_equal(q_row, q_g)
    assert np.all(s_g == s_row[:, None])


# --------------------------------------------------------------- packing
def test_pack_nibble_order_and_twos_complement():
    q = np.array([[1, -1, 7, -8, 0, 3]], dtype=np.int8)
    p = O.pack_int4(q)
    # byte 0: low nibble k=0 (1), high nibble k=1 (-1 -> 0xF) -> 0xF1
    assert list(p[0]) == [0xF1, 0x87, 0x30]
    assert np.array_equal(O.unpack_int4(p), q)


def test_pack_roundtrip_all_codes():
    q = np.array([np.arange(-8, 8)] * 2, dtype=np.int8)
    assert np.array_equal(O.unpack_int4(O.pack_int4(q)), q)


# --------------------------------------------------------------- GEMM
def test_gemm_matches_loops_on_tiny_shapes():
    rng = np.random.default_rng(0)
    qx = rng.integers(-8, 8, (3, 256)).astype(np.int8)
    qw = rng.integers(-8, 8, (4, 256)).astype(np.int8)
    assert np.array_equal(O.gemm_acc(qx, qw), O.gemm_acc_loops(qx, qw))


def test_gemm_hand_expanded():
    qx = np.array([[1, 2, 3, 4]], dtype=np.int8)
    qw = np.array([[1, 0, -1, 2], [7, 7, 7, 7]], dtype=np.int8)
    assert O.gemm_acc(qx, qw).tolist() == [[1 - 3 + 8, 70]]


def test_unrotated_integer_inputs_reduce_to_integer_matmul():
    # rot_group=0, integer inputs in [-7,7] whose row amax is 7: scales are 1, codes = inputs
    rng = np.random.default_rng(1)
    xi = rng.integers(-7, 8, (5, 64)).astype(np.float64)
    wi = rng.integers(-7, 8, (6, 64)).astype(np.float64)
    xi[:, 0] = 7
    wi[:, 0] = 7
    xb = I.f32_to_bf16_bits(xi.astype(np.float32))
    wb = I.f32_to_bf16_bits(wi.astype(np.float32))
    out = O.linear_reference(xb, wb, 4, rot_group=0)
    assert np.all(out["sx"] == 1) and np.all(out["sw"] == 1)
    assert np.array_equal(out["y64"], xi @ wi.T)


def test_group_partials_sum_to_row_accumulator():
    rng = np.random.default_rng(2)
    qx = rng.integers(-7, 8, (4, 256)).astype(np.int8)
    qw = rng.integers(-7, 8, (5, 256)).astype(np.int8)
    assert np.array_equal(O.gemm_acc_grouped(qx, qw, 64).sum(axis=0), O.gemm_acc(qx, qw))
    ones_x = np.ones((4, 4), np.float32)
    ones_w = np.ones((5, 4), np.float32)
    assert np.allclose(O.dequant(qx, ones_x, qw, ones_w, 64), O.gemm_acc(qx, qw))


def test_dequant_scales_each_operand_once():
    rng = np.random.default_rng(3)
    qx = rng.integers(-7, 8, (2, 64)).astype(np.int8)
    qw = rng.integers(-7, 8, (3, 64)).astype(np.int8)
    sx = np.array([2.0, 0.5], np.float32)
    sw = np.array([1.0, 4.0, 0.25], np.float32)
    acc = O.gemm_acc(qx, qw)
    assert np.array_equal(O.dequant(qx, sx, qw, sw), acc * np.outer(sx, sw))


# --------------------------------------------------------------- epilogue
def test_epilogue_special_cases():
    rng = np.random.default_rng(4)
    y = rng.standard_normal((4, 8))
    res = I.gaussian_bf16(5, (4, 8))
    zero_g = np.zeros(8, dtype=np.uint16)
    # g = 0: out = residual
    assert np.array_equal(O.epilogue(y, gate_mode=2, gate_bits=zero_g, residual_bits=res), O.bf16_to_f64(res))
    # g = 1, residual = 0: out = y
    one_g = I.f32_to_bf16_bits(np.ones(8, np.float32))
    zres = np.zeros((4, 8), np.uint16)
    assert np.array_equal(O.epilogue(y, gate_mode=2, gate_bits=one_g, residual_bits=zres), y)
    # L2 = 0 leaves y unchanged; bias adds per column
    ld = rng.standard_normal((4, 2))
    assert np.array_equal(O.epilogue(y, ld=ld, l2_bits=np.zeros((2, 8), np.uint16)), y)
    b = I.f32_to_bf16_bits(np.arange(8, dtype=np.float32))
    assert np.array_equal(O.epilogue(y, bias=b), y + np.arange(8)[None, :])
    # sigmoid on the gate columns only; sigmoid(0) = 1/2 exactly
    z = np.zeros((2, 8))
    out = O.epilogue(z, gate_mode=1, gate_cols=(4, 8))
    assert np.all(out[:, 4:] == 0.5) and np.all(out[:, :4] == 0.0)


def test_epilogue_sigmoid_values_symmetry_and_sign():
    # closed forms: sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4; a sign slip inside the
    # exponential swaps them, which the value at 0 alone cannot show
    y = np.array([[math.log(3.0), -math.log(3.0), 0.0, math.log(9.0)]])
    out = O.epilogue(y, gate_mode=1, gate_cols=(0, 4))
    assert np.allclose(out, [[0.75, 0.25, 0.5, 0.9]], rtol=0, atol=1e-15)
    rng = np.random.default_rng(41)
    v = rng.standard_normal((6, 40)) * 4.0
    s_pos = O.epilogue(v, gate_mode=1, gate_cols=(0, 40))
    s_neg = O.epilogue(-v, gate_mode=1, gate_cols=(0, 40))
    # sigmoid(-y) = 1 - sigmoid(y)
    assert np.allclose(s_neg, 1.0 - s_pos, rtol=0, atol=1e-15)
    # strictly increasing in y, inside (0, 1), above 1/2 exactly where y > 0
    order = np.argsort(v.ravel())
    assert np.all(np.diff(s_pos.ravel()[order]) >= 0)
    assert np.all((s_pos > 0) & (s_pos < 1))
    assert np.array_equal(s_pos > 0.5, v > 0)
    # the gate applies to the gate columns only, after bias is added
    b = I.f32_to_bf16_bits(np.full(8, 2.0, np.float32))
    z = np.zeros((1, 8))
    g = O.epilogue(z, bias=b, gate_mode=1, gate_cols=(6, 8))
    assert np.allclose(g[0, 6:], 1.0 / (1.0 + math.exp(-2.0)), rtol=0, atol=1e-15)
    assert np.array_equal(g[0, :6], np.full(6, 2.0))


def test_lowrank_branch_is_parallel_linear():
    # (W + L1 L2)-style branch: X L1 L2 added once, on the unrotated input
    x = I.gaussian_bf16(6, (3, 256))
    l1 = I.gaussian_bf16(7, (256, 4), 0.1)
    l2 = I.gaussian_bf16(8, (4, 5), 0.1)
    ld = O.lowrank_down(x, l1)
    xd, l1d, l2d = O.bf16_to_f64(x), O.bf16_to_f64(l1), O.bf16_to_f64(l2)
    assert np.allclose(O.epilogue(np.zeros((3, 5)), ld=ld, l2_bits=l2), xd @ (l1d @ l2d), rtol=1e-12, atol=1e-15)


def test_bf16_rounding_ties_and_against_torch():
    # direct float64 -> bf16, nearest even; compare with torch on float32-exact values
    rng = np.random.default_rng(5)
    v = rng.standard_normal(20000).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.f64_to_bf16(v), ref)
    # exact ties: 1 + 2^-8 lies half-way between 1 and 1 + 2^-7 -> 1 (even)
    assert O.f64_to_bf16(np.array([1 + 2.0 ** -8]))[0] == 0x3F80
    assert O.f64_to_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 0x3F82
    # a value just above the tie in float64 (not representable in float32) rounds up
    assert O.f64_to_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -40]))[0] == 0x3F81


def test_end_to_end_tiny_layer_matches_float_reference():
    # at 4 bits the quantised layer stays close to the float layer (sanity of scale placement)
    cfg = I.CONFIGS["tiny_w4a4"]
    t = I.make_layer_inputs(cfg, seed=0)
    out = O.linear_reference(t["x"], t["w"], 4)
    ref = O.bf16_to_f64(t["x"]) @ O.bf16_to_f64(t["w"]).T
    rel = np.linalg.norm(out["y64"] - ref) / np.linalg.norm(ref)
    assert rel < 0.25
    # and reconstructing from codes reproduces y64
    qw = O.unpack_int4(out["wq"])
    xd = out["codes"].astype(np.float64) * out["sx"].astype(np.float64)[:, None]
    wd = qw.astype(np.float64) * out["sw"].astype(np.float64)[:, None]
    assert np.allclose(out["y64"], xd @ wd.T, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------- NVFP4
def test_e2m1_rounding_brute_force():
    grid = np.concatenate([-O.E2M1_GRID[::-1], O.E2M1_GRID])
    enc = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    vals = np.concatenate([np.linspace(-7, 7, 2801), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]])
    got = O.round_e2m1(vals)
    for v, g in zip(vals, got):
        a = min(abs(v), 6.0)
        d = np.abs(np.abs(grid) - a)
        best = d.min()
        cands = sorted({abs(float(x)) for x in grid[d == best]})
        pick = cands[0] if len(cands) == 1 else [c for c in cands if enc[c] % 2 == 0][0]
        assert abs(g) == pick and (g == 0 or np.sign(g) == np.sign(v))


def test_e4m3_rounding_against_torch():
    rng = np.random.default_rng(6)
    v = np.concatenate([rng.standard_normal(20000) * 50, rng.standard_normal(2000) * 1e-2,
                        [448.0, -448.0, 0.0, 2.0 ** -9, 3 * 2.0 ** -10]]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    sel = np.abs(v) <= 448
    assert np.array_equal(O.round_e4m3(v.astype(np.float64))[sel], ref[sel])
    assert np.all(O.round_e4m3(np.array([1000.0, -500.0])) == [448.0, -448.0])


def test_nvfp4_block_error_bound_and_scale_range():
    xr = O.rotate(_rand_bf16(20, (8, 512), 1.0, 0.01, 30.0))
    q, bs, gs = O.nvfp4_quantize(xr)
    deq = q * np.repeat(bs, 16, axis=1) * float(gs)
    assert np.all(bs <= 448) and np.all(bs >= 0)
    # the block holding the tensor amax has scale 448 (up to E4M3 rounding of the ratio)
    assert bs.max() == 448.0
    # error within half a grid step at the largest step (2 * bs * gs) per element, plus scale rounding
    step = 2.0 * np.repeat(bs, 16, axis=1) * float(gs)
    assert np.all(np.abs(xr - deq) <= step / 2 * 1.0001 + 1e-30)
    rel = np.linalg.norm(xr - deq) / np.linalg.norm(xr)
    assert rel < 0.12


def _nvfp4_exact_operand(seed, rows, k, tensor_scale):
    """bf16 rows whose 16-blocks are E2M1 grid values times one E4M3 block scale times a
    power-of-two tensor scale; every block holds a +-6 and one block has scale 448, so the
    two-level quantiser reproduces them exactly."""
    rng = np.random.default_rng(seed)
    grid = np.concatenate([-O.E2M1_GRID[1:], O.E2M1_GRID])
    e4m3 = np.array([0.125, 0.25, 0.375, 0.5, 0.75, 1.0, 1.25, 2.5, 3.0, 6.5, 13.0, 24.0, 104.0, 448.0])
    q = rng.choice(grid, (rows, k // 16, 16))
    q[:, :, 0] = rng.choice([-6.0, 6.0], (rows, k // 16))
    bs = rng.choice(e4m3, (rows, k // 16))
    bs[0, 0] = 448.0
    v = (q * bs[..., None] * tensor_scale).reshape(rows, k)
    bits = I.f32_to_bf16_bits(v.astype(np.float32))
    assert np.array_equal(O.bf16_to_f64(bits), v)            # exactly representable
    return bits


def test_nvfp4_linear_exact_on_representable_operands():
    # unrotated, operands already on the two-level NVFP4 grid: the layer must return the
    # plain float64 product exactly (catches a tensor scale applied once instead of twice,
    # a block scale repeated wrongly, or a transposed operand)
    x = _nvfp4_exact_operand(50, 5, 64, 2.0 ** -3)
    w = _nvfp4_exact_operand(51, 7, 64, 2.0 ** -9)
    got = O.nvfp4_linear(x, w, rot_group=0)
    want = O.bf16_to_f64(x) @ O.bf16_to_f64(w).T
    assert np.array_equal(got, want)


def test_nvfp4_linear_rotated_within_the_quantisation_bound():
    # with rotation both operands are rotated: X W^T = (XR)(WR)^T, so the result stays within the
    # per-element half-step bound of the unrotated float64 product.  W holds X's own rows, so the
    # diagonal is the large |x|^2; forgetting to rotate W would leave (XR) W^T, outside the bound
    x = I.gaussian_bf16(52, (6, 512), 1.0, 0.01, 30.0)
    w = np.concatenate([x, I.gaussian_bf16(53, (3, 512), 0.02)])
    got = O.nvfp4_linear(x, w)
    xr, wr = O.rotate(O.bf16_to_f64(x)), O.rotate(O.bf16_to_f64(w))
    qx, bsx, gsx = O.nvfp4_quantize(xr)
    qw, bsw, gsw = O.nvfp4_quantize(wr)
    hx = np.repeat(bsx, 16, axis=1) * float(gsx)       # half of the largest grid step, per element
    hw = np.repeat(bsw, 16, axis=1) * float(gsw)
    bound = hx @ (np.abs(wr) + hw).T + np.abs(xr) @ hw.T
    exact = O.bf16_to_f64(x) @ O.bf16_to_f64(w).T
    assert np.all(np.abs(got - exact) <= bound * (1 + 1e-9) + 1e-12)
    # the test has the power to see the slip: W quantised unrotated breaks the bound
    qu, bsu, gsu = O.nvfp4_quantize(O.bf16_to_f64(w))
    slip = (qx * hx) @ (qu * np.repeat(bsu, 16, axis=1) * float(gsu)).T
    assert np.any(np.abs(slip - exact) > bound)


# --------------------------------------------------------------- normalising prologue
def _bits(a) -> np.ndarray:
    return (np.asarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_norm_hand_worked_example():
    # x = (3, 4): mean square 12.5, r = 1/sqrt(12.5) -> u = (0.848528, 1.131371);
    # 1 + scale = (2, 1), shift = (0.5, -1): v = (2.197056, 0.131371) -> bf16
    # 2.203125 (1.1015625 * 2) and 0.1318359375 (1.0546875 / 8)
    out = O.bf16_to_f64(O.norm_modulate(_bits([[3.0, 4.0]]), None, _bits([0.5, -1.0]), _bits([1.0, 0.0]), 0.0))
    assert out.tolist() == [[2.203125, 0.1318359375]]


def test_norm_power_of_two_scale_invariance():
    # without eps, scaling a row by 2^j changes nothing, bit for bit (catches a
    # missing square root or a wrong power of the mean)
    xb = I.gaussian_bf16(30, (6, 512), 1.0, 0.01, 20.0)
    base = O.norm_modulate(xb, eps=0.0)
    for j in (-7, 3, 20):
        scaled = _bits(O.bf16_to_f64(xb) * 2.0 ** j)
        assert np.array_equal(O.norm_modulate(scaled, eps=0.0), base)
    # with eps the invariance is gone: eps is added to the mean square
    assert not np.array_equal(O.norm_modulate(_bits(O.bf16_to_f64(xb) * 2.0 ** -12), eps=1e-3), base)


def test_norm_unit_rms_and_constant_rows():
    xb = I.gaussian_bf16(31, (5, 3072), 1.0, 0.005, 30.0)
    u = O.bf16_to_f64(O.norm_modulate(xb, eps=0.0))
    # mean of squares is 1 up to the bf16 rounding of each element (catches sum-instead-of-mean)
    assert np.all(np.abs((u ** 2).mean(axis=1) - 1.0) < 2.0 ** -7)
    # a constant row normalises to +-1 exactly; a zero row stays zero
    const = np.full((3, 256), 3.0, np.float32)
    const[1] = -0.375
    const[2] = 0.0
    c = O.bf16_to_f64(O.norm_modulate(_bits(const), eps=0.0))
    assert np.all(c[0] == 1.0) and np.all(c[1] == -1.0) and np.all(c[2] == 0.0)


def test_norm_matches_float64_formula_and_each_vector_acts_per_channel():
    xb = I.gaussian_bf16(32, (7, 768), 1.0, 0.01, 25.0)
    gamma = _bits(1.0 + O.bf16_to_f64(I.gaussian_bf16(33, (768,), 0.1)))
    shift, scale = I.gaussian_bf16(34, (768,), 0.5), I.gaussian_bf16(35, (768,), 0.3)
    x = O.bf16_to_f64(xb)
    ref = (x / np.sqrt((x ** 2).mean(axis=1, keepdims=True) + 1e-6) * O.bf16_to_f64(gamma)
           * (1.0 + O.bf16_to_f64(scale)) + O.bf16_to_f64(shift))
    got = O.bf16_to_f64(O.norm_modulate(xb, gamma, shift, scale, 1e-6))
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-6)
    # swapping shift and scale (or dropping one) is detected
    swapped = O.bf16_to_f64(O.norm_modulate(xb, gamma, scale, shift, 1e-6))
    assert np.abs(swapped - ref).max() > 0.1


def test_norm_rot_quant_is_the_composition():
    xb = I.gaussian_bf16(36, (4, 512), 1.0, 0.01, 30.0)
    shift = I.gaussian_bf16(37, (512,), 0.2)
    q, s = O.norm_rot_quant(xb, 4, 256, 64, None, shift, None, 1e-6)
    q2, s2 = O.rot_quant(O.norm_modulate(xb, None, shift, None, 1e-6), 4, 256, 64)
    assert np.array_equal(q, q2) and np.array_equal(s, s2)


# --------------------------------------------------------------- INT4 KV-cache codec
def test_kv4_groups_follow_the_rotary_bands():
    for n in (1, 2, 4):
        sizes = O.kv4_group_sizes(n)
        edges = set(np.cumsum([0] + sizes).tolist())
        assert len(sizes) == 3 * n and sum(sizes) == 128
        assert {0, 44, 86, 128} <= edges           # no group straddles the 44 | 42 | 42 split
        assert max(sizes) - min(sizes) <= 1 + (44 - 42) // n


def test_kv4_hand_worked_head():
    # time band 7.0 -> scale 1, code 7; height band -3.5 -> scale 0.5, code -7; width band 0
    x = np.zeros((1, 1, 128), np.float32)
    x[0, 0, :44] = 7.0
    x[0, 0, 44:86] = -3.5
    xb = I.f32_to_bf16_bits(x)
    packed, scales = O.kv4_encode(xb, 1)
    assert scales.tolist() == [[[1.0, 0.5, 0.0]]]
    assert np.all(packed[0, 0, :22] == 0x77) and np.all(packed[0, 0, 22:43] == 0x99)
    assert np.all(packed[0, 0, 43:] == 0x00)
    assert np.array_equal(O.kv4_decode(packed, scales, 1), xb)


def test_kv4_band_isolation_and_error_bound():
    xb = I.gaussian_bf16(50, (5, 3, 128), 1.0)
    spiked = O.bf16_to_f64(xb).copy()
    spiked[:, :, 60] *= 1000.0                       # inside the height band
    sb = O.f64_to_bf16(spiked)
    for n in (1, 2, 4):
        p0, s0 = O.kv4_encode(xb, n)
        p1, s1 = O.kv4_encode(sb, n)
        sizes = O.kv4_group_sizes(n)
        gh = np.searchsorted(np.cumsum(sizes), 60, side="right")   # the group holding channel 60
        keep = [g for g in range(len(sizes)) if g != gh]
        assert np.array_equal(s0[:, :, keep], s1[:, :, keep])
        c0 = int(np.sum(sizes[:gh]))
        q0 = O.unpack_int4(p0.reshape(15, 64)).reshape(5, 3, 128)
        q1 = O.unpack_int4(p1.reshape(15, 64)).reshape(5, 3, 128)
        outside = np.r_[0:c0, c0 + sizes[gh]:128]
        assert np.array_equal(q0[:, :, outside], q1[:, :, outside])
        # reconstruction within half a step (plus the bf16 rounding of the product)
        y = O.bf16_to_f64(O.kv4_decode(p0, s0, n))
        s = np.repeat(s0, sizes, axis=2)
        assert np.all(np.abs(y - O.bf16_to_f64(xb)) <= s / 2 + np.abs(y) * 2.0 ** -8 + 1e-30)


# --------------------------------------------------------------- offline SVDQuant fit
def _lowrank_plus_noise(seed, n=64, k=256, r=8, noise=0.01):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((n, r)) @ rng.standard_normal((r, k)) * 0.05 + noise * rng.standard_normal((n, k))
    return O.f64_to_bf16(w)


@pytest.mark.parametrize("bits,sg", [(4, 0), (4, 64), (8, 0)])
def test_weight_dequantisation_error_bound(bits, sg):
    wb = I.gaussian_bf16(60, (32, 512), 0.02)
    q, s = O.quantize_weights(wb, bits, 256, sg)
    deq = O.dequantize_weights(q, s, bits, 256, sg)
    # R is orthonormal: the Frobenius error equals the rotated-domain error, at most half a step per element
    step = np.repeat(s, sg, axis=1) if sg else np.repeat(s[:, None], 512, axis=1)
    assert np.linalg.norm(O.bf16_to_f64(wb) - deq) <= np.linalg.norm(step / 2) * 1.0001 + 1e-12


def test_randomized_svd_exact_rank_and_eckart_young():
    rng = np.random.default_rng(61)
    a = rng.standard_normal((80, 6)) @ rng.standard_normal((6, 200))
    u, s, vt = O.randomized_svd(a, 6, rng.standard_normal((200, 14)))
    assert np.linalg.norm(a - (u * s) @ vt) <= 1e-10 * np.linalg.norm(a)
    # a spectral gap after rank 5: the sketch reaches the optimal truncation error
    uu, _ = np.linalg.qr(rng.standard_normal((80, 80)))
    vv, _ = np.linalg.qr(rng.standard_normal((200, 80)))
    sig = np.concatenate([[100, 80, 60, 40, 20], 0.01 * np.ones(75)])
    b = (uu * sig) @ vv.T
    u, s, vt = O.randomized_svd(b, 5, rng.standard_normal((200, 15)))
    optimal = np.sqrt((sig[5:] ** 2).sum())
    assert abs(np.linalg.norm(b - (u * s) @ vt) - optimal) <= 1e-6 * optimal
    assert np.allclose(s, sig[:5], rtol=1e-9)


def test_svdquant_fit_keeps_the_best_and_never_does_worse_than_the_single_shot():
    wb = _lowrank_plus_noise(62)
    rng = np.random.default_rng(63)
    omegas = [rng.standard_normal((256, 16)) for _ in range(4)]
    single = O.svdquant_fit(wb, 8, 4, omegas[:1])
    refined = O.svdquant_fit(wb, 8, 4, omegas)
    assert single["err"] == refined["errs"][0]          # iteration one is the single-shot split
    assert refined["err"] == min(refined["errs"]) <= single["err"]
    # the kept factors and codes reproduce the kept error
    w = O.bf16_to_f64(wb)
    deq = O.dequantize_weights(refined["q"], refined["scales"], 4)
    assert np.isclose(np.linalg.norm(w - (deq + (refined["l1"] @ refined["l2"]).T)), refined["err"], rtol=1e-9)
    # the branch carries the low-rank part: far below quantising W alone
    q, s = O.quantize_weights(wb, 4)
    assert refined["err"] < 0.2 * np.linalg.norm(w - O.dequantize_weights(q, s, 4))


def test_svdquant_activation_weights():
    # mean-1 normalisation, then the 0.05 floor for a dead channel
    d = O.act_weights(np.r_[0.0, np.ones(255)])
    assert d[0] == 0.05 and np.allclose(d[1:], 256 / 255)
    wb = _lowrank_plus_noise(64)
    rng = np.random.default_rng(65)
    omegas = [rng.standard_normal((256, 16)) for _ in range(2)]
    plain = O.svdquant_fit(wb, 8, 4, omegas)
    const = O.svdquant_fit(wb, 8, 4, omegas, act_rms=np.full(256, 2.0))   # constant RMS: weights exactly 1
    assert plain["errs"] == const["errs"] and np.array_equal(plain["q"], const["q"])
    # competing structure: a rank-4 part in channels 0-31 and a larger rank-4 part in the others.
    # With a rank-4 budget the plain fit's branch takes the larger part; weighting channels 0-31
    # by 8 moves the branch onto them.  (The total error there need not drop: the residual's
    # per-row scale then carries the large part, which a weighting of the branch cannot change.)
    r4 = np.random.default_rng(66)
    w = np.zeros((64, 256))
    w[:, :32] = r4.standard_normal((64, 4)) @ r4.standard_normal((4, 32)) * 0.03
    w[:, 32:] = r4.standard_normal((64, 4)) @ r4.standard_normal((4, 224)) * 0.06
    cb = O.f64_to_bf16(w + 1e-3 * r4.standard_normal((64, 256)))
    rms = np.ones(256)
    rms[:32] = 8.0
    om4 = [r4.standard_normal((256, 12)) for _ in range(2)]
    wc = O.bf16_to_f64(cb)
    def branch_miss(fit):           # how far the branch is from the heavy channels' structure
        return np.linalg.norm(wc[:, :32] - (fit["l1"] @ fit["l2"]).T[:, :32])
    assert branch_miss(O.svdquant_fit(cb, 4, 4, om4, act_rms=rms)) < 0.5 * branch_miss(O.svdquant_fit(cb, 4, 4, om4))


# --------------------------------------------------------------- Q/K RMSNorm + RoPE, quantized attention
def _rope_apply(u, cos, sin):
    """Turn pairs of a float64 [T, D] by complex multiplication (an independent form of the rotation)."""
    z = (u[:, 0::2] + 1j * u[:, 1::2]) * (cos + 1j * sin)
    out = np.empty_like(u)
    out[:, 0::2], out[:, 1::2] = z.real, z.imag
    return out


def test_rope_tables_bands_and_first_pairs():
    cos, sin = O.rope_tables(np.array([[0, 0, 0], [1, 0, 0], [0, 2, 0], [0, 0, 3]]))
    assert np.array_equal(cos[0], np.ones(64)) and np.array_equal(sin[0], np.zeros(64))
    # position 1 on the time axis turns only the 22 pairs of the 44-channel band, its first pair by 1 rad
    assert np.all(sin[1, :22] > 0) and not sin[1, 22:].any()
    assert cos[1, 0] == np.cos(1.0) and sin[1, 0] == np.sin(1.0)
    # the height band holds pairs 22..42, the width band pairs 43..63; their first pairs turn by pos rad
    assert not sin[2, :22].any() and np.all(sin[2, 22:43] != 0) and not sin[2, 43:].any()
    assert sin[2, 22] == np.sin(2.0) and sin[3, 43] == np.sin(3.0) and not sin[3, :43].any()
    # inside each band the frequencies form a geometric sequence spanning a factor of the base: the
    # ratio of neighbouring pairs, raised to the band's pair count, is 1 / base
    c, s = O.rope_tables(np.array([[1, 1, 1]]))
    ang = np.arctan2(s[0], c[0])
    p0 = 0
    for w in (44, 42, 42):
        a = ang[p0:p0 + w // 2]
        ratio = a[1:] / a[:-1]
        assert np.allclose(ratio, ratio[0], rtol=1e-12, atol=0)
        assert abs(ratio[0] ** (w // 2) * O.ROPE_BASE - 1.0) < 1e-10
        p0 += w // 2


def test_rope_relative_position():
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal((1, 128)), rng.standard_normal((1, 128))
    base = np.array([[3, 5, 7], [1, 2, 9]])
    for shift in ([4, 0, 0], [0, 6, 0], [0, 0, 11], [2, 3, 1]):
        c, s = O.rope_tables(base + np.array(shift))
        c0, s0 = O.rope_tables(base)
        d0 = _rope_apply(q, c0[:1], s0[:1]) @ _rope_apply(k, c0[1:], s0[1:]).T
        d1 = _rope_apply(q, c[:1], s[:1]) @ _rope_apply(k, c[1:], s[1:]).T
        assert abs(d0 - d1) < 1e-12


def test_qk_norm_rope_reduces_to_rms_norm_at_position_zero():
    g = I.gaussian_bf16(1001, (128,), 0.1)
    g = I.f32_to_bf16_bits((O.bf16_to_f64(g) + 1.0).astype(np.float32))
    cos, sin = np.ones((5, 64)), np.zeros((5, 64))
    for std, eps in ((2.0, 1e-6), (1e-3, 1e-6)):     # the second case: eps comparable to the mean square
        x = I.gaussian_bf16(1000, (5, 3, 128), std, 0.02, 20.0)
        got = O.qk_norm_rope(x, g, cos, sin, eps)
        xt = torch.from_numpy(O.bf16_to_f64(x))
        want = torch.nn.functional.rms_norm(xt, (128,), torch.from_numpy(O.bf16_to_f64(g)), eps).numpy()
        assert np.array_equal(got, O.f64_to_bf16(want))


def test_qk_norm_rope_zero_head_gives_zero():
    # a head whose radicand mean(x^2) + eps is 0 (all zero, eps = 0) normalises to 0, not NaN;
    # with eps > 0 the same head is 0 too, and a nonzero head next to it is unaffected
    x = np.zeros((3, 2, 128), np.uint16)
    x[:, 1] = I.gaussian_bf16(1003, (3, 128), 1.0)
    cos, sin = O.rope_tables(np.array([[1, 2, 3], [4, 5, 6], [0, 0, 0]]))
    for eps in (0.0, 1e-6):
        out = O.qk_norm_rope_f64(x, None, cos, sin, eps)
        assert np.all(np.isfinite(out))
        assert np.all(out[:, 0] == 0.0)
        assert np.allclose((out[:, 1] ** 2).mean(axis=-1), 1.0, rtol=1e-5)


def test_qk_norm_rope_quarter_turn_and_pair_norms():
    x = I.gaussian_bf16(1002, (4, 2, 128), 1.0)
    u = O.bf16_to_f64(O.qk_norm_rope(x, None, np.ones((4, 64)), np.zeros((4, 64)), 0.0))
    turned = O.bf16_to_f64(O.qk_norm_rope(x, None, np.zeros((4, 64)), np.ones((4, 64)), 0.0))
    assert np.array_equal(turned[..., 0::2], -u[..., 1::2]) and np.array_equal(turned[..., 1::2], u[..., 0::2])
    cos, sin = O.rope_tables(np.array([[7, 3, 1], [0, 40, 2], [9, 9, 9], [1, 1, 60]]))
    y = O.bf16_to_f64(O.qk_norm_rope(x, None, cos, sin, 0.0))
    # each pair keeps its length up to the final bf16 rounding; the whole head keeps unit mean square
    n0 = np.hypot(u[..., 0::2], u[..., 1::2])
    n1 = np.hypot(y[..., 0::2], y[..., 1::2])
    assert np.all(np.abs(n1 - n0) <= 2 ** -7 * n0 + 1e-30)
    assert np.allclose((y * y).mean(axis=-1), 1.0, rtol=1e-2)
    # the complex-multiplication form of the turn agrees
    xs = O.bf16_to_f64(x)
    xs = xs / np.sqrt((xs * xs).mean(axis=-1, keepdims=True))
    ref = np.stack([_rope_apply(xs[:, h], cos, sin) for h in range(2)], axis=1)
    assert np.array_equal(O.f64_to_bf16(ref), O.f64_to_bf16(y))


def _sdpa64(q, k, v):
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(a.transpose(1, 0, 2))) for a in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).numpy().transpose(1, 0, 2)


def test_attention_without_quantisation_is_textbook_sdpa():
    q = I.gaussian_bf16(1003, (7, 2, 128), 1.0)
    k = I.gaussian_bf16(1004, (9, 2, 128), 1.0)
    v = I.gaussian_bf16(1005, (9, 2, 128), 1.0)
    want = _sdpa64(O.bf16_to_f64(q), O.bf16_to_f64(k), O.bf16_to_f64(v))
    assert np.abs(O.sage_attention(q, k, v, smooth=False, quant=False) - want).max() < 1e-12
    # smoothing shifts every score of a query row equally; only the float32 rounding of the
    # smoothed keys (relative 2^-24 per element) remains
    assert np.abs(O.sage_attention(q, k, v, smooth=True, quant=False) - want).max() < 1e-6


def test_attention_lossless_int8_codes():
    """Q and K that are exactly INT8 codes times a power of two, with a code of 127 in every (token,
    head) and keys in +- pairs (zero mean): quantisation is exact, so the scheme equals SDPA."""
    rng = np.random.default_rng(9)

    def coded(t, sign_pairs):
        c = rng.integers(-127, 128, (t, 2, 128)).astype(np.float64)
        c[..., 5] = 127
        if sign_pairs:
            c = np.concatenate([c, -c])
        e = rng.integers(-6, 3, (c.shape[0], 2, 1)).astype(np.float64)
        return I.f32_to_bf16_bits((c * 2.0 ** e).astype(np.float32))

    q, k = coded(6, False), coded(5, True)
    v = I.gaussian_bf16(1006, (10, 2, 128), 1.0)
    qc, sq = O.quantize_heads_int8(O.bf16_to_f64(q).astype(np.float32))
    assert np.all(np.abs(qc).max(axis=-1) == 127)
    assert np.array_equal(qc.astype(np.float64) * sq[..., None], O.bf16_to_f64(q))
    got = O.sage_attention(q, k, v)
    want = _sdpa64(O.bf16_to_f64(q), O.bf16_to_f64(k), O.bf16_to_f64(v))
    assert np.abs(got - want).max() < 1e-12


def test_attention_smoothing_removes_a_common_key_offset():
    """A large per-channel key offset wastes the INT8 range; smoothing removes it and the error to the
    exact attention drops.  The output stays inside the convex hull of the value rows."""
    q = I.gaussian_bf16(1007, (16, 2, 128), 1.0)
    k64 = O.bf16_to_f64(I.gaussian_bf16(1008, (32, 2, 128), 1.0)) + 40.0 * np.sin(np.arange(128))
    k = I.f32_to_bf16_bits(k64.astype(np.float32))
    v = I.gaussian_bf16(1009, (32, 2, 128), 1.0)
    exact = O.sage_attention(q, k, v, smooth=False, quant=False)
    e_plain = np.abs(O.sage_attention(q, k, v, smooth=False) - exact).max()
    e_smooth = np.abs(O.sage_attention(q, k, v, smooth=True) - exact).max()
    assert e_smooth < 0.25 * e_plain
    out = O.sage_attention(q, k, v)
    vv = O.bf16_to_f64(v)
    assert np.all(out <= vv.max(axis=0)[None] + 1e-12) and np.all(out >= vv.min(axis=0)[None] - 1e-12)


def test_attention_tiled_fp16_p_stays_within_the_output_tolerance():
    """Reading of the FP16 P.V step: a flash-style evaluation over 128-key tiles (running max and sum,
    the unnormalised P rounded to fp16 for the product, float32 accumulation, a ragged last tile)
    stays within the output tolerance of the oracle's float64 softmax."""
    from tests.helpers import check_output

    Tq, Tk, H = 256, 1000, 2
    q = I.gaussian_bf16(1010, (Tq, H, 128), 1.0, 0.02, 10.0)
    k = I.gaussian_bf16(1011, (Tk, H, 128), 1.0, 0.02, 10.0)
    v = I.gaussian_bf16(1012, (Tk, H, 128), 1.0)
    ref64 = O.sage_attention(q, k, v)
    s2 = O.attention_scores(q, k).astype(np.float32) * np.float32(np.log2(np.e))   # [H, Tq, Tk]
    v16 = O.bf16_to_f64(v).astype(np.float16).astype(np.float32)
    out = np.zeros((Tq, H, 128))
    for h in range(H):
        m = np.full(Tq, -np.inf, np.float32)
        l = np.zeros(Tq, np.float32)
        acc = np.zeros((Tq, 128), np.float32)
        for j0 in range(0, Tk, 128):
            st = s2[h, :, j0:j0 + 128]
            m_new = np.maximum(m, st.max(axis=1))
            alpha = np.where(np.isinf(m), 0.0, np.exp2(m - m_new)).astype(np.float32)
            p = np.exp2(st - m_new[:, None]).astype(np.float32)
            l = l * alpha + p.sum(axis=1, dtype=np.float32)
            acc = acc * alpha[:, None] + p.astype(np.float16).astype(np.float32) @ v16[j0:j0 + 128, h]
            m = m_new
        out[:, h] = acc / l[:, None]
    got = O.f64_to_bf16(out)
    check_output(got.reshape(Tq, -1), ref64.reshape(Tq, -1), O.f64_to_bf16(ref64).reshape(Tq, -1))


def test_exact_to_f32_matches_an_independent_rounding():
    """exact_to_f32 (exact rational -> float32, nearest, ties to even) against numpy's own
    float64 -> float32 conversion, which rounds the same way, on values a float64 holds exactly:
    random magnitudes over the normal and subnormal range, exact halfway points between
    neighbouring float32 values (both parities of the lower neighbour), and signs."""
    rng = np.random.default_rng(7)
    vals = list(rng.standard_normal(2000) * np.exp2(rng.integers(-140, 100, 2000)))
    # exact ties: midpoint of f and its upper neighbour, for f with even and odd significands
    for f in np.float32([1.0, 1.0 + 2.0 ** -23, 3.0, 1.5 + 2.0 ** -22, 1e-40, 7.0e-39, 123.456]):
        up = np.nextafter(f, np.float32(np.inf))
        vals.append((float(f) + float(up)) / 2.0)
        vals.append(-(float(f) + float(up)) / 2.0)
    for v in vals:
        want = np.float32(np.float64(v))
        got = O.exact_to_f32(Fraction(float(v)))
        assert got == want and np.signbit(got) == np.signbit(want), (v, got, want)
