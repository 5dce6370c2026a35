"""CPU oracle for the rotated low-bit quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or links
this module: only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline /
reference leg may use it.  It shares no code with the CUDA path (no common
tables, constants or helpers); both sides only read the same seeded bf16 inputs.

What it computes (plain, slow, float64 unless a step fixes the precision):

1. Rotation.  Every 256-wide block of the K axis is multiplied by R = H/16, H
   the regular Hadamard matrix (J4 - 2 I4) Kronecker-powered four times.
   Source: Krea-2 Turbo -- INT4 tensorwise W4A4 (+ConvRot, mixed int8 fallback),
   header (a regular Hadamard rotation over groups of 256 channels, applied
   to activations at run time); Krea-2-SVDQuant-ComfyUI, "Why this exists"
   (rotating by Hadamard blocks spreads outlier channels in closed form, with
   no calibration).  The rotated value is
   the exact sum rounded once to float32.
2. Dynamic symmetric quantisation per token (or per 64-wide group) to signed
   INT4 (qmax 7) or INT8 (qmax 127), round half to even, clamp.
   Source: the INT4 tensorwise model card header (the kernel computes the
   activation scales itself, at run time); Krea 2 Turbo OrbitQuant W4A4, "What is quantized"
   (per-row INT8 ff.down weights with INT8 activations); Krea 2 Turbo Nunchaku
   Lite INT4 r32, header (group size 64, rank 32).
3. Packed signed INT4 weights, two codes per byte (even k in the low nibble).
   Source: INT4 tensorwise model card header (signed four-bit weight codes, packed).
4. Integer GEMM, exact (int64 here), one partial per 64-group in group mode.
5. Epilogue in float64: dequant scales, + bias, + low-rank branch
   (X L1) L2 on the unrotated input, then a sigmoid on the gate columns or a
   gated residual out = R + g * y, then one round to bf16.
   Source: OrbitQuant W4A4 card, "Fused transformer" (the Q|K|V|gate GEMM
   applies the sigmoid gate on its way out; residual adds with their gates are
   also done in GEMM epilogues); Krea-2-SVDQuant-ComfyUI, "LoRA" (a low-rank
   term distributes over the product: (W + BA)x = Wx + B(Ax)) and "Why this
   exists" (the W4A4 kernel carries an extra low-rank term beside it).
6. NVFP4 variant: E2M1 codes with an E4M3 scale per 16 elements and a float32
   tensor scale.  Source: Nunchaku Lite INT4 r32 card, "Benchmark" (NVFP4 build
   on native FP4 tensor cores).
7. Normalising prologue: RMSNorm and adaLN-style modulation ahead of the
   rotation.  Source: OrbitQuant W4A4 card, "Fused transformer" (the norm and
   the modulation are folded into the kernels that quantise activations).
8. INT4 KV-cache codec: packed codes with one float32 scale per token, head
   and group, groups inside the 44 | 42 | 42 rotary bands.  Source: "lab",
   Study 6 (the cache goes to four bits).
9. Offline SVDQuant fit of the low-rank branch (randomized SVD, alternating
   refit / requantise keeping the best, optional activation weighting).
   Source: Krea-2-SVDQuant-ComfyUI, "Low-rank refinement, and what the
   objective actually is", "Activation-aware branch".
10. Q/K RMSNorm + RoPE over the 44 | 42 | 42 rotary bands, and attention with
   INT8 Q.K^T (smoothed keys, one scale per token and head) and FP16 P.V.
   Source: OrbitQuant W4A4 card, "Fused transformer" (the SageAttention v1
   scheme); "lab", Study 6 (the rotary bands).

Readings of points the pages leave open are listed where they are used.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

GROUP = 256          # rotation group width
INV_GROUP_NORM = 1.0 / 16.0   # 1/sqrt(256): R = H/16 is orthonormal


# ---------------------------------------------------------------------------
# 1. The regular Hadamard matrix
# ---------------------------------------------------------------------------

def hadamard_regular_kron(n: int = GROUP) -> np.ndarray:
    """(J4 - 2 I4) Kronecker-powered to order n (n a power of 4), as int64.

    Reading: the pages say only "regular-Hadamard".  J4 - 2I4 is the order-4
    regular Hadamard matrix (every row sums to 2); its Kronecker powers stay
    regular, symmetric and Hadamard, and 256 = 4^4.
    """
    h4 = np.ones((4, 4), dtype=np.int64) - 2 * np.eye(4, dtype=np.int64)
    h = np.ones((1, 1), dtype=np.int64)
    while h.shape[0] < n:
        h = np.kron(h, h4)
    if h.shape[0] != n:
        raise ValueError("order must be a power of 4")
    return h


def hadamard_regular_digits(n: int = GROUP) -> np.ndarray:
    """The same matrix built entry by entry: H[i][j] = prod over base-4 digits of
    (-1 if the digits are equal else +1)."""
    d = 0
    while 4 ** d < n:
        d += 1
    h = np.empty((n, n), dtype=np.int64)
    for i in range(n):
        for j in range(n):
            v = 1
            a, b = i, j
            for _ in range(d):
                if a % 4 == b % 4:
                    v = -v
                a //= 4
                b //= 4
            h[i, j] = v
    return h


def hadamard_sylvester(n: int = GROUP) -> np.ndarray:
    """Sylvester's construction [[1,1],[1,-1]]^{(x)k}.  Test-only alternative reading."""
    h = np.ones((1, 1), dtype=np.int64)
    h2 = np.array([[1, 1], [1, -1]], dtype=np.int64)
    while h.shape[0] < n:
        h = np.kron(h, h2)
    return h


def rotation_matrix(n: int = GROUP) -> np.ndarray:
    """R = H / sqrt(n) in float64 (exact: the entries are +-1/16)."""
    return hadamard_regular_kron(n).astype(np.float64) / np.sqrt(float(n))


# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns (uint16) as float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16, nearest with ties to even, directly from the
    float64 value (no intermediate float32 rounding).  Returns uint16 patterns."""
    v = np.asarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.float64)
    a = np.abs(v)
    nz = a > 0
    _, ex = np.frexp(a[nz])                # a = m * 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -126)           # exponent of the leading bit; bf16 subnormals below
    ulp = np.ldexp(1.0, e - 7)             # 8 significant bits
    out[nz] = np.sign(v[nz]) * np.rint(a[nz] / ulp) * ulp
    out[~nz] = v[~nz]                       # +-0 keep their sign
    big = np.abs(out) > 3.3895313892515355e38
    out[big] = np.copysign(np.inf, out[big])
    return (out.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def exact_to_f32(q: Fraction) -> np.float32:
    """Round an exact rational to float32, nearest with ties to even."""
    if q == 0:
        return np.float32(0.0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)
    scaled = a / (Fraction(2) ** (e - 23))           # in [2^23, 2^24) for normals
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return np.float32(sign * float(n) * 2.0 ** (e - 23))


# ---------------------------------------------------------------------------
# 2. Rotation, exact then rounded once to float32
# ---------------------------------------------------------------------------

def _group_span_ok(xg: np.ndarray) -> np.ndarray:
    """Per 256-group: True when every partial sum of +-x_j/16 is exact in float64.

    Each bf16 input is an integer multiple of 2^(e_min-7) (e_min: the smallest
    leading-bit exponent in the group, -126 for subnormals) and |sum| is below
    2^(e_max+1) * 256/16.  All partial sums then need at most
    (e_max - e_min) + 16 significant bits, so the float64 sum is exact, in any
    order, whenever e_max - e_min <= 37.
    """
    a = np.abs(xg)
    nz = a > 0
    _, ex = np.frexp(np.where(nz, a, 1.0))
    e = np.maximum(ex - 1, -126)
    emax = np.where(nz, e, -10**6).max(axis=-1)
    emin = np.where(nz, e, 10**6).min(axis=-1)
    return (~nz.any(axis=-1)) | (emax - emin <= 37)


def rotate(x: np.ndarray, group: int = GROUP) -> np.ndarray:
    """x [rows, K] float64 (bf16 values) -> float32 RN(x_block @ R) per K-block.

    group == 0 means no rotation (the value is only rounded to float32, which is
    exact for bf16 inputs).
    """
    x = np.asarray(x, dtype=np.float64)
    if group == 0:
        return x.astype(np.float32)
    rows, k = x.shape
    if k % group:
        raise ValueError("K must be a multiple of the rotation group")
    r = rotation_matrix(group)
    xg = x.reshape(rows, k // group, group)
    y = np.matmul(xg, r)                       # exact when _group_span_ok (float64 BLAS)
    out = y.astype(np.float32)                 # one round to nearest even
    ok = _group_span_ok(xg)
    if not ok.all():
        h = hadamard_regular_kron(group)
        for ri, gi in zip(*np.nonzero(~ok)):
            xs = [Fraction(float(v)) for v in xg[ri, gi]]
            for i in range(group):
                s = sum((xs[j] if h[i, j] > 0 else -xs[j] for j in range(group)), Fraction(0))
                out[ri, gi, i] = exact_to_f32(s / 16)
    return out.reshape(rows, k)


def rotate_exact_fraction(x_row: np.ndarray, group: int = GROUP) -> np.ndarray:
    """Brute force: every rotated value as an exact rational, rounded once (tiny inputs only)."""
    h = hadamard_regular_kron(group)
    out = np.empty(len(x_row), dtype=np.float32)
    for g0 in range(0, len(x_row), group):
        xs = [Fraction(float(v)) for v in x_row[g0:g0 + group]]
        for i in range(group):
            s = sum((xs[j] * int(h[j, i]) for j in range(group)), Fraction(0))
            out[g0 + i] = exact_to_f32(s / 16)
    return out


# ---------------------------------------------------------------------------
# 3. Quantisation
# ---------------------------------------------------------------------------

def qmax_of(bits: int) -> int:
    if bits not in (4, 8):
        raise ValueError("bits must be 4 or 8")
    return 7 if bits == 4 else 127


def quantize(xr: np.ndarray, bits: int, scale_group: int = 0):
    """Symmetric dynamic quantisation of float32 rows.

    Per row (scale_group 0) or per scale_group-wide block of a row:
      amax = max |xr|;  s = amax / qmax;  inv = qmax / amax  (IEEE float32 divisions)
      q = clamp(rint_half_even(xr * inv), -qmax-1, qmax)   (float32 product)
    An all-zero row or block gets s = 0 and q = 0.
    Returns (codes int8 [rows, K], scales float32 [rows] or [rows, K/scale_group]).
    """
    xr = np.asarray(xr, dtype=np.float32)
    rows, k = xr.shape
    qmax = np.float32(qmax_of(bits))
    g = k if scale_group == 0 else scale_group
    if k % g:
        raise ValueError("K must be a multiple of the scale group")
    xb = xr.reshape(rows, k // g, g)
    amax = np.abs(xb).max(axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        s = (amax / qmax).astype(np.float32)
        inv = np.where(amax > 0, qmax / amax, np.float32(0.0)).astype(np.float32)
    prod = (xb * inv[..., None]).astype(np.float32)
    q = np.clip(np.rint(prod), -qmax - 1, qmax).astype(np.int8)
    scales = s if scale_group else s[:, 0]
    return q.reshape(rows, k), scales.astype(np.float32)


def rot_quant(x_bits: np.ndarray, bits: int, rot_group: int = GROUP, scale_group: int = 0):
    """The activation path: bf16 x [M,K] -> (codes int8 [M,K], scales)."""
    xr = rotate(bf16_to_f64(x_bits), rot_group)
    return quantize(xr, bits, scale_group)


def norm_modulate(x_bits: np.ndarray, gamma_bits=None, shift_bits=None, scale_bits=None,
                  eps: float = 1e-6) -> np.ndarray:
    """RMSNorm and adaLN-style modulation of bf16 rows, returned as bf16 patterns.

    Source: Krea 2 Turbo OrbitQuant W4A4, "Fused transformer": the norm and the
    modulation are folded into the kernels that quantise activations.  The pages
    print no formula; the readings (plainest ones) are:
      - RMS over the whole row: S = sum_k x_k^2 (exact, rounded once to
        float64), ms = S / K, d = ms + eps, r = 1 / sqrt(d), all float64 IEEE
        operations; r is rounded once to float32.  A row with d == 0 gets r = 0.
      - per element, single IEEE float32 operations in this order:
        u = x * r;  u = u * gamma (when given);  v = u * (1 + scale);
        v = v + shift;  gamma, shift, scale are bf16 [K] vectors (batch 1: one
        modulation vector per call), 1 + scale rounded to float32 first.
      - the result is rounded once to bf16, the activation dtype the quantiser
        receives in an unfused pipeline.
    eps is the float32 value the caller passes, used exactly.
    """
    x = bf16_to_f64(x_bits)
    rows, k = x.shape
    eps64 = float(np.float32(eps))
    r32 = np.empty(rows, dtype=np.float32)
    for i in range(rows):
        s = math.fsum(float(v) * float(v) for v in x[i])      # exact squares, one rounding
        d = s / k + eps64
        r32[i] = np.float32(1.0 / math.sqrt(d)) if d > 0 else np.float32(0.0)
    u = (x.astype(np.float32) * r32[:, None]).astype(np.float32)
    if gamma_bits is not None:
        u = (u * bf16_to_f64(gamma_bits).astype(np.float32)[None, :]).astype(np.float32)
    if scale_bits is not None:
        a = (np.float32(1.0) + bf16_to_f64(scale_bits).astype(np.float32)).astype(np.float32)
        u = (u * a[None, :]).astype(np.float32)
    if shift_bits is not None:
        u = (u + bf16_to_f64(shift_bits).astype(np.float32)[None, :]).astype(np.float32)
    return f64_to_bf16(u.astype(np.float64))


def norm_rot_quant(x_bits: np.ndarray, bits: int, rot_group: int = GROUP, scale_group: int = 0,
                   gamma_bits=None, shift_bits=None, scale_bits=None, eps: float = 1e-6):
    """The normalising prologue: norm_modulate, then the activation path (rot_quant)."""
    xm = norm_modulate(x_bits, gamma_bits, shift_bits, scale_bits, eps)
    return rot_quant(xm, bits, rot_group, scale_group)


def pack_int4(q: np.ndarray) -> np.ndarray:
    """Two's-complement nibbles, row-major, even k in the low nibble -> uint8 [rows, K/2].

    Reading: the pages fix only that the codes are signed four-bit values stored two to a byte.
    """
    q = np.asarray(q, dtype=np.int64)
    if q.min(initial=0) < -8 or q.max(initial=0) > 7:
        raise ValueError("INT4 codes must lie in [-8, 7]")
    nib = (q & 0xF).astype(np.uint8)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def unpack_int4(p: np.ndarray) -> np.ndarray:
    p = np.asarray(p, dtype=np.uint8)
    lo = (p & 0xF).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def quantize_weights(w_bits: np.ndarray, bits: int, rot_group: int = GROUP, scale_group: int = 0):
    """Offline weight path: each output row of W [N,K] is rotated and quantised like a token.
    Returns (packed uint8 [N,K/2] for 4 bits or int8 [N,K] for 8 bits, scales)."""
    q, s = rot_quant(w_bits, bits, rot_group, scale_group)
    return (pack_int4(q) if bits == 4 else q), s


# ---------------------------------------------------------------------------
# 4. Integer GEMM
# ---------------------------------------------------------------------------

def gemm_acc(qx: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """acc[m,n] = sum_k qx[m,k] qw[n,k] as int64.  A float64 matmul of small integer
    codes is exact while |acc| < 2^53; the result must also fit int32."""
    acc = np.matmul(np.asarray(qx, np.float64), np.asarray(qw, np.float64).T)
    if np.abs(acc).max(initial=0) >= 2 ** 31:
        raise OverflowError("accumulator exceeds int32")
    return acc.astype(np.int64)


def gemm_acc_loops(qx: np.ndarray, qw: np.ndarray) -> np.ndarray:
    """The same accumulators by explicit int64 loops (tiny shapes only)."""
    m, k = qx.shape
    n = qw.shape[0]
    acc = np.zeros((m, n), dtype=np.int64)
    for i in range(m):
        for j in range(n):
            s = 0
            for t in range(k):
                s += int(qx[i, t]) * int(qw[j, t])
            acc[i, j] = s
    return acc


def gemm_acc_grouped(qx: np.ndarray, qw: np.ndarray, group: int) -> np.ndarray:
    """One int64 partial per `group`-wide K block: acc[g, m, n]."""
    k = qx.shape[1]
    return np.stack([gemm_acc(qx[:, g:g + group], qw[:, g:g + group]) for g in range(0, k, group)])


# ---------------------------------------------------------------------------
# 5. Dequant and epilogue (float64)
# ---------------------------------------------------------------------------

def dequant(qx, sx, qw, sw, scale_group: int = 0) -> np.ndarray:
    """y[m,n] = sx[m] sw[n] acc[m,n], or sum_g sx[m,g] sw[n,g] acc_g[m,n] in group mode."""
    sx = np.asarray(sx, np.float64)
    sw = np.asarray(sw, np.float64)
    if scale_group == 0:
        return gemm_acc(qx, qw).astype(np.float64) * sx[:, None] * sw[None, :]
    k = qx.shape[1]
    y = np.zeros((qx.shape[0], qw.shape[0]), dtype=np.float64)
    for gi, g in enumerate(range(0, k, scale_group)):
        acc = gemm_acc(qx[:, g:g + scale_group], qw[:, g:g + scale_group]).astype(np.float64)
        y += acc * sx[:, gi, None] * sw[None, :, gi]
    return y


def lowrank_down(x_bits: np.ndarray, l1_bits: np.ndarray) -> np.ndarray:
    """Ld = X L1 on the unrotated bf16 input, float64 (the branch's first factor).

    Reading: the branch is a parallel linear on the layer input,
    (W + L1 L2) x = W x + L2 (L1 x) -- Krea-2-SVDQuant-ComfyUI, "LoRA".
    """
    return bf16_to_f64(x_bits) @ bf16_to_f64(l1_bits)


def epilogue(y: np.ndarray, bias=None, ld=None, l2_bits=None, gate_mode: int = 0,
             gate_cols=(0, 0), gate_bits=None, residual_bits=None) -> np.ndarray:
    """Float64 epilogue: + bias, + Ld L2, then sigmoid on gate columns (gate_mode 1)
    or out = residual + g * y (gate_mode 2).  Returns float64 (round with f64_to_bf16)."""
    y = np.array(y, dtype=np.float64, copy=True)
    if bias is not None:
        y += bf16_to_f64(bias)[None, :]
    if ld is not None:
        y += np.asarray(ld, np.float64) @ bf16_to_f64(l2_bits)
    if gate_mode == 1:
        c0, c1 = gate_cols
        y[:, c0:c1] = 1.0 / (1.0 + np.exp(-y[:, c0:c1]))
    elif gate_mode == 2:
        y = bf16_to_f64(residual_bits) + bf16_to_f64(gate_bits)[None, :] * y
    elif gate_mode != 0:
        raise ValueError("gate_mode must be 0, 1 or 2")
    return y


def linear_reference(x_bits, w_bits, bits: int, rot_group: int = GROUP, scale_group: int = 0,
                     bias=None, l1=None, l2=None, gate_mode: int = 0, gate_cols=(0, 0),
                     gate=None, residual=None, rows=None):
    """The whole layer: returns dict(codes, sx, wq, sw, y64, ref64, ref_bf16).

    rows: optional token indices; the layer is evaluated on those rows only
    (rows are independent, so a sampled row is fully checked).
    """
    if rows is not None:
        x_bits = np.asarray(x_bits)[rows]
        if residual is not None:
            residual = np.asarray(residual)[rows]
    qx, sx = rot_quant(x_bits, bits, rot_group, scale_group)
    wq, sw = quantize_weights(w_bits, bits, rot_group, scale_group)
    qw = unpack_int4(wq) if bits == 4 else wq
    y = dequant(qx, sx, qw, sw, scale_group)
    ld = lowrank_down(x_bits, l1) if l1 is not None else None
    ref64 = epilogue(y, bias, ld, l2, gate_mode, gate_cols, gate, residual)
    return dict(codes=qx, sx=sx, wq=wq, sw=sw, y64=y, ld=ld, ref64=ref64, ref_bf16=f64_to_bf16(ref64))


# ---------------------------------------------------------------------------
# 6. NVFP4 variant
# ---------------------------------------------------------------------------

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E4M3_MAX = 448.0
E2M1_MAX = 6.0


def round_e2m1(v: np.ndarray) -> np.ndarray:
    """Nearest E2M1 value, ties to the even encoding, saturating at +-6 (float64 in/out)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.minimum(np.abs(v), E2M1_MAX)
    # grid spacing: 0.5 below 2, 1 in [2,4), 2 in [4,6]
    step = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    n = a / step
    r = np.rint(n)              # ties to even multiple of step
    q = r * step
    # A tie at a binade edge (e.g. 1.75 between 1.5 and 2) resolves by encoding parity:
    # even encodings are 0, 1, 2, 4.  rint of 3.5 half-steps gives 4 -> 2.0 (correct);
    # at 3.5 (between 3 and 4) rint(3.5) = 4 -> 4.0 (encoding 110, even: correct);
    # at 5 (between 4 and 6): step 2, n = 2.5 -> rint 2 -> 4 (even: correct).
    return np.sign(v) * np.minimum(q, E2M1_MAX)


def round_e4m3(v: np.ndarray) -> np.ndarray:
    """Nearest E4M3 (bias 7, no infinities, max 448) value, ties to even, saturating."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    out = np.zeros_like(a)
    nz = a > 0
    _, ex = np.frexp(a[nz])
    e = np.maximum(ex - 1, -6)                 # subnormals below 2^-6, step 2^-9
    ulp = np.ldexp(1.0, e - 3)
    out[nz] = np.rint(a[nz] / ulp) * ulp
    out = np.minimum(out, E4M3_MAX)
    return np.sign(v) * out


def nvfp4_quantize(xr: np.ndarray):
    """Two-level NVFP4 quantisation of float32 rows [rows, K] (K % 16 == 0).

    gs = amax(tensor) / (6 * 448)              float32
    bs = E4M3(amax(block16) / (6 * gs))        float32 division, E4M3 RN satfinite
    q  = E2M1(xr / (bs * gs))                  float32 product and division, E2M1 RN
    Returns (q float64 grid values [rows,K], bs float64 [rows,K/16], gs float32).
    Reading: the pages name only "E4M3 scale per 16 elements"; the float32 tensor
    scale keeps the E4M3 block scales out of the E4M3 subnormal range.
    """
    xr = np.asarray(xr, dtype=np.float32)
    rows, k = xr.shape
    amax_t = np.float32(np.abs(xr).max(initial=0.0))
    gs = np.float32(amax_t / np.float32(6.0 * 448.0))
    xb = xr.reshape(rows, k // 16, 16)
    amax_b = np.abs(xb).max(axis=-1).astype(np.float32)
    six_gs = np.float32(np.float32(6.0) * gs)
    with np.errstate(divide="ignore", invalid="ignore"):
        bs = round_e4m3(np.where(six_gs > 0, amax_b / six_gs, np.float32(0)).astype(np.float32))
        denom = (bs.astype(np.float32) * gs).astype(np.float32)
        ratio = np.where(denom[..., None] > 0, xb / denom[..., None], np.float32(0)).astype(np.float32)
    q = round_e2m1(ratio)
    return q.reshape(rows, k), bs, gs


def nvfp4_linear(x_bits, w_bits, rot_group: int = GROUP) -> np.ndarray:
    """y = sum_k (qx bsx gsx)(qw bsw gsw) in float64 (exact products)."""
    xq, xbs, xgs = nvfp4_quantize(rotate(bf16_to_f64(x_bits), rot_group))
    wq, wbs, wgs = nvfp4_quantize(rotate(bf16_to_f64(w_bits), rot_group))
    xd = xq * np.repeat(xbs, 16, axis=1) * float(xgs)
    wd = wq * np.repeat(wbs, 16, axis=1) * float(wgs)
    return xd @ wd.T


# ---------------------------------------------------------------------------
# 8. INT4 KV-cache codec
# ---------------------------------------------------------------------------
# Source: "lab", Study 6 ("The cache becomes the model"): four-bit codes, two
# to a byte, with a scale for each (token, head, rotary band); a head's 128
# channels form three rotary bands -- channels 0-43 carry time, 44-85 height,
# 86-127 width; finer scale groups stay inside one band (3, 6 or 12 groups
# per head); a read unpacks and rescales in a single pass.
# Readings (the pages give the structure, not the arithmetic):
#   - a band of b channels split into n groups is cut into contiguous runs whose
#     sizes differ by at most one, the longer runs first;
#   - each group is quantised like an activation row: amax, s = amax / 7,
#     inv = 7 / amax (float32 IEEE divisions), q = clamp(rint(x * inv), -8, 7);
#     an all-zero group gets s = 0 and q = 0; scales are stored as float32;
#   - two codes per byte, the even channel in the low nibble;
#   - reading gives RN_bf16(q * s), the product a float32 multiplication.

KV_HEAD_DIM = 128
KV_BANDS = (44, 42, 42)


def kv4_group_sizes(groups_per_band: int) -> list:
    """Group sizes along the 128 channels of a head, band by band."""
    if groups_per_band not in (1, 2, 4):
        raise ValueError("groups_per_band must be 1, 2 or 4")
    sizes = []
    for b in KV_BANDS:
        base, extra = divmod(b, groups_per_band)
        sizes += [base + 1 if i < extra else base for i in range(groups_per_band)]
    return sizes


def kv4_encode(x_bits: np.ndarray, groups_per_band: int):
    """bf16 [T, H, 128] -> (packed uint8 [T, H, 64], scales float32 [T, H, G])."""
    x = bf16_to_f64(x_bits).astype(np.float32)
    t, h, d = x.shape
    if d != KV_HEAD_DIM:
        raise ValueError("head dimension must be 128")
    sizes = kv4_group_sizes(groups_per_band)
    q = np.zeros((t, h, d), dtype=np.int8)
    scales = np.zeros((t, h, len(sizes)), dtype=np.float32)
    c0 = 0
    for gi, n in enumerate(sizes):
        seg = x[:, :, c0:c0 + n].reshape(t * h, n)
        qs, ss = quantize(seg, 4, 0)               # one group = one "row" of the activation quantiser
        q[:, :, c0:c0 + n] = qs.reshape(t, h, n)
        scales[:, :, gi] = ss.reshape(t, h)
        c0 += n
    packed = pack_int4(q.reshape(t * h, d)).reshape(t, h, d // 2)
    return packed, scales


def kv4_decode(packed: np.ndarray, scales: np.ndarray, groups_per_band: int) -> np.ndarray:
    """(packed [T, H, 64], scales [T, H, G]) -> bf16 patterns [T, H, 128]."""
    t, h, _ = packed.shape
    q = unpack_int4(packed.reshape(t * h, -1)).reshape(t, h, KV_HEAD_DIM).astype(np.float32)
    sizes = kv4_group_sizes(groups_per_band)
    s = np.repeat(scales, sizes, axis=2).astype(np.float32)
    return f64_to_bf16((q * s).astype(np.float32).astype(np.float64))


# ---------------------------------------------------------------------------
# 9. Offline SVDQuant fit of the low-rank branch
# ---------------------------------------------------------------------------
# Source: Krea-2-SVDQuant-ComfyUI, "Low-rank refinement, and what the
# objective actually is" and "Activation-aware branch": the objective is the
# Frobenius distance between W and the quantised part plus the branch; the
# first split comes from a seeded randomized SVD; after that the branch is
# re-fitted to what quantisation currently misses and the remainder is
# quantised again, several times, and the best iterate wins, so extra
# iterations cannot hurt; with activation statistics each input channel's
# error counts by that channel's RMS d (scaled to mean 1, never below 0.05).
# Readings: the residual is rounded to bf16 before it is quantised (the
# packer's input type); the quantised residual is the layer's own rotated
# INT4/INT8 format; the randomized SVD's Gaussian test matrices are inputs
# (one per iteration); the rank-r product is split evenly, L1 = V sqrt(S),
# L2 = sqrt(S) U^T, so that (x L1) L2 = x (U S V^T)^T.

def dequantize_weights(q: np.ndarray, scales: np.ndarray, bits: int, rot_group: int = GROUP,
                       scale_group: int = 0) -> np.ndarray:
    """Codes times scales in the rotated domain, rotated back (R = H/16 is symmetric and
    orthonormal, so R^-1 = R): the float64 weight the quantised format stands for, [N, K]."""
    codes = (unpack_int4(q) if bits == 4 else np.asarray(q)).astype(np.float64)
    n, k = codes.shape
    s = np.asarray(scales, dtype=np.float64)
    s = np.repeat(s, scale_group, axis=1) if scale_group else s[:, None]
    wr = codes * s
    if rot_group:
        wr = np.matmul(wr.reshape(n, k // rot_group, rot_group), rotation_matrix(rot_group)).reshape(n, k)
    return wr


def randomized_svd(a: np.ndarray, rank: int, omega: np.ndarray, power_iters: int = 1):
    """Rank-`rank` factors (U [n, r], S [r], Vt [r, k]) of a [n, k] by a Gaussian sketch:
    Y = A Omega (Omega [k, r + p] given), `power_iters` rounds of Y = A (A^T Y) with
    re-orthonormalisation, Q = orth(Y), B = Q^T A = U_b S V^T, U = Q U_b; truncated to r."""
    a = np.asarray(a, dtype=np.float64)
    y = a @ omega
    qy, _ = np.linalg.qr(y)
    for _ in range(power_iters):
        z, _ = np.linalg.qr(a.T @ qy)
        qy, _ = np.linalg.qr(a @ z)
    ub, s, vt = np.linalg.svd(qy.T @ a, full_matrices=False)
    return (qy @ ub)[:, :rank], s[:rank], vt[:rank]


def act_weights(act_rms: np.ndarray) -> np.ndarray:
    """Per-input-channel weights of the activation-aware objective: mean 1, floor 0.05."""
    d = np.asarray(act_rms, dtype=np.float64)
    d = d / d.mean()
    return np.maximum(d, 0.05)


def svdquant_fit(w_bits: np.ndarray, rank: int, bits: int, omegas, rot_group: int = GROUP,
                 scale_group: int = 0, act_rms=None):
    """The alternating fit.  omegas: one Gaussian test matrix [K, rank + p] per iteration (the first
    is the single-shot split, each further one a refinement).  Returns the best iterate:
    dict(l1 [K, r], l2 [r, N] float64, q, scales, err, errs) where err is the (weighted) Frobenius
    error ||(W - (deq(Q) + (L1 L2)^T)) diag(d)|| and errs the error of every iterate."""
    w = bf16_to_f64(w_bits)
    d = np.ones(w.shape[1]) if act_rms is None else act_weights(act_rms)
    target = w                              # what the branch approximates in this iterate
    best, errs = None, []
    for omega in omegas:
        u, s, vt = randomized_svd(target * d[None, :], rank, omega)
        low = (u * s) @ vt / d[None, :]     # the branch's part of W, [N, K]
        q, sc = quantize_weights(f64_to_bf16(w - low), bits, rot_group, scale_group)
        deq = dequantize_weights(q, sc, bits, rot_group, scale_group)
        err = float(np.linalg.norm((w - (deq + low)) * d[None, :]))
        errs.append(err)
        if best is None or err < best["err"]:
            root = np.sqrt(s)
            vd = vt / d[None, :]             # undo the channel weighting on the input side
            best = dict(l1=(vd.T * root[None, :]), l2=(root[:, None] * u.T), q=q, scales=sc, err=err)
        target = w - deq                    # next branch: what the current quantisation misses
    best["errs"] = errs
    return best


# ---------------------------------------------------------------------------
# 10. Q/K RMSNorm + RoPE and quantized attention (SageAttention-v1 scheme)
# ---------------------------------------------------------------------------
# Source: OrbitQuant W4A4 card, "Fused transformer": each block runs a Q/K
# RMSNorm + RoPE kernel after the Q|K|V|gate GEMM, and attention takes Q.K^T in
# INT8 with P.V in FP16, as SageAttention v1 does; "lab", Study 6: the
# rotary bands of a head are channels 0-43 (time), 44-85 (height) and 86-127
# (width).
# Readings (the pages name the scheme, not its steps):
#   - RoPE turns channel pairs (2i, 2i+1) of a head; pair i belongs to the band
#     holding channels 2i and 2i+1 and turns by pos[band] * base**(-2j / w),
#     j its index inside the band of width w, base 10000; the angles reach the
#     kernel as float32 cos / sin tables [T, 64], inputs like the activations;
#   - Q/K RMSNorm is per token and head over the 128 channels with a bf16
#     gamma [128] shared by the heads (r = 0 when mean(x^2) + eps is 0),
#     computed with the RoPE turn in float64 and rounded once to bf16;
#   - keys are smoothed before quantisation by subtracting their mean over the
#     tokens (per head and channel; softmax is unchanged by it in exact
#     arithmetic), the mean in float64 and the smoothed key rounded once to
#     float32;
#   - Q and the smoothed K are quantised per token and head to INT8 with the
#     activation quantiser's float32 steps (qmax 127); the score is the exact
#     integer dot product times s_q s_k / sqrt(128);
#   - softmax over the keys, then P.V with V converted from bf16 to fp16 (exact
#     inside fp16's range).  The oracle keeps P in float64; a kernel that rounds
#     the unnormalised P to fp16 for its MMA stays within the output tolerance.

ATTN_HEAD_DIM = 128
ROPE_BANDS = KV_BANDS
ROPE_BASE = 10000.0


def rope_tables(pos: np.ndarray, base: float = ROPE_BASE):
    """pos int [T, 3] (time, height, width) -> (cos, sin) float64 [T, 64], one angle per pair."""
    pos = np.asarray(pos, dtype=np.float64)
    ang = np.zeros((pos.shape[0], ATTN_HEAD_DIM // 2))
    p0 = 0
    for axis, w in enumerate(ROPE_BANDS):
        for j in range(w // 2):
            ang[:, p0 + j] = pos[:, axis] * base ** (-2.0 * j / w)
        p0 += w // 2
    return np.cos(ang), np.sin(ang)


def qk_norm_rope_f64(x_bits: np.ndarray, gamma_bits, cos: np.ndarray, sin: np.ndarray, eps: float) -> np.ndarray:
    """bf16 [T, H, 128] -> float64 [T, H, 128]: x / sqrt(mean(x^2) + eps) * gamma (r = 0 for a head whose
    radicand is 0, as in the normalising prologue), then pair i of token t turned by the angle whose
    cosine and sine are cos[t, i], sin[t, i]."""
    x = bf16_to_f64(x_bits)
    rad = (x * x).mean(axis=-1, keepdims=True) + eps
    with np.errstate(divide="ignore"):
        r = np.where(rad > 0, 1.0 / np.sqrt(rad), 0.0)
    u = x * r
    if gamma_bits is not None:
        u = u * bf16_to_f64(gamma_bits)[None, None, :]
    c = np.asarray(cos, np.float64)[:, None, :]
    s = np.asarray(sin, np.float64)[:, None, :]
    a, b = u[..., 0::2], u[..., 1::2]
    out = np.empty_like(u)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def qk_norm_rope(x_bits: np.ndarray, gamma_bits, cos: np.ndarray, sin: np.ndarray, eps: float) -> np.ndarray:
    """qk_norm_rope_f64 rounded once to bf16."""
    return f64_to_bf16(qk_norm_rope_f64(x_bits, gamma_bits, cos, sin, eps))


def smooth_keys(k: np.ndarray) -> np.ndarray:
    """float [T, H, D] -> float32 keys minus their float64 mean over the tokens."""
    k = np.asarray(k, np.float64)
    return (k - k.mean(axis=0, keepdims=True)).astype(np.float32)


def quantize_heads_int8(x: np.ndarray):
    """float32 [T, H, D] -> (codes int8 [T, H, D], scales float32 [T, H]), one scale per token and head."""
    t, h, d = x.shape
    q, s = quantize(np.asarray(x, np.float32).reshape(t * h, d), 8, 0)
    return q.reshape(t, h, d), s.reshape(t, h)


def attention_scores(q_bits: np.ndarray, k_bits: np.ndarray, smooth: bool = True, quant: bool = True):
    """Scores S [H, Tq, Tk] float64.  quant: the INT8 scheme; otherwise the plain q.k / sqrt(D)."""
    q = bf16_to_f64(q_bits).astype(np.float32)
    k = bf16_to_f64(k_bits).astype(np.float32)
    if smooth:
        k = smooth_keys(k)
    d = q.shape[-1]
    if not quant:
        return np.einsum("qhd,khd->hqk", q.astype(np.float64), k.astype(np.float64)) / math.sqrt(d)
    qq, sq = quantize_heads_int8(q)
    kq, sk = quantize_heads_int8(k)
    acc = np.einsum("qhd,khd->hqk", qq.astype(np.int64), kq.astype(np.int64))
    return acc * (sq.T.astype(np.float64)[:, :, None] * sk.T.astype(np.float64)[:, None, :]) / math.sqrt(d)


def sage_attention(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, smooth: bool = True,
                   quant: bool = True) -> np.ndarray:
    """bf16 q [Tq, H, D], k / v [Tk, H, D] -> float64 output [Tq, H, D]."""
    s = attention_scores(q_bits, k_bits, smooth, quant)
    s = s - s.max(axis=-1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=-1, keepdims=True)
    v16 = bf16_to_f64(v_bits).astype(np.float16).astype(np.float64)
    return np.einsum("hqk,khd->qhd", p, v16)
