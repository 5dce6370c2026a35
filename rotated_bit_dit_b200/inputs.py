"""Seeded synthetic inputs for the rotated low-bit linear layer.

This module only draws numbers; it holds none of the layer's arithmetic
(no rotation, no quantisation, no matmul).  The CPU oracle and the CUDA path
both consume the bf16 bit patterns produced here, so both see identical
inputs.

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) over a counter, two 53-bit uniforms per
normal draw, Box-Muller transform, scale, optional channel outliers, then
round-to-nearest-even to bf16.

Workload shapes follow the diffusion-transformer layers described on the
Krea-2 model cards ("Fused transformer" section of Krea-2-Turbo-OrbitQuant-W4A4:
grouped Q|K|V|gate projection, SwiGLU gate|up, protected ff.down): hidden 3072,
MLP 12288, 4096 tokens for a 1024x1024 image and 16384 for 2048x2048.
"""
from __future__ import annotations

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Per-tensor seed offsets (added to a base seed).
SEED_X, SEED_W, SEED_L1, SEED_L2, SEED_RES, SEED_GATE, SEED_BIAS, SEED_OUTLIER = range(8)


def splitmix64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """n successive SplitMix64 outputs for stream `seed`, starting at counter `offset`."""
    with np.errstate(over="ignore"):
        i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) * np.uint64(0x632BE59BD9B4E019) + i * _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        z = z ^ (z >> np.uint64(31))
    return z


def uniform01(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """Uniforms in (0, 1]: the top 53 bits of each SplitMix64 output, plus one ulp."""
    z = splitmix64(seed, n, offset)
    return ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def normal(seed: int, n: int) -> np.ndarray:
    """n standard normals (float64), Box-Muller cosine branch, two uniforms per draw."""
    u = uniform01(seed, 2 * n)
    u1, u2 = u[0::2], u[1::2]
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rnd = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    out = ((u + rnd) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def outlier_channels(seed: int, k: int, frac: float) -> np.ndarray:
    """The round(frac*k) (at least one) channel indices chosen for outliers, sorted."""
    n = max(1, int(round(frac * k)))
    keys = splitmix64(seed + SEED_OUTLIER, k)
    return np.sort(np.argsort(keys, kind="stable")[:n])


def gaussian_bf16(seed: int, shape, std: float = 1.0, outlier_frac: float = 0.0,
                  outlier_scale: float = 1.0, outlier_seed: int | None = None) -> np.ndarray:
    """bf16 bit patterns of N(0, std^2) draws; whole last-axis channels scaled for outliers."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    v = normal(seed, n).reshape(shape) * std
    if outlier_frac > 0.0:
        ch = outlier_channels(seed if outlier_seed is None else outlier_seed, shape[-1], outlier_frac)
        v[..., ch] *= outlier_scale
    return f32_to_bf16_bits(v.astype(np.float32))


# ---------------------------------------------------------------------------
# Workloads.  Every tensor is generated from base_seed + a fixed per-tensor offset.
# ---------------------------------------------------------------------------

CONFIGS = {
    # 64x256x256 W4A4, one rotation group, per-token / per-row scales.
    "tiny_w4a4": dict(M=64, K=256, N=256, bits=4, scale_group=0, x_outlier=(0.01, 20.0),
                      rank=0, gate_mode=0),
    # ff.down-style W8A8 layer with a gated residual add.
    "w8a8_ffdown": dict(M=4096, K=12288, N=3072, bits=8, scale_group=0, x_outlier=(0.005, 30.0),
                        rank=0, gate_mode=2),
    # Grouped Q|K|V|gate W4A4 projection, group-64 scales, rank-32 branch, sigmoid on the gate quarter.
    "w4a4_qkvg": dict(M=4096, K=3072, N=4 * 3072, bits=4, scale_group=64, x_outlier=(0.005, 30.0),
                      rank=32, gate_mode=1, gate_cols=(3 * 3072, 4 * 3072)),
    # Small-M sweep layer (K = N = 3072), per-token / per-row scales, no branch.
    "smallm_w4a4": dict(M=1, K=3072, N=3072, bits=4, scale_group=0, x_outlier=(0.005, 30.0),
                        rank=0, gate_mode=0),
}


def video_positions(frames: int, height: int, width: int, t0: int = 0) -> np.ndarray:
    """int32 [frames * height * width, 3] (time, row, column) of a patch grid, frame-major, times
    starting at t0: the token positions of a video (or, with one frame, an image) latent."""
    t, h, w = np.meshgrid(np.arange(frames) + t0, np.arange(height), np.arange(width), indexing="ij")
    return np.stack([t.ravel(), h.ravel(), w.ravel()], axis=1).astype(np.int32)


def make_layer_inputs(cfg: dict, seed: int = 0, M: int | None = None) -> dict:
    """All bf16 inputs of one layer call as uint16 bit-pattern arrays.

    Keys: x [M,K], w [N,K], and when used l1 [K,r], l2 [r,N], residual [M,N],
    gate [N], bias [N].
    """
    M = cfg["M"] if M is None else M
    K, N = cfg["K"], cfg["N"]
    frac, scale = cfg.get("x_outlier", (0.0, 1.0))
    out = {
        "x": gaussian_bf16(seed + SEED_X, (M, K), 1.0, frac, scale, outlier_seed=seed),
        "w": gaussian_bf16(seed + SEED_W, (N, K), 0.02),
    }
    r = cfg.get("rank", 0)
    if r:
        out["l1"] = gaussian_bf16(seed + SEED_L1, (K, r), 0.01)
        out["l2"] = gaussian_bf16(seed + SEED_L2, (r, N), 0.01)
    if cfg.get("gate_mode", 0) == 2:
        out["residual"] = gaussian_bf16(seed + SEED_RES, (M, N), 1.0)
        out["gate"] = gaussian_bf16(seed + SEED_GATE, (N,), 1.0)
    if cfg.get("bias", False):
        out["bias"] = gaussian_bf16(seed + SEED_BIAS, (N,), 0.1)
    return out
