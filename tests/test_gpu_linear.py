"""GPU parity of the low-bit linear (tcgen05 GEMM + fused epilogue) against the
CPU oracle: exact int32 accumulators on small shapes, bf16 outputs within the
stated tolerance, every epilogue option, ragged token counts, the config-size
layers on sampled rows, and run-to-run determinism."""
import numpy as np
import pytest
import torch

import rotated_bit_dit_b200 as R
from oracle import rbd_oracle as O
from rotated_bit_dit_b200 import inputs as I
from tests.helpers import check_output, dev_bf16, host_u16

pytestmark = pytest.mark.gpu


def build_case(M, N, K, bits, sg, seed=0, rank=0, bias=False, gate_mode=0, gate_cols=(0, 0), cf=None):
    xb = I.gaussian_bf16(seed + 1, (M, K), 1.0, 0.01, 20.0)
    wb = I.gaussian_bf16(seed + 2, (N, K), 0.02)
    case = dict(M=M, N=N, K=K, bits=bits, sg=sg, x=xb, w=wb, gate_mode=gate_mode, gate_cols=gate_cols, cf=cf)
    case["bias"] = I.gaussian_bf16(seed + 3, (N,), 0.1) if bias else None
    case["l1"] = I.gaussian_bf16(seed + 4, (K, rank), 0.01) if rank else None
    case["l2"] = I.gaussian_bf16(seed + 5, (rank, N), 0.01) if rank else None
    if gate_mode == 2:
        case["residual"] = I.gaussian_bf16(seed + 6, (M, N), 1.0)
        case["gate"] = I.gaussian_bf16(seed + 7, (N,), 1.0)
    else:
        case["residual"] = case["gate"] = None
    return case


def run_layer(case, acc_debug=False):
    M, N, K, bits, sg = case["M"], case["N"], case["K"], case["bits"], case["sg"]
    dv = lambda a: None if a is None else dev_bf16(a)
    layer = R.RotatedLowBitLinear(dv(case["w"]), bits=bits, scale_group=sg, bias=dv(case["bias"]),
                                  l1=dv(case["l1"]), l2=dv(case["l2"]), gate_mode=case["gate_mode"],
                                  gate_cols=case["gate_cols"], gate=dv(case["gate"]), code_format=case.get("cf"))
    acc = None
    if acc_debug:
        shape = (K // 64, M, N) if sg else (M, N)
        acc = torch.zeros(shape, dtype=torch.int32, device="cuda")
    y = layer(dv(case["x"]), residual=dv(case["residual"]), acc_debug=acc)
    assert R.rbd_check() == 0
    return host_u16(y), (acc.cpu().numpy() if acc is not None else None), layer


def reference(case, rows=None):
    return O.linear_reference(case["x"], case["w"], case["bits"], 256, case["sg"], bias=case["bias"],
                              l1=case["l1"], l2=case["l2"], gate_mode=case["gate_mode"],
                              gate_cols=case["gate_cols"], gate=case["gate"], residual=case["residual"],
                              rows=rows)


def exact_acc(case, ref):
    qw = O.unpack_int4(ref["wq"]) if case["bits"] == 4 else ref["wq"]
    if case["sg"]:
        return O.gemm_acc_grouped(ref["codes"], qw, 64)
    return O.gemm_acc(ref["codes"], qw)


VARIANTS = {
    "plain": dict(),
    "bias": dict(bias=True),
    "rank16": dict(rank=16),
    "rank32": dict(rank=32),
    "rank64": dict(rank=64),
    "sigmoid": dict(gate_mode=1, gate_cols=(128, 256)),
    "gated_residual": dict(gate_mode=2),
    "all": dict(bias=True, rank=32, gate_mode=1, gate_cols=(64, 200)),
}


# (bits, scale group, activation code format): INT4 with group scales runs both the FP8 (E4M3 codes,
# the layer's default) and the INT8 tensor-core paths
PATHS = [(4, 0, None), (4, 64, None), (4, 64, 0), (8, 0, None), (8, 64, None)]


# 64 tokens run on the small-token kernel, 96 on the tiled tcgen05 kernel
@pytest.mark.parametrize("M", [64, 96])
@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("bits,sg,cf", PATHS)
def test_tiny_layer_variants(variant, bits, sg, cf, M):
    case = build_case(M, 256, 256, bits, sg, seed=10, cf=cf, **VARIANTS[variant])
    y, acc, _ = run_layer(case, acc_debug=True)
    ref = reference(case)
    assert np.array_equal(acc.astype(np.int64), exact_acc(case, ref))
    check_output(y, ref["ref64"], ref["ref_bf16"])


@pytest.mark.parametrize("M", [1, 7, 13, 33, 64, 65, 128, 200, 333])
@pytest.mark.parametrize("bits,sg,cf", PATHS)
def test_ragged_tokens_several_tiles(M, bits, sg, cf):
    # M <= 64: the small-token kernel (one to eight 8-token MMA columns, ragged);
    # M > 64: the tiled kernel
    # N spans 3 feature tiles, K spans 6 stages (wraps the 4-deep ring), M ends ragged
    case = build_case(M, 384, 768, bits, sg, seed=20 + M, bias=True, rank=16, cf=cf)
    y, acc, _ = run_layer(case, acc_debug=True)
    ref = reference(case)
    assert np.array_equal(acc.astype(np.int64), exact_acc(case, ref))
    check_output(y, ref["ref64"], ref["ref_bf16"])


@pytest.mark.parametrize("M,N,K", [
    (1, 12288, 3072),    # the Q|K|V|gate shape at one token: 768 blocks of 16 features
    (16, 3072, 12288),   # ff.down shape: 24 groups per warp, rings wrap many times
    (40, 128, 1280),     # 20 groups over 8 warps (uneven split), 5 token columns
    (3, 256, 256),       # 4 groups: four of the eight warps have no work
])
@pytest.mark.parametrize("bits,sg,cf", PATHS)
def test_small_token_kernel_shapes(M, N, K, bits, sg, cf):
    case = build_case(M, N, K, bits, sg, seed=50 + M, bias=True, rank=32 if N <= 4096 else 0,
                      gate_mode=2 if bits == 8 else 1, gate_cols=(N // 2, N), cf=cf)
    y, acc, _ = run_layer(case, acc_debug=True)
    ref = reference(case)
    assert np.array_equal(acc.astype(np.int64), exact_acc(case, ref))
    check_output(y, ref["ref64"], ref["ref_bf16"])


@pytest.mark.parametrize("bits,rank", [(8, 0), (4, 32)])
def test_long_k_group_scales_two_stage_pipeline(bits, rank):
    # K = 12288 with group scales: the per-tile scale table leaves room for two
    # pipeline stages only (fewer stages than producer warps)
    case = build_case(300, 256, 12288, bits, 64, seed=40, rank=rank, bias=True)
    y, acc, _ = run_layer(case, acc_debug=False)
    ref = reference(case)
    check_output(y, ref["ref64"], ref["ref_bf16"])


@pytest.mark.parametrize("M,N,K,bits,sg,rank,cf", [
    (2048, 2560, 512, 4, 64, 32, None),   # group scales, FP8 path: 320 tiles of 128 x 128 over 148 CTAs
    (2048, 2560, 512, 4, 64, 32, 0),      # the same on the INT8 path
    (4096, 2048, 1024, 8, 0, 0, None),    # row scales: 256 tiles of 128 x 256
    (4096, 2048, 512, 4, 0, 16, None),    # INT4 row scales, 256 tiles
    (1500, 2304, 256, 8, 64, 0, None),    # INT8 group scales, 216 tiles, ragged last token tile
])
def test_persistent_grid_exact_accumulators(M, N, K, bits, sg, rank, cf):
    # more tiles than CTAs: every CTA walks several tiles, so the accumulator buffers' phases wrap
    # across tiles and the per-tile scale tables are restaged; every int32 accumulator is checked
    case = build_case(M, N, K, bits, sg, seed=80 + M % 97, rank=rank, bias=True, cf=cf)
    y, acc, _ = run_layer(case, acc_debug=True)
    ref = reference(case)
    assert np.array_equal(acc.astype(np.int64), exact_acc(case, ref))
    check_output(y, ref["ref64"], ref["ref_bf16"])


def test_deterministic_run_to_run():
    case = build_case(300, 512, 1024, 4, 64, seed=30, rank=32, bias=True, gate_mode=1, gate_cols=(0, 128))
    y1, _, layer = run_layer(case)
    x = dev_bf16(case["x"])
    y2 = host_u16(layer(x))
    assert np.array_equal(y1, y2)


def _sample_rows(M, n=48, seed=0):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, M - 1], rng.choice(M, n, replace=False)]))
    return rows


def test_w8a8_ffdown_config_sampled_rows():
    cfg = I.CONFIGS["w8a8_ffdown"]
    t = I.make_layer_inputs(cfg, seed=0)
    case = dict(M=cfg["M"], N=cfg["N"], K=cfg["K"], bits=8, sg=0, x=t["x"], w=t["w"], bias=None, l1=None,
                l2=None, gate_mode=2, gate_cols=(0, 0), gate=t["gate"], residual=t["residual"])
    y, _, _ = run_layer(case)
    rows = _sample_rows(cfg["M"])
    ref = reference(case, rows=rows)
    check_output(y[rows], ref["ref64"], ref["ref_bf16"])


def test_w4a4_qkvg_config_sampled_rows():
    cfg = I.CONFIGS["w4a4_qkvg"]
    t = I.make_layer_inputs(cfg, seed=0)
    case = dict(M=cfg["M"], N=cfg["N"], K=cfg["K"], bits=4, sg=64, x=t["x"], w=t["w"], bias=None,
                l1=t["l1"], l2=t["l2"], gate_mode=1, gate_cols=cfg["gate_cols"], gate=None, residual=None)
    y, _, _ = run_layer(case)
    rows = _sample_rows(cfg["M"], seed=1)
    ref = reference(case, rows=rows)
    stats = check_output(y[rows], ref["ref64"], ref["ref_bf16"])
    assert stats["rel64"] < 5e-3


@pytest.mark.parametrize("bits,sg,rank,gate_mode", [(4, 64, 32, 1), (8, 0, 0, 2), (4, 0, 16, 0)])
def test_forward_host_matches_the_device_call(bits, sg, rank, gate_mode):
    # host-resident tokens streamed in chunks (ragged last chunk) give the device call's output bit for bit
    case = build_case(1000, 256, 512, bits, sg, seed=60, rank=rank, bias=True, gate_mode=gate_mode,
                      gate_cols=(128, 256))
    y_dev, _, layer = run_layer(case)
    xh = torch.from_numpy(np.ascontiguousarray(case["x"]).view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = torch.empty((1000, 256), dtype=torch.bfloat16).pin_memory()
    rh = None
    if case["residual"] is not None:
        rh = torch.from_numpy(np.ascontiguousarray(case["residual"]).view(np.int16)).view(torch.bfloat16).pin_memory()
    layer.forward_host(xh, yh, rh, chunk=384)
    torch.cuda.synchronize()
    assert R.rbd_check() == 0
    assert np.array_equal(yh.view(torch.int16).numpy().view(np.uint16), y_dev)


def test_intermediates_are_kept_per_stream():
    # calls queued on two streams must not share codes / scales / Ld buffers
    case = build_case(64, 256, 256, 4, 64, seed=70, rank=16)
    _, _, layer = run_layer(case)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    with torch.cuda.stream(s1):
        b1 = layer.buffers(64, torch.device("cuda"))
    with torch.cuda.stream(s2):
        b2 = layer.buffers(64, torch.device("cuda"))
    with torch.cuda.stream(s1):
        b1b = layer.buffers(64, torch.device("cuda"))
    assert b1[0].data_ptr() != b2[0].data_ptr() and b1[1].data_ptr() != b2[1].data_ptr()
    assert b1[0].data_ptr() == b1b[0].data_ptr()


# The small-M sweep's layer (K = N = 3072) at every token count it times, on both kernels
# (M <= 64 the small-token kernel, above it the tiled one): every output and accumulator.
@pytest.mark.parametrize("M", [1, 16, 64, 256, 1024])
@pytest.mark.parametrize("sg,cf", [(0, None), (64, None)])
def test_small_m_sweep_layer_shapes(M, sg, cf):
    case = dict(M=M, N=3072, K=3072, bits=4, sg=sg, cf=cf, x=I.gaussian_bf16(2 + M, (M, 3072), 1.0, 0.005, 30.0),
                w=I.gaussian_bf16(1, (3072, 3072), 0.02), bias=None, l1=None, l2=None, gate_mode=0,
                gate_cols=(0, 0), gate=None, residual=None)
    y, acc, _ = run_layer(case, acc_debug=True)
    ref = reference(case)
    assert np.array_equal(acc.astype(np.int64), exact_acc(case, ref))
    check_output(y, ref["ref64"], ref["ref_bf16"])


# The 28-block stack's layer shapes at its token count (M = 16384, per-row scales, the INT4
# and the protected INT8 layers), in the launch configuration the stack sweep times: sampled
# rows against the oracle.
STACK_SHAPES = [(4, 3072, 3072), (8, 3072, 3072), (4, 3072, 12288), (4, 12288, 3072), (8, 12288, 3072)]


@pytest.mark.parametrize("bits,K,N", STACK_SHAPES)
def test_stack_layer_shapes_sampled_rows(bits, K, N):
    M = 16384
    case = dict(M=M, N=N, K=K, bits=bits, sg=0, x=I.gaussian_bf16(K, (M, K), 1.0, 0.005, 30.0),
                w=I.gaussian_bf16(7 + N, (N, K), 0.02), bias=None, l1=None, l2=None, gate_mode=0,
                gate_cols=(0, 0), gate=None, residual=None)
    y, _, _ = run_layer(case)
    rows = _sample_rows(M, n=32, seed=K + N + bits)
    ref = reference(case, rows=rows)
    check_output(y[rows], ref["ref64"], ref["ref_bf16"])
