"""The C-ABI library on the CPU: it loads, exports every declared entry point,
and rejects invalid calls before launching anything (no GPU needed: the
validation paths return before the first CUDA call)."""
import ctypes
import os
import re

import pytest

import rotated_bit_dit_b200 as R
from rotated_bit_dit_b200 import _binding as B

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "rbd.h")


def declared_entry_points():
    text = open(HDR).read()
    return re.findall(r"^(?:rbd_status|const char\*|int64_t)\s+(rbd_\w+)\(", text, re.M)


def test_library_loads_and_exports_every_declared_symbol():
    lib = R.load()
    names = declared_entry_points()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.EXPORTED)
    assert R.rbd_version().startswith("rotated_bit_dit_b200")


def test_status_strings():
    for code, name in B.STATUS_NAMES.items():
        assert R.rbd_status_string(code) == name
    assert R.rbd_status_string(99) == "RBD_ERR_UNKNOWN"


FAKE = ctypes.c_void_p(0x10000)          # 16-byte aligned, never dereferenced
FAKE_MIS = ctypes.c_void_p(0x10001)      # misaligned


def q(bits=4, rot=256, sg=0, cf=0):
    return B.QCfg(bits, rot, sg, cf)


def test_code_format_validation_without_gpu():
    lib = R.load()
    e4 = B.CODES_E4M3
    # an unknown format; E4M3 with 8-bit codes
    assert lib.rbd_rot_quant_act(FAKE, 4, 256, 256, q(cf=2), FAKE, FAKE, None) == 1
    assert lib.rbd_rot_quant_act(FAKE, 4, 256, 256, q(bits=8, cf=e4), FAKE, FAKE, None) == 2
    assert lib.rbd_lowrank_fused(FAKE, 4, 256, 256, q(bits=8, sg=64, cf=e4), FAKE, FAKE, FAKE, 32, FAKE, None) == 2
    # weight packers store two's-complement codes only
    assert lib.rbd_pack_weights_int4(FAKE, 4, 256, q(cf=e4), FAKE, FAKE, None) == 2
    assert lib.rbd_pack_weights_int8(FAKE, 4, 256, q(bits=8, cf=e4), FAKE, FAKE, None) == 2
    # the E4M3 linear is the W4A4 group-scale path
    assert _lin(lib.rbd_w4a4_linear, cfg=q(sg=0, cf=e4)) == 2
    assert _lin(lib.rbd_w8a8_linear, cfg=q(bits=8, sg=64, cf=e4)) == 2
    assert _lin(lib.rbd_w4a4_linear, cfg=q(sg=64, cf=3)) == 1
    assert _lin(lib.rbd_w4a4_linear, M=0, cfg=q(sg=64, cf=e4)) == 0
    # the struct is four int32 fields, as the header declares
    assert ctypes.sizeof(B.QCfg) == 16


@pytest.mark.parametrize("args,expect", [
    ((FAKE, 4, 100, 100, q(), FAKE, FAKE, None), 2),            # K not a multiple of 256
    ((FAKE, 4, 256, 256, q(bits=5), FAKE, FAKE, None), 1),      # bad bits
    ((FAKE, 4, 256, 256, q(rot=128), FAKE, FAKE, None), 2),     # unsupported rotation group
    ((FAKE, 4, 256, 256, q(sg=32), FAKE, FAKE, None), 2),       # unsupported scale group
    ((FAKE, -1, 256, 256, q(), FAKE, FAKE, None), 1),           # negative M
    ((None, 4, 256, 256, q(), FAKE, FAKE, None), 1),            # null input
    ((FAKE, 4, 256, 128, q(), FAKE, FAKE, None), 1),            # ldx < K
    ((FAKE_MIS, 4, 256, 256, q(), FAKE, FAKE, None), 3),        # misaligned x
    ((FAKE, 4, 256, 260, q(), FAKE, FAKE, None), 3),            # row stride not 16-byte aligned
    ((FAKE, 4, 32768, 32768, q(), FAKE, FAKE, None), 2),        # K above the supported maximum
])
def test_rot_quant_rejects_before_launch(args, expect):
    assert R.load().rbd_rot_quant_act(*args) == expect


def test_zero_rows_is_a_noop_without_pointers():
    assert R.load().rbd_rot_quant_act(None, 0, 256, 256, q(), None, None, None) == 0


def _lin(lib_fn, M=128, N=128, K=256, cfg=None, epi=None, codes=FAKE, w=FAKE, y=FAKE, ldy=None):
    cfg = cfg or q()
    e = epi if epi is not None else B.Epilogue()
    return lib_fn(codes, FAKE, w, FAKE, M, N, K, cfg, ctypes.byref(e), y, N if ldy is None else ldy, None)


def test_linear_rejects_before_launch():
    lib = R.load()
    w4, w8 = lib.rbd_w4a4_linear, lib.rbd_w8a8_linear
    assert _lin(w4, cfg=q(bits=8)) == 1                      # W4A4 with 8-bit config
    assert _lin(w8, cfg=q(bits=4)) == 1
    assert _lin(w4, K=192) == 2                              # K % 128
    assert _lin(w4, N=96) == 2                               # N % 128
    assert _lin(w4, codes=FAKE_MIS) == 3
    assert _lin(w4, y=FAKE_MIS) == 3
    assert _lin(w4, ldy=64) == 1                             # ldy < N
    e = B.Epilogue()
    e.r = 24
    assert _lin(w4, epi=e) == 2                              # unsupported rank
    e = B.Epilogue()
    e.r = 32
    assert _lin(w4, epi=e) == 1                              # rank without factors
    e = B.Epilogue()
    e.gate_mode = 2
    assert _lin(w4, epi=e) == 1                              # gated residual without tensors
    e = B.Epilogue()
    e.gate_mode = 1
    e.gate_col0, e.gate_col1 = 64, 512
    assert _lin(w4, epi=e) == 1                              # gate columns out of range
    e = B.Epilogue()
    e.gate_mode = 3
    assert _lin(w4, epi=e) == 1
    assert _lin(w4, M=0) == 0                                # empty batch: nothing to do


def test_lowrank_and_pack_reject_before_launch():
    lib = R.load()
    assert lib.rbd_lowrank_fused(FAKE, 4, 256, 256, q(), FAKE, FAKE, FAKE, 24, FAKE, None) == 2
    assert lib.rbd_lowrank_fused(FAKE, 4, 256, 256, q(), FAKE, FAKE, None, 32, FAKE, None) == 1
    assert lib.rbd_pack_weights_int4(FAKE, 4, 256, q(bits=8), FAKE, FAKE, None) == 1
    assert lib.rbd_pack_weights_int8(FAKE, 4, 256, q(bits=4), FAKE, FAKE, None) == 1
    assert lib.rbd_debug_timeout_probe(0, None) == 1


def test_nvfp4_validation_without_gpu():
    lib = R.load()
    assert lib.rbd_nvfp4_scale_bytes(1, 256) == 128 * 16
    assert lib.rbd_nvfp4_scale_bytes(129, 512) == 256 * 32
    assert lib.rbd_nvfp4_scale_bytes(4, 100) == -1
    null = ctypes.c_void_p(0)
    # K not a multiple of 256; unsupported rotation group; null output
    assert lib.rbd_nvfp4_quant(FAKE, 4, 320, 320, 256, FAKE, FAKE, FAKE, FAKE, null) == 2
    assert lib.rbd_nvfp4_quant(FAKE, 4, 256, 256, 64, FAKE, FAKE, FAKE, FAKE, null) == 2
    assert lib.rbd_nvfp4_quant(FAKE, 4, 256, 256, 256, null, FAKE, FAKE, FAKE, null) == 1
    assert lib.rbd_nvfp4_quant(FAKE_MIS, 4, 256, 256, 256, FAKE, FAKE, FAKE, FAKE, null) == 3
    assert lib.rbd_nvfp4_quant(FAKE, 0, 256, 256, 256, null, null, null, null, null) == 0
    # linear: N not a multiple of 128, unsupported rank, rank without factors, misaligned scales
    e = B.Epilogue()
    assert lib.rbd_nvfp4_linear(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 64, 256, ctypes.byref(e), FAKE, 64, null) == 2
    e.r = 24
    assert lib.rbd_nvfp4_linear(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 128, 256, ctypes.byref(e), FAKE, 128,
                                null) == 2
    e.r = 16
    assert lib.rbd_nvfp4_linear(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 128, 256, ctypes.byref(e), FAKE, 128,
                                null) == 1
    e.ld, e.l2t = FAKE_MIS.value, FAKE.value
    assert lib.rbd_nvfp4_linear(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 128, 256, ctypes.byref(e), FAKE, 128,
                                null) == 3
    e.ld = e.l2t = None
    e.r = 0
    assert lib.rbd_nvfp4_linear(FAKE, FAKE_MIS, FAKE, FAKE, FAKE, FAKE, 4, 128, 256, ctypes.byref(e), FAKE, 128,
                                null) == 3


def test_nvfp4_noalloc_validation_without_gpu():
    lib = R.load()
    null = ctypes.c_void_p(0)
    assert lib.rbd_nvfp4_quant_noalloc(FAKE, 0, 256, 256, 256, null, null, null, null) == 0
    assert lib.rbd_nvfp4_quant_noalloc(FAKE, 0, 320, 320, 256, null, null, null, null) == 2
    assert lib.rbd_nvfp4_quant_noalloc(FAKE, -1, 256, 256, 256, FAKE, FAKE, FAKE, null) == 1
    assert lib.rbd_nvfp4_quant_noalloc(FAKE, 4, 256, 256, 256, null, FAKE, FAKE, null) == 1


def test_norm_rot_quant_validation_without_gpu():
    lib = R.load()
    null = ctypes.c_void_p(0)
    eps = ctypes.c_float(1e-6)
    assert lib.rbd_norm_rot_quant_act(FAKE, 4, 256, 256, None, None, None, -1.0, q(), FAKE, FAKE, None) == 1
    assert lib.rbd_norm_rot_quant_act(FAKE, 4, 256, 256, None, None, None, float("nan"), q(), FAKE, FAKE, None) == 1
    assert lib.rbd_norm_rot_quant_act(FAKE, 4, 256, 256, None, None, None, float("inf"), q(), FAKE, FAKE, None) == 1
    assert lib.rbd_norm_rot_quant_act(FAKE, 4, 256, 256, FAKE_MIS, None, None, eps, q(), FAKE, FAKE, None) == 3
    assert lib.rbd_norm_rot_quant_act(FAKE, 4, 256, 256, None, FAKE_MIS, None, eps, q(), FAKE, FAKE, None) == 3
    assert lib.rbd_norm_rot_quant_act(FAKE, 4, 100, 100, None, None, None, eps, q(), FAKE, FAKE, None) == 2
    assert lib.rbd_norm_rot_quant_act(FAKE, 4, 256, 256, None, None, None, eps, q(bits=5), FAKE, FAKE, None) == 1
    assert lib.rbd_norm_rot_quant_act(FAKE, 4, 256, 256, None, None, None, eps, q(), null, FAKE, None) == 1
    assert lib.rbd_norm_rot_quant_act(FAKE, 0, 256, 256, None, None, None, eps, q(), null, null, None) == 0


def test_lowrank_down_validation_without_gpu():
    lib = R.load()
    null = ctypes.c_void_p(0)
    assert lib.rbd_lowrank_down(FAKE, 4, 256, 256, FAKE, 24, FAKE, None) == 2      # rank
    assert lib.rbd_lowrank_down(FAKE, 4, 192, 192, FAKE, 32, FAKE, None) == 2      # K % 128
    assert lib.rbd_lowrank_down(FAKE, 4, 256, 256, null, 32, FAKE, None) == 1      # no factor
    assert lib.rbd_lowrank_down(FAKE, 4, 256, 128, FAKE, 32, FAKE, None) == 1      # ldx < K
    assert lib.rbd_lowrank_down(FAKE_MIS, 4, 256, 256, FAKE, 32, FAKE, None) == 3
    assert lib.rbd_lowrank_down(FAKE, 0, 256, 256, null, 32, null, None) == 0      # empty batch


def test_kv4_validation_without_gpu():
    lib = R.load()
    null = ctypes.c_void_p(0)
    enc, dec = lib.rbd_kv4_encode, lib.rbd_kv4_decode
    assert enc(FAKE, 4, 2, 256, 3, FAKE, FAKE, 8, 0, None) == 2          # groups per band
    assert enc(FAKE, 9, 2, 256, 1, FAKE, FAKE, 8, 0, None) == 1          # slice longer than the ring
    assert enc(FAKE, 4, 2, 256, 1, FAKE, FAKE, 8, 8, None) == 1          # slot0 outside the ring
    assert enc(FAKE, 4, 2, 200, 1, FAKE, FAKE, 8, 0, None) == 1          # ldt < 128 H
    assert enc(FAKE_MIS, 4, 2, 256, 1, FAKE, FAKE, 8, 0, None) == 3
    assert enc(FAKE, 4, 2, 260, 1, FAKE, FAKE, 8, 0, None) == 3          # row stride not 16-byte aligned
    assert enc(FAKE, 0, 2, 256, 1, null, null, 8, 0, None) == 0          # empty slice
    assert dec(FAKE, FAKE, 8, 0, 4, 0, 1, FAKE, 256, None) == 1          # no heads
    assert dec(null, FAKE, 8, 0, 4, 2, 1, FAKE, 256, None) == 1


@pytest.mark.parametrize("lang,std", [("c", "-std=c99"), ("c++", "-std=c++17")])
def test_header_is_plain_c_and_cxx(lang, std):
    # the boundary header carries no torch or CUDA types: it compiles alone as C99 and as C++
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    r = subprocess.run([cc, "-fsyntax-only", "-Wall", "-Wextra", "-Werror", "-x", lang, std, HDR],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_qk_norm_rope_validation_without_gpu():
    lib = R.load()
    null = ctypes.c_void_p(0)
    f = lib.rbd_qk_norm_rope
    assert f(FAKE, 0, 2, 256, null, null, null, 1e-6, null, 256, null) == 0        # empty: nothing to do
    assert f(FAKE, -1, 2, 256, null, FAKE, FAKE, 1e-6, FAKE, 256, null) == 1
    assert f(FAKE, 4, 0, 256, null, FAKE, FAKE, 1e-6, FAKE, 256, null) == 1
    assert f(FAKE, 4, 2, 256, null, FAKE, FAKE, float("nan"), FAKE, 256, null) == 1
    assert f(FAKE, 4, 2, 256, null, FAKE, FAKE, -1.0, FAKE, 256, null) == 1
    assert f(FAKE, 4, 2, 256, null, null, FAKE, 1e-6, FAKE, 256, null) == 1
    assert f(FAKE, 4, 2, 200, null, FAKE, FAKE, 1e-6, FAKE, 256, null) == 1        # row shorter than the heads
    assert f(FAKE, 4, 2, 256, null, FAKE, FAKE, 1e-6, FAKE, 100, null) == 1
    assert f(FAKE_MIS, 4, 2, 256, null, FAKE, FAKE, 1e-6, FAKE, 256, null) == 3
    assert f(FAKE, 4, 2, 256, FAKE_MIS, FAKE, FAKE, 1e-6, FAKE, 256, null) == 3
    assert f(FAKE, 4, 2, 260, null, FAKE, FAKE, 1e-6, FAKE, 256, null) == 3        # stride not a multiple of 8
    assert f(FAKE, 1 << 30, 4, 512, null, FAKE, FAKE, 1e-6, FAKE, 512, null) == 2  # T * H beyond 2^30
    t = lib.rbd_rope_tables
    assert t(FAKE, 0, 10000.0, null, null, null) == 0
    assert t(FAKE, -1, 10000.0, FAKE, FAKE, null) == 1
    assert t(FAKE, 4, 0.0, FAKE, FAKE, null) == 1
    assert t(FAKE, 4, float("inf"), FAKE, FAKE, null) == 1
    assert t(null, 4, 10000.0, FAKE, FAKE, null) == 1
    assert t(ctypes.c_void_p(0x10002), 4, 10000.0, FAKE, FAKE, null) == 3
    assert t(FAKE, 4, 10000.0, FAKE_MIS, FAKE, null) == 3
    assert t(FAKE, 1 << 26, 10000.0, FAKE, FAKE, null) == 2


def test_attention_validation_without_gpu():
    lib = R.load()
    null = ctypes.c_void_p(0)
    assert lib.rbd_attn_workspace_bytes(1000, 2) == (4 + 1) * 2 * 128 * 8     # 4 chunks of 256 keys + the mean
    assert lib.rbd_attn_workspace_bytes(0, 2) == -1
    aq, ai = lib.rbd_attn_quant, lib.rbd_attn_int8
    args = lambda **kw: [kw.get(n, d) for n, d in (
        ("q", FAKE), ("ldq", 256), ("k", FAKE), ("ldk", 256), ("v", FAKE), ("ldv", 256), ("Tq", 4), ("Tk", 8),
        ("H", 2), ("qc", FAKE), ("sq", FAKE), ("kc", FAKE), ("sk", FAKE), ("vt", FAKE), ("tkp", 8), ("work", FAKE),
        ("stream", null))]
    assert aq(*args(tkp=4)) == 1                 # padded key count below Tk
    assert aq(*args(tkp=12)) == 1                # padded key count not a multiple of 8
    assert aq(*args(Tk=0)) == 1                  # queries without keys
    assert aq(*args(Tq=0, Tk=0)) == 0            # nothing to do
    assert aq(*args(ldk=200)) == 1               # row shorter than the heads
    assert aq(*args(work=null)) == 1
    assert aq(*args(v=FAKE_MIS)) == 3
    assert aq(*args(ldq=260)) == 3
    assert aq(*args(H=300)) == 2
    assert ai(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8, 2, 8, FAKE, 200, null) == 1   # ldo < H * 128
    assert ai(FAKE, FAKE, FAKE, FAKE, FAKE, 4, 0, 2, 8, FAKE, 256, null) == 1   # no keys
    assert ai(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 8, 2, 8, FAKE, 256, null) == 0   # no queries
    assert ai(FAKE, FAKE, FAKE, FAKE_MIS, FAKE, 4, 8, 2, 8, FAKE, 256, null) == 3


def test_svdquant_validation_without_gpu():
    lib = R.load()
    null = ctypes.c_void_p(0)
    assert lib.rbd_svdquant_workspace_bytes(384, 3072, 32, 8, q()) > 384 * 3072 * 24
    assert lib.rbd_svdquant_workspace_bytes(384, 3072, 300, 8, q()) == -1          # rank + oversample > 256
    assert lib.rbd_svdquant_workspace_bytes(384, 3000, 32, 8, q()) == -1           # K not a multiple of 256
    assert lib.rbd_svdquant_workspace_bytes(384, 3072, 32, 8, q(cf=1)) == -1       # codes of weights are int8
    f = lib.rbd_svdquant_fit
    ok = lambda **kw: [kw.get(n, dflt) for n, dflt in (
        ("w", FAKE), ("N", 384), ("K", 3072), ("cfg", q()), ("rank", 32), ("os", 8), ("iters", 3), ("om", FAKE),
        ("ar", null), ("q", FAKE), ("sc", FAKE), ("l1", FAKE), ("l2", FAKE), ("errs", FAKE), ("best", null),
        ("work", FAKE), ("stream", null))]
    assert f(*ok(iters=0)) == 1
    assert f(*ok(om=null)) == 1
    assert f(*ok(rank=0)) == 1
    assert f(*ok(N=16)) == 2                     # rank + oversample > N
    assert f(*ok(w=FAKE_MIS)) == 3
