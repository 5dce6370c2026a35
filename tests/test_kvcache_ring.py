"""Int4KVCache, the ring of INT4 slots over the KV codec: a script of slice writes,
rolling evictions and slice reads must leave the cache reading back exactly the
oracle's encode/decode of the tokens it holds, in order.  On the CPU the two codec
calls are replaced by oracle-backed stand-ins that enforce the C ABI's ring
preconditions (the bookkeeping is what is under test); on the GPU the same script
runs through librbd.so."""
import numpy as np
import pytest
import torch

import rotated_bit_dit_b200 as R
from oracle import rbd_oracle as O
from rotated_bit_dit_b200 import inputs as I
from rotated_bit_dit_b200 import kvcache as K

CAP, H = 16, 2
# (op, argument): write t tokens, evict n, read (first, count) with count None = to the end
SCRIPT = [("write", 5), ("read", (0, None)), ("write", 7), ("read", (3, 6)), ("write", 0),
          ("write", 6), ("read", (0, None)), ("read", (1, 14)), ("evict", 4), ("read", (0, None)),
          ("write", 16), ("read", (0, None)), ("read", (15, 1)), ("write", 3), ("evict", 0),
          ("read", (2, 9)), ("write", 1), ("evict", 16), ("read", (0, None)), ("write", 11),
          ("write", 9), ("read", (0, None)), ("read", (5, 0))]


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def _bf16(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def run_script(n: int, device) -> None:
    cache = R.Int4KVCache(CAP, H, n, device=device)
    held = []                                        # bf16 bits [H, 128] of the tokens held, oldest first
    seed = 900 + n
    for op, arg in SCRIPT:
        if op == "write":
            xb = I.gaussian_bf16(seed, (arg, H, 128), 1.0, 0.02, 12.0)
            seed += 1
            cache.write(_bf16(xb.reshape(arg, H * 128), device))
            held = (held + list(xb))[-CAP:]
        elif op == "evict":
            cache.evict(arg)
            held = held[arg:]
        else:
            first, count = arg
            count = len(held) - first if count is None else count
            y = cache.read(first, None if arg[1] is None else count)
            assert tuple(y.shape) == (count, H * 128)
            if count:
                p, s = O.kv4_encode(np.stack(held[first:first + count]), n)
                want = O.kv4_decode(p, s, n)
                assert np.array_equal(_bits(y).reshape(count, H, 128), want), (op, arg)
        assert cache.size == len(held)


@pytest.fixture
def oracle_codec(monkeypatch):
    """Stand-ins for the two codec calls with the C ABI's argument rules (T <= capacity,
    0 <= slot0 < capacity, slot of token t = (slot0 + t) mod capacity)."""
    calls = []

    def encode(x, codes, scales, n=1, slot0=0, stream=None):
        cap, T = codes.shape[0], x.shape[0]
        assert T <= cap and 0 <= slot0 < cap
        p, s = O.kv4_encode(_bits(x).reshape(T, codes.shape[1], 128), n)
        for t in range(T):
            codes[(slot0 + t) % cap] = torch.from_numpy(p[t])
            scales[(slot0 + t) % cap] = torch.from_numpy(s[t])
        calls.append(("encode", T, slot0))

    def decode(codes, scales, y, n=1, slot0=0, stream=None):
        cap, T = codes.shape[0], y.shape[0]
        assert T <= cap and 0 <= slot0 < cap
        idx = [(slot0 + t) % cap for t in range(T)]
        out = O.kv4_decode(codes.numpy()[idx], scales.numpy()[idx], n)
        y.copy_(_bf16(out.reshape(T, -1), "cpu"))
        calls.append(("decode", T, slot0))

    monkeypatch.setattr(K.B, "rbd_kv4_encode", encode)
    monkeypatch.setattr(K.B, "rbd_kv4_decode", decode)
    return calls


@pytest.mark.parametrize("n", [1, 2, 4])
def test_ring_script_against_the_oracle(oracle_codec, n):
    run_script(n, "cpu")
    assert ("encode", 16, 2) in oracle_codec       # a full-capacity write that wraps the ring
    assert any(c[0] == "decode" and c[1] + c[2] > CAP for c in oracle_codec)   # a read across the wrap


def test_ring_rolling_eviction_slots(oracle_codec):
    cache = R.Int4KVCache(8, 1, 1, device="cpu")
    x = _bf16(I.gaussian_bf16(950, (6, 128)), "cpu")
    cache.write(x)
    cache.write(x[:5])                              # 3 oldest evicted; the write starts at slot 6
    assert (cache.start, cache.size) == (3, 8)
    assert oracle_codec[-1] == ("encode", 5, 6)
    cache.read(2, 4)
    assert oracle_codec[-1] == ("decode", 4, 5)


def test_ring_slices_and_overwrite(oracle_codec):
    n = 2
    cache = R.Int4KVCache(8, 2, n, device="cpu")
    xa = I.gaussian_bf16(960, (6, 2, 128), 1.0, 0.02, 12.0)
    xb = I.gaussian_bf16(961, (5, 2, 128), 1.0, 0.02, 12.0)
    xc = I.gaussian_bf16(962, (3, 2, 128), 1.0, 0.02, 12.0)
    cache[len(cache):] = _bf16(xa.reshape(6, 256), "cpu")
    cache[len(cache):] = _bf16(xb.reshape(5, 256), "cpu")     # rolls: 3 oldest evicted, the ring wraps
    held = list(xa[3:]) + list(xb)
    assert len(cache) == 8 and cache.start == 3
    cache[2:5] = _bf16(xc.reshape(3, 256), "cpu")               # held tokens 2..4 re-encoded in place
    held[2:5] = list(xc)
    assert (len(cache), cache.start) == (8, 3)

    def want(lo, hi):
        p, s = O.kv4_encode(np.stack(held[lo:hi]), n)
        return O.kv4_decode(p, s, n)

    for lo, hi, key in ((0, 8, slice(None)), (1, 7, slice(1, 7)), (5, 8, slice(-3, None)), (4, 6, slice(4, 6))):
        got = cache[key]
        assert np.array_equal(_bits(got).reshape(hi - lo, 2, 128), want(lo, hi)), key
    assert cache[6:2].shape[0] == 0
    with pytest.raises(ValueError):
        cache[::2]
    with pytest.raises(TypeError):
        cache[3]
    with pytest.raises(ValueError):
        cache[0:2] = _bf16(xc.reshape(3, 256), "cpu")
    with pytest.raises(ValueError):
        cache.overwrite(6, _bf16(xc.reshape(3, 256), "cpu"))


def test_ring_argument_errors(oracle_codec):
    cache = R.Int4KVCache(4, 1, 2, device="cpu")
    with pytest.raises(ValueError):
        cache.write(torch.zeros((5, 128), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        cache.write(torch.zeros((2, 256), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        cache.write(torch.zeros((2, 128), dtype=torch.float32))
    cache.write(torch.zeros((3, 128), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        cache.evict(4)
    with pytest.raises(ValueError):
        cache.read(2, 2)
    with pytest.raises(ValueError):
        cache.read(0, 3, out=torch.empty((2, 128), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        cache.write(torch.zeros((1, 128), dtype=torch.bfloat16, device="meta"))      # another device
    for bad in [dict(capacity=0, heads=1), dict(capacity=4, heads=0), dict(capacity=4, heads=1, groups_per_band=3)]:
        with pytest.raises(ValueError):
            R.Int4KVCache(device="cpu", **bad)
    assert not [c for c in oracle_codec if c[1] > 4]


def test_refused_write_leaves_the_ring_unchanged(oracle_codec, monkeypatch):
    # a write that would roll the ring but whose encode is refused (here: the stand-in raises the
    # library's error for any slice of 3 tokens) must not evict anything or move the ring
    cache = R.Int4KVCache(6, 1, 1, device="cpu")
    xb = I.gaussian_bf16(970, (5, 1, 128), 1.0, 0.02, 12.0)
    cache.write(_bf16(xb.reshape(5, 128), "cpu"))
    good = K.B.rbd_kv4_encode

    def refusing(x, codes, scales, n=1, slot0=0, stream=None):
        if x.shape[0] == 3:
            raise K.B.RbdError(3, "rbd_kv4_encode")
        return good(x, codes, scales, n, slot0, stream)

    monkeypatch.setattr(K.B, "rbd_kv4_encode", refusing)
    with pytest.raises(K.B.RbdError):
        cache.write(_bf16(I.gaussian_bf16(971, (3, 128)), "cpu"))
    assert (cache.start, len(cache)) == (0, 5)
    p, s = O.kv4_encode(xb, 1)
    assert np.array_equal(_bits(cache[:]).reshape(5, 1, 128), O.kv4_decode(p, s, 1))
    # an accepted write afterwards rolls as usual
    cache.write(_bf16(I.gaussian_bf16(972, (2, 128)), "cpu"))
    assert (cache.start, len(cache)) == (1, 6)


@pytest.mark.gpu
@pytest.mark.parametrize("n", [1, 2, 4])
def test_gpu_ring_script_against_the_oracle(n):
    run_script(n, "cuda")
    assert R.rbd_check() == 0
