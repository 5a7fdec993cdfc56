"""Bit-exact GPU cache operations against the oracle: append scatter,
copy-on-write block copy, int8 quantiser, and the device error word."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_395_b200 import pa, runner, workloads as W

from .gpu_util import bits, np_bits
from .oracle_replay import make_pool, replay

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_flags():
    pa.pa_get_error_flags(reset=True)
    yield


@pytest.mark.parametrize("make", [W.tiny, lambda: W.random_case([3, 16, 33, 1], dtype="bfloat16"),
                                  lambda: W.random_case([40, 17], head_dim=128, num_kv_heads=4,
                                                        num_q_heads=8, dtype="float16")],
                         ids=["tiny_fp32", "bf16", "fp16_d128"])
def test_reshape_and_cache_bit_exact(make):
    w = make()
    _, kc, vc = replay(w, want=lambda s: False)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    for i in range(len(w.steps)):
        dw.run_step(i, decode=False)
    torch.cuda.synchronize()
    # written slots equal the inputs, unwritten ones keep their NaN fill
    assert np.array_equal(bits(dw.kc), np_bits(kc))
    assert np.array_equal(bits(dw.vc), np_bits(vc))
    assert pa.pa_get_error_flags() == 0


def test_reshape_strided_padding_and_unaligned():
    """Token stride larger than the row (k, v as views of a fused buffer),
    padding slots (-1), and 2-byte-aligned rows take the narrow-vector path."""
    dev = "cuda"
    T, H, d, N = 37, 3, 64, 12
    rng = np.random.default_rng(3)
    fused = torch.from_numpy(rng.standard_normal((T, 3 * H * d + 1)).astype(np.float16)).to(dev)
    k = fused[:, 1:1 + H * d].view(T, H, d)  # 2-byte offset: rows not 16-byte aligned
    v = fused[:, 1 + H * d:1 + 2 * H * d].view(T, H, d)
    slots = rng.choice(N * 16, size=T, replace=False).astype(np.int64)
    slots[[0, 5, 36]] = -1
    kc = torch.full((N, H, 16, d), float("nan"), dtype=torch.float16, device=dev)
    vc = kc.clone()
    pa.pa_reshape_and_cache(k, v, kc, vc, torch.from_numpy(slots).to(dev))
    ek = np.full((N, H, 16, d), np.nan, dtype=np.float16)
    ev = ek.copy()
    oracle.reshape_and_cache(k.cpu().numpy(), v.cpu().numpy(), ek, ev, slots)
    assert np.array_equal(bits(kc), np_bits(ek)) and np.array_equal(bits(vc), np_bits(ev))


def _host_rows(t):
    """Device tensor -> (numpy array, oracle dtype code); bf16 as uint16 bits."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16), oracle.BF16
    return t.cpu().numpy(), None


@pytest.mark.parametrize("dtype,d", [(torch.float16, 128), (torch.bfloat16, 64), (torch.float32, 128)])
def test_append_int8_bit_exact(dtype, d):
    """Single tokens appended into a quantised int8 pool, in distinct blocks: tokens
    that fit a tile's scale and tokens that raise it (re-rounding the tile), an
    empty tile, padding and an out-of-pool slot.  Codes and scales bit-exact with
    the oracle's rule."""
    dev = "cuda"
    N, H = 24, 4
    rng = np.random.default_rng(21)
    src = torch.from_numpy((rng.standard_normal((N, H, 16, d)) * 2).astype(np.float32)).to(dev).to(dtype)
    kc = torch.empty((N, H, 16, d), dtype=torch.int8, device=dev)
    vc = torch.empty_like(kc)
    ks = torch.empty((N, H), dtype=torch.float32, device=dev)
    vs = torch.empty_like(ks)
    pa.pa_quantize_int8(src, kc, ks)
    pa.pa_quantize_int8(src.flip(0).contiguous(), vc, vs)
    kc[5].zero_(); ks[5].zero_()  # an empty tile
    T = 14
    blocks = rng.choice([b for b in range(N) if b != 5], size=T, replace=False)  # one token per block
    slots = blocks.astype(np.int64) * 16 + rng.integers(0, 16, size=T)
    slots[3] = -1
    slots[8] = N * 16 + 7  # outside the pool
    slots[0] = 5 * 16 + 9  # into the empty tile
    mag = np.where(np.arange(T) % 2 == 0, 0.2, 12.0)[:, None, None]  # fit, raise
    k = torch.from_numpy((rng.standard_normal((T, H, d)) * mag).astype(np.float32)).to(dev).to(dtype)
    v = torch.from_numpy((rng.standard_normal((T, H, d)) * mag[::-1]).astype(np.float32)).to(dev).to(dtype)
    torch.cuda.synchronize()
    ekc, evc = kc.cpu().numpy(), vc.cpu().numpy()
    eks, evs = ks.cpu().numpy(), vs.cpu().numpy()
    ks0 = eks.copy()
    kh, code = _host_rows(k)
    vh, _ = _host_rows(v)
    oracle.append_int8(kh, vh, ekc, evc, eks, evs, slots, code=code)
    pa.pa_append_int8(k, v, kc, vc, ks, vs, torch.from_numpy(slots).to(dev))
    torch.cuda.synchronize()
    assert pa.pa_get_error_flags(reset=True) == pa.PA_EFLAG_BAD_SLOT
    assert np.array_equal(ks.cpu().numpy().view(np.uint32), eks.view(np.uint32))
    assert np.array_equal(vs.cpu().numpy().view(np.uint32), evs.view(np.uint32))
    assert np.array_equal(kc.cpu().numpy(), ekc) and np.array_equal(vc.cpu().numpy(), evc)
    # the case mix happened: some tiles' scales were raised, the others kept theirs
    after = ks.cpu().numpy()
    assert (after > ks0).any() and (after == ks0).any()


def test_append_int8_token_by_token_into_one_block():
    """Sixteen calls, each appending the next token of one block (the decode-step
    pattern), on fp16 tokens of growing size: every call may raise the scale and
    re-round what is there.  Bit-exact with the oracle after every call."""
    dev = "cuda"
    H, d, N = 2, 128, 3
    rng = np.random.default_rng(22)
    kc = torch.zeros((N, H, 16, d), dtype=torch.int8, device=dev)
    vc = torch.zeros_like(kc)
    ks = torch.zeros((N, H), dtype=torch.float32, device=dev)
    vs = torch.zeros_like(ks)
    ekc, evc = kc.cpu().numpy(), vc.cpu().numpy()
    eks, evs = ks.cpu().numpy(), vs.cpu().numpy()
    for o in range(16):
        k = (rng.standard_normal((1, H, d)) * (0.5 + o)).astype(np.float16)
        v = (rng.standard_normal((1, H, d)) * (16 - o)).astype(np.float16)
        slot = np.array([1 * 16 + o], dtype=np.int64)
        oracle.append_int8(k, v, ekc, evc, eks, evs, slot)
        pa.pa_append_int8(torch.from_numpy(k).to(dev), torch.from_numpy(v).to(dev), kc, vc, ks, vs,
                          torch.from_numpy(slot).to(dev))
        torch.cuda.synchronize()
        assert np.array_equal(kc.cpu().numpy(), ekc) and np.array_equal(vc.cpu().numpy(), evc), f"slot {o}"
        assert np.array_equal(ks.cpu().numpy(), eks) and np.array_equal(vs.cpu().numpy(), evs), f"slot {o}"


def test_reshape_bad_slot_sets_flag_and_skips():
    dev = "cuda"
    k = torch.ones((2, 1, 64), dtype=torch.float16, device=dev)
    kc = torch.zeros((2, 1, 16, 64), dtype=torch.float16, device=dev)
    vc = kc.clone()
    slots = torch.tensor([5, 32], dtype=torch.int64, device=dev)  # 32 = 2 blocks * 16: outside
    pa.pa_reshape_and_cache(k, k, kc, vc, slots)
    assert pa.pa_get_error_flags() == pa.PA_EFLAG_BAD_SLOT
    assert kc[0, 0, 5].eq(1).all() and kc.sum().item() == 64


def test_block_copy_mha_prefix_bit_exact():
    w = W.mha_prefix()
    _, kc, vc = replay(w, want=lambda s: False)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    dw.run_step(0, decode=False)
    torch.cuda.synchronize()
    assert np.array_equal(bits(dw.kc), np_bits(kc))
    assert np.array_equal(bits(dw.vc), np_bits(vc))


def test_block_copy_scales_and_untouched():
    dev = "cuda"
    rng = np.random.default_rng(8)
    N, H, d = 9, 2, 128
    kc = rng.integers(-127, 128, size=(N, H, 16, d)).astype(np.int8)
    vc = rng.integers(-127, 128, size=(N, H, 16, d)).astype(np.int8)
    ks = rng.random((N, H)).astype(np.float32)
    vs = rng.random((N, H)).astype(np.float32)
    pairs = np.array([[2, 7], [2, 8], [4, 0]], dtype=np.int64)
    g = [torch.from_numpy(x.copy()).to(dev) for x in (kc, vc, ks, vs)]
    pa.pa_block_copy(g[0], g[1], torch.from_numpy(pairs).to(dev), g[2], g[3])
    oracle.block_copy(kc, vc, pairs, ks, vs)
    for t, e in zip(g, (kc, vc, ks, vs)):
        assert np.array_equal(bits(t), np_bits(e))


def test_block_copy_bad_pair_flag():
    dev = "cuda"
    kc = torch.zeros((4, 1, 16, 64), dtype=torch.float16, device=dev)
    vc = kc.clone()
    pa.pa_block_copy(kc, vc, torch.tensor([[0, 4], [-1, 2]], dtype=torch.int64, device=dev))
    assert pa.pa_get_error_flags() == pa.PA_EFLAG_BAD_PAIR
    assert kc.abs().sum().item() == 0


@pytest.mark.parametrize("dtype", ["float16", "bfloat16", "float32"])
def test_quantize_int8_bit_exact(dtype):
    dev = "cuda"
    rng = np.random.default_rng(12)
    N, H, d = 64, 4, 128
    x = rng.standard_normal((N, H, 16, d)) * rng.uniform(0.01, 30, size=(N, H, 1, 1))
    x[3, 1] = 0.0                                   # all-zero tile
    x[5, 2].reshape(-1)[:8] = [127, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5]  # absmax 127: s = 1
    x[5, 2].reshape(-1)[8:] = 0
    if dtype == "bfloat16":
        t = torch.from_numpy(x).to(torch.bfloat16)
        host = t.view(torch.int16).numpy().view(np.uint16)
        dsrc = t.to(dev)
        code = oracle.BF16
    else:
        host = x.astype(dtype)
        dsrc = torch.from_numpy(host).to(dev)
        code = None
    q_ref, s_ref = oracle.quantize_int8(host, code=code)
    q = torch.empty((N, H, 16, d), dtype=torch.int8, device=dev)
    s = torch.empty((N, H), dtype=torch.float32, device=dev)
    pa.pa_quantize_int8(dsrc, q, s)
    assert np.array_equal(bits(q), np_bits(q_ref))
    assert np.array_equal(bits(s), np_bits(s_ref))


def test_quantize_long_config_bit_exact():
    """The int8 pool of the long-context workload, GPU quantiser vs oracle."""
    w = W.long(batch=2, seq_len=2048)
    _, kc, vc = replay(w, want=lambda s: False, fill_nan=False)
    dw = runner.DeviceWorkload(w, fill_nan=False)
    dw.run_setup()
    dw.quantize_int8()
    for dev_q, dev_s, host in ((dw.kc8, dw.k_scales, kc), (dw.vc8, dw.v_scales, vc)):
        q_ref, s_ref = oracle.quantize_int8(host)
        assert np.array_equal(bits(dev_q), np_bits(q_ref))
        assert np.array_equal(bits(dev_s), np_bits(s_ref))


@pytest.mark.parametrize("dtype", ["float16", "bfloat16", "float32"])
def test_quantize_int4_bit_exact(dtype):
    """The 4-bit quantiser byte for byte (and its scales bit for bit) against the
    oracle: random tiles of very different ranges, an all-zero tile, and a tile
    with absmax 7 (s = 1) holding round-half-even cases."""
    dev = "cuda"
    rng = np.random.default_rng(14)
    N, H, d = 64, 4, 128
    x = rng.standard_normal((N, H, 16, d)) * rng.uniform(0.01, 30, size=(N, H, 1, 1))
    x[3, 1] = 0.0
    x[5, 2] = 0.0
    x[5, 2].reshape(-1)[:10] = [7, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 6.5, -6.5, -7]
    if dtype == "bfloat16":
        t = torch.from_numpy(x).to(torch.bfloat16)
        host = t.view(torch.int16).numpy().view(np.uint16)
        dsrc = t.to(dev)
        code = oracle.BF16
    else:
        host = x.astype(dtype)
        dsrc = torch.from_numpy(host).to(dev)
        code = None
    q_ref, s_ref = oracle.quantize_int4(host, code=code)
    q = torch.empty((N, H, 16, d // 2), dtype=torch.uint8, device=dev)
    s = torch.empty((N, H), dtype=torch.float32, device=dev)
    pa.pa_quantize_int4(dsrc, q, s)
    assert np.array_equal(bits(q), np_bits(q_ref))
    assert np.array_equal(bits(s), np_bits(s_ref))


def test_block_copy_int4():
    """Copy-on-write of packed 4-bit blocks (rows of d / 2 bytes) with their scales."""
    dev = "cuda"
    rng = np.random.default_rng(9)
    N, H, d = 9, 2, 128
    kc = rng.integers(0, 256, size=(N, H, 16, d // 2)).astype(np.uint8)
    vc = rng.integers(0, 256, size=(N, H, 16, d // 2)).astype(np.uint8)
    ks = rng.random((N, H)).astype(np.float32)
    vs = rng.random((N, H)).astype(np.float32)
    pairs = np.array([[1, 6], [3, 0]], dtype=np.int64)
    g = [torch.from_numpy(x.copy()).to(dev) for x in (kc, vc, ks, vs)]
    pa.pa_block_copy(g[0], g[1], torch.from_numpy(pairs).to(dev), g[2], g[3])
    oracle.block_copy(kc, vc, pairs, ks, vs)
    for t, e in zip(g, (kc, vc, ks, vs)):
        assert np.array_equal(bits(t), np_bits(e))
