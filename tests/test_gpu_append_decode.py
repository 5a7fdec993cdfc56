"""pa_decode_append (append the step's new tokens, then decode; one kernel on the
tensor-core family) against the oracle's append followed by its decode: outputs
at |err| <= 2e-3 + 2e-3 |ref| (bf16 through the fp32 result, see gpu_util), caches
bit-exact afterwards, error flags for the documented misuse."""
import copy

import numpy as np
import pytest
import torch

from paged_kv_cache_395_b200 import pa, runner, workloads as W

from .gpu_util import assert_close, bits, check_bf16
from .oracle_replay import replay

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_flags():
    pa.pa_get_error_flags(reset=True)
    yield
    assert pa.pa_get_error_flags(reset=True) == 0


def last_token_step(w, slot_override=None, extra=None):
    """The random case w with every sequence's last token taken out of the setup
    append and appended by the step instead (row b of the step's append is
    sequence b's token; an empty sequence gets slot -1).  slot_override {b: slot}
    replaces slots; extra [(b, slot)] gives an empty sequence b a token."""
    (setup,) = w.setup
    dec = w.steps[0][0]
    B = len(dec.seq_lens)
    H, d = w.num_kv_heads, w.head_dim
    keep, off = [], 0
    kn = np.zeros((B, H, d), dtype=setup.k.dtype)
    vn = np.zeros_like(kn)
    sn = np.full(B, -1, dtype=np.int64)
    for b, L in enumerate(dec.seq_lens):
        L = int(L)
        if L > 0:
            keep.extend(range(off, off + L - 1))
            kn[b], vn[b], sn[b] = setup.k[off + L - 1], setup.v[off + L - 1], setup.slot_mapping[off + L - 1]
        off += L
    for b, s in (extra or []):
        kn[b], vn[b], sn[b] = setup.k[0], setup.v[1], s
    for b, s in (slot_override or {}).items():
        sn[b] = s
    keep = np.array(keep, dtype=np.int64)
    w.setup = [W.Reshape(setup.k[keep], setup.v[keep], setup.slot_mapping[keep])]
    w.steps = [[W.Reshape(kn, vn, sn), dec]]
    return w


def free_block(w):
    """A physical block no sequence of w's decode reads."""
    dec = w.steps[0][-1]
    used = set()
    for b, L in enumerate(dec.seq_lens):
        used |= {int(x) for x in dec.block_tables[b, :(int(L) + 15) // 16]}
    return min(set(range(w.num_blocks)) - used)


def run_fused(w, part, expect_fused=True, algo=pa.PA_ALGO_AUTO):
    """Setup, then the step's append and decode as one pa_decode_append call."""
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    (_, k, v, s), dec = dw.steps[0]
    _, q, bt, sl, mx, out = dec
    assert pa.pa_decode_append_fused(q, k, v, dw.kc, bt, mx, part, algo) == expect_fused
    ws = dw.workspace_for(dec, part, False, algo) if part != 0 else None
    pa.pa_decode_append(out, q, k, v, s, dw.kc, dw.vc, bt, sl, w.scale, mx, part, ws, algo)
    torch.cuda.synchronize()
    return out, dw


def seq_rows(w, seqs):
    return [(b, h) for b in seqs for h in range(w.num_q_heads)]


CASES = {
    "g4_d128_f16": dict(lens=[1, 16, 17, 100, 513, 1000], num_q_heads=32, num_kv_heads=8, head_dim=128,
                        dtype="float16"),
    "g8_d64_bf16": dict(lens=[33, 300, 2, 129], num_q_heads=16, num_kv_heads=2, head_dim=64, dtype="bfloat16"),
    "g1_d256_f16": dict(lens=[15, 64, 257], num_q_heads=4, num_kv_heads=4, head_dim=256, dtype="float16"),
    "g2_d128_bf16": dict(lens=[31, 48, 7, 600], num_q_heads=8, num_kv_heads=4, head_dim=128, dtype="bfloat16"),
    "g16_rows_f16": dict(lens=[5, 77, 256], num_q_heads=32, num_kv_heads=2, head_dim=128, dtype="float16"),
}


@pytest.mark.parametrize("part", [0, 16, -1])
@pytest.mark.parametrize("case", sorted(CASES))
def test_fused_append_then_decode(case, part):
    """One new token per sequence at its last position (a partial or a just-started
    block, rows cut by chunks or whole): output and both caches as the oracle's
    append then decode."""
    c = CASES[case]
    w = last_token_step(W.random_case(seed=sorted(CASES).index(case) + 300, **c))
    ref, kc, vc = replay(w)
    fused = not (case == "g16_rows_f16" and part != 0)  # 16 heads per KV head split: the cooperative mode
    got, dw = run_fused(w, part, fused)
    if w.dtype == "bfloat16":
        # the fp32 result of the same decode, over the cache the call left
        f32 = torch.empty(got.shape, dtype=torch.float32, device=got.device)
        _, q, bt, sl, mx, _ = dw.steps[0][1]
        ws = dw.workspace_for(dw.steps[0][1], part) if part != 0 else None
        pa.pa_decode(f32, q, dw.kc, dw.vc, bt, sl, w.scale, mx, partition_size=part, workspace=ws)
        torch.cuda.synchronize()
        check_bf16(got, f32, ref[0], case)
    else:
        assert_close(got, ref[0], w.dtype, case)
    assert np.array_equal(bits(dw.kc), kc.view(np.uint8))
    assert np.array_equal(bits(dw.vc), vc.view(np.uint8))


@pytest.mark.parametrize("part", [0, -1])
def test_fused_append_edge_slots(part):
    """Sequence 1 has no new token (slot -1: its last position keeps what the cache
    held); empty sequence 3 gets a token in a free block (written, output zero);
    empty sequence 4's token is outside the pool (PA_EFLAG_BAD_SLOT, skipped)."""
    lens = [40, 17, 5, 0, 0, 64]
    full = W.random_case(lens, num_q_heads=8, num_kv_heads=2, head_dim=128, seed=11, extra_blocks=4)
    fb = free_block(full)
    w = last_token_step(W.random_case(lens, num_q_heads=8, num_kv_heads=2, head_dim=128, seed=11,
                                      extra_blocks=4),
                        slot_override={1: -1}, extra=[(3, fb * 16 + 3), (4, full.num_blocks * 16 + 5)])
    # sequence 1's last token stays in the cache from the setup
    (setup,), fs = w.setup, full.setup[0]
    i1 = lens[0] + lens[1] - 1
    w.setup = [W.Reshape(np.concatenate([setup.k, fs.k[i1:i1 + 1]]), np.concatenate([setup.v, fs.v[i1:i1 + 1]]),
                         np.concatenate([setup.slot_mapping, fs.slot_mapping[i1:i1 + 1]]))]
    # the oracle's append is given the skip the library makes for the slot outside the pool
    rw = copy.deepcopy(w)
    rw.steps[0][0].slot_mapping[4] = -1
    ref, kc, vc = replay(rw)
    got, dw = run_fused(w, part)
    assert pa.pa_get_error_flags(reset=True) == pa.PA_EFLAG_BAD_SLOT
    assert_close(got, ref[0], "float16", "edge slots")
    assert not np.any(ref[0][3:5])
    assert np.array_equal(bits(dw.kc), kc.view(np.uint8))
    assert np.array_equal(bits(dw.vc), vc.view(np.uint8))


def test_fused_append_misplaced_slot_is_flagged():
    """A new token whose slot is not its sequence's last position: PA_EFLAG_APPEND_SLOT,
    the token still lands in its slot (caches as the oracle's append), the other
    sequences' outputs are unaffected."""
    lens = [40, 33, 70]
    base = W.random_case(lens, num_q_heads=8, num_kv_heads=2, head_dim=128, seed=12, extra_blocks=2)
    w = last_token_step(base, slot_override={1: free_block(base) * 16 + 9})
    ref, kc, vc = replay(w)
    got, dw = run_fused(w, -1)
    assert pa.pa_get_error_flags(reset=True) == pa.PA_EFLAG_APPEND_SLOT
    assert_close(got, ref[0], "float16", "misplaced slot", rows=seq_rows(w, [0, 2]))
    assert np.array_equal(bits(dw.kc), kc.view(np.uint8))
    assert np.array_equal(bits(dw.vc), vc.view(np.uint8))


@pytest.mark.parametrize("case", ["fp32_simt", "mqa_coop"])
def test_unfused_calls_are_the_two_kernels(case):
    """Where the library does not fuse (fp32 caches; the cooperative mode of 32 heads
    per KV head), pa_decode_append is the append then the decode."""
    if case == "fp32_simt":
        base = W.random_case([3, 45, 20], num_q_heads=8, num_kv_heads=1, head_dim=64, dtype="float32", seed=13)
        part = 16
    else:
        base = W.random_case([7, 129, 640], num_q_heads=32, num_kv_heads=1, head_dim=128, seed=14)
        part = -1
    w = last_token_step(base)
    ref, kc, vc = replay(w)
    got, dw = run_fused(w, part, expect_fused=False)
    assert_close(got, ref[0], w.dtype, case)
    assert np.array_equal(bits(dw.kc), kc.view(np.uint8))
    assert np.array_equal(bits(dw.vc), vc.view(np.uint8))


@pytest.mark.slow
def test_ragged_trace_fused_back_to_back():
    """The benchmark's issue pattern: all 128 ragged steps on one stream, admitted
    prompts appended with PA_APPEND_OVERLAP_PREVIOUS, new tokens and decode as one
    pa_decode_append (flagged PA_DECODE_INPUTS_READY).  Sampled steps against the
    oracle, caches bit-exact at the end."""
    w = W.ragged()
    sample = {0, 3, 64, 127}
    ref, kc, vc = replay(w, want=lambda s: s in sample)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    calls = runner.StepCalls(dw, -1, False, pa.PA_ALGO_AUTO, stream, flags=pa.PA_DECODE_INPUTS_READY,
                             fused=True, prompt_flags=pa.PA_APPEND_OVERLAP_PREVIOUS)
    assert calls.fused_steps == len(w.steps)
    with torch.cuda.stream(stream):
        for i in range(len(w.steps)):
            calls.run(i)
    torch.cuda.synchronize()
    for i in sorted(sample):
        assert_close(dw.steps[i][-1][-1], ref[i], "float16", f"ragged step {i}")
    assert np.array_equal(bits(dw.kc), kc.view(np.uint8))
    assert np.array_equal(bits(dw.vc), vc.view(np.uint8))
