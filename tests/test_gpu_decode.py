"""GPU paged decode against the oracle, element by element, plus invariants.

Every case runs through the C ABI (paged_kv_cache_395_b200.pa).  Tolerance:
|err| <= 2e-3 + 2e-3 |ref| for fp16/bf16 outputs (fp32 accumulation), and
1e-5 + 1e-5 |ref| for the fp32 case; int8 caches are compared with the oracle
dequantising the same int8 values and scales in fp64.  A bf16 case checks that
bound on the fp32 result before the output's rounding (the same call with a
float32 out) and that the bf16 output is that result rounded to nearest even
(gpu_util.check_bf16).
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_395_b200 import pa, runner, workloads as W

from .gpu_util import assert_close, bits, check_bf16
from .oracle_replay import replay

pytestmark = pytest.mark.gpu

ALGOS = [pa.PA_ALGO_SIMT, pa.PA_ALGO_TENSOR, pa.PA_ALGO_AUTO]


def algo_ok(algo, dtype):
    """The tensor-core family covers fp16/bf16 q with a cache of the same dtype."""
    return algo != pa.PA_ALGO_TENSOR or dtype in ("float16", "bfloat16")
PARTS = [0, 16, 32, 256, -1]


@pytest.fixture(autouse=True)
def _clear_flags():
    pa.pa_get_error_flags(reset=True)
    yield
    assert pa.pa_get_error_flags(reset=True) == 0


def check(got, ref, dtype, what, dw, part, algo, int8=False, rows=None):
    """The oracle comparison of step 0's output; a bf16 output is checked with its
    fp32 result, which a second decode of the same step (into a float32 out) gives."""
    if dtype != "bfloat16":
        return assert_close(got, ref, dtype, what, rows=rows)
    f32 = dw.decode_again(0, part, int8=int8, algo=algo, out_f32=True)
    torch.cuda.synchronize()
    check_bf16(got, f32, ref, what, rows=rows)


def run_gpu(w, partition_size=0, algo=pa.PA_ALGO_AUTO, int8=False, dw=None):
    dw = dw or runner.DeviceWorkload(w)
    dw.run_setup()
    if int8:
        dw.quantize_int8()
    outs = {}
    for i in range(len(w.steps)):
        o = dw.run_step(i, partition_size, int8=int8, algo=algo)
        outs[i] = o.clone()
    torch.cuda.synchronize()
    return outs, dw


@pytest.mark.parametrize("algo", [pa.PA_ALGO_SIMT, pa.PA_ALGO_AUTO])
@pytest.mark.parametrize("part", [0, 16, -1])
def test_tiny_fp32(algo, part):
    w = W.tiny()
    ref, _, _ = replay(w)
    got, _ = run_gpu(w, part, algo)
    assert_close(got[0], ref[0], "float32", "tiny")


CASES = {
    # lengths hit 1, a full block, block + 1, a ragged tail, several partitions
    "g4_d128_f16": dict(lens=[1, 16, 17, 100, 513, 1000], num_q_heads=32, num_kv_heads=8,
                        head_dim=128, dtype="float16"),
    "g8_d128_bf16": dict(lens=[33, 300, 2, 129], num_q_heads=16, num_kv_heads=2, head_dim=128,
                         dtype="bfloat16"),
    "g1_d128_f16": dict(lens=[15, 64, 257], num_q_heads=4, num_kv_heads=4, head_dim=128,
                        dtype="float16"),
    "g2_d64_f16": dict(lens=[31, 48, 7, 600], num_q_heads=8, num_kv_heads=4, head_dim=64,
                       dtype="float16"),
    "g4_d64_bf16": dict(lens=[5, 77, 256], num_q_heads=8, num_kv_heads=2, head_dim=64,
                        dtype="bfloat16"),
    "g8_d64_f32": dict(lens=[3, 45], num_q_heads=8, num_kv_heads=1, head_dim=64, dtype="float32"),
    "sharp_softmax": dict(lens=[200, 37], num_q_heads=8, num_kv_heads=2, head_dim=128,
                          dtype="float16", q_scale=6.0),
}


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("part", PARTS)
@pytest.mark.parametrize("case", sorted(CASES))
def test_random_cases(case, part, algo):
    if not algo_ok(algo, CASES[case]["dtype"]):
        pytest.skip("fp32 has no tensor-core path")
    w = W.random_case(seed=sorted(CASES).index(case) + 100, **CASES[case])
    ref, _, _ = replay(w)
    got, dw = run_gpu(w, part, algo)
    check(got[0], ref[0], w.dtype, case, dw, part, algo)


@pytest.mark.parametrize("algo", ALGOS)
@pytest.mark.parametrize("part", [0, 32, -1])
@pytest.mark.parametrize("qdt", ["float16", "bfloat16"])
def test_int8_random(qdt, part, algo):
    if algo == pa.PA_ALGO_TENSOR and qdt != "float16":
        pytest.skip("the tensor-core family reads int8 caches with fp16 q")
    w = W.random_case([1, 17, 96, 400], num_q_heads=16, num_kv_heads=4, head_dim=128, dtype=qdt,
                      seed=4)
    dw = runner.DeviceWorkload(w)
    got, dw = run_gpu(w, part, algo, int8=True, dw=dw)
    # the oracle dequantises the very same int8 values and scales
    kc8, vc8 = dw.kc8.cpu().numpy(), dw.vc8.cpu().numpy()
    ks, vs = dw.k_scales.cpu().numpy(), dw.v_scales.cpu().numpy()
    op = w.steps[0][0]
    ref = oracle.decode(op.q, kc8, vc8, op.block_tables, op.seq_lens, w.scale, ks, vs)
    check(got[0], ref, qdt, "int8", dw, part, algo, int8=True)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 4), (32, 8)])
@pytest.mark.parametrize("part", [0, 16, -1])
def test_int8_tensor_group_sizes(hq, hkv, part):
    """int8 caches on the tensor-core family for every group size, ragged tails,
    one-pass, one-block and library-picked partitions, against the oracle
    dequantising the same int8 values."""
    w = W.random_case([1, 15, 16, 33, 250, 777], num_q_heads=hq, num_kv_heads=hkv, head_dim=128,
                      dtype="float16", seed=hq + hkv)
    dw = runner.DeviceWorkload(w)
    got, dw = run_gpu(w, part, pa.PA_ALGO_TENSOR, int8=True, dw=dw)
    kc8, vc8 = dw.kc8.cpu().numpy(), dw.vc8.cpu().numpy()
    ks, vs = dw.k_scales.cpu().numpy(), dw.v_scales.cpu().numpy()
    op = w.steps[0][0]
    ref = oracle.decode(op.q, kc8, vc8, op.block_tables, op.seq_lens, w.scale, ks, vs)
    assert_close(got[0], ref, "float16", f"int8 tensor G={hq // hkv} part={part}")


def test_tensor_path_rejects_unsupported():
    w = W.random_case([20], num_q_heads=4, num_kv_heads=2, head_dim=64, dtype="float32")
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    _, q, bt, sl, mx, out = dw.steps[0][-1]
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(out, q, dw.kc, dw.vc, bt, sl, w.scale, mx, algo=pa.PA_ALGO_TENSOR)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED


@pytest.mark.parametrize("algo", [pa.PA_ALGO_SIMT, pa.PA_ALGO_TENSOR])
def test_long_one_pass_and_many_partitions(algo):
    """One pass over 40 blocks (more than one 32-entry table chunk) and a split
    into 70 partitions, both against the oracle."""
    w = W.random_case([640, 1120, 33], num_q_heads=16, num_kv_heads=4, head_dim=128, seed=12)
    ref, _, _ = replay(w)
    for part in (0, 16, 512):
        got, _ = run_gpu(w, part, algo)
        assert_close(got[0], ref[0], "float16", f"part={part}")


def test_workspace_reused_across_calls():
    """The workspace needs no initialisation: filled with 0xff bytes (NaN floats)
    before every call, it still gives the oracle's result."""
    w = W.random_case([300, 77, 513], num_q_heads=32, num_kv_heads=8, head_dim=128, seed=13)
    ref, _, _ = replay(w)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    op = dw.steps[0][-1]
    ws = dw.workspace_for(op, 32)
    _, q, bt, sl, mx, out = op
    for _ in range(5):
        out.zero_()
        ws.fill_(0xFF)
        pa.pa_decode(out, q, dw.kc, dw.vc, bt, sl, w.scale, mx, partition_size=32, workspace=ws,
                     algo=pa.PA_ALGO_TENSOR)
        assert_close(out, ref[0], "float16", "reuse")


def test_zero_length_and_empty_batch():
    w = W.random_case([0, 5, 0, 40], num_q_heads=8, num_kv_heads=2, head_dim=64, dtype="float16")
    ref, _, _ = replay(w)
    for part in (0, 16):
        got, _ = run_gpu(w, part)
        assert_close(got[0], ref[0], "float16", "zero length")
        assert torch.count_nonzero(got[0][0]) == 0 and torch.count_nonzero(got[0][2]) == 0
    # B = 0 is a no-op
    q = torch.empty((0, 8, 64), dtype=torch.float16, device="cuda")
    kc = torch.zeros((4, 2, 16, 64), dtype=torch.float16, device="cuda")
    bt = torch.zeros((0, 1), dtype=torch.int32, device="cuda")
    sl = torch.zeros((0,), dtype=torch.int32, device="cuda")
    pa.pa_decode(torch.empty_like(q), q, kc, kc, bt, sl, 0.125, 0)


def test_permutation_invariance_bitwise():
    """Moving the physical blocks leaves the GPU output bit-identical."""
    w = W.random_case([70, 300, 17], num_q_heads=32, num_kv_heads=8, head_dim=128, seed=9)
    for part in (0, 32):
        got, dw = run_gpu(w, part)
        sigma = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(1)).cuda()
        kc2 = torch.empty_like(dw.kc)
        vc2 = torch.empty_like(dw.vc)
        kc2[sigma] = dw.kc
        vc2[sigma] = dw.vc
        _, q, bt, sl, mx, out = dw.steps[0][-1]
        bt2 = bt.clone()
        valid = bt2 >= 0
        bt2[valid] = sigma[bt2[valid].long()].int()
        out2 = torch.empty_like(out)
        ws = dw.workspace_for(dw.steps[0][-1], part)
        pa.pa_decode(out2, q, kc2, vc2, bt2, sl, w.scale, mx, partition_size=part, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(bits(out2), bits(got[0])), f"part={part}"


def test_deterministic_and_split_matches_single():
    w = W.random_case([900, 1500, 64], num_q_heads=32, num_kv_heads=8, head_dim=128, seed=10)
    a, _ = run_gpu(w, 0)
    b, _ = run_gpu(w, 0)
    assert np.array_equal(bits(a[0]), bits(b[0]))
    c, _ = run_gpu(w, 128)
    d, _ = run_gpu(w, 128)
    assert np.array_equal(bits(c[0]), bits(d[0]))
    ref, _, _ = replay(w)
    assert_close(c[0], ref[0], "float16", "split")
    assert_close(a[0], ref[0], "float16", "single")


def test_bad_block_id_flagged():
    """A table entry outside the pool is skipped by the kernel's own bounds
    check (no memory access) and reported in the error word."""
    w = W.random_case([40, 20], num_q_heads=8, num_kv_heads=2, head_dim=64, seed=2)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    _, q, bt, sl, mx, out = dw.steps[0][-1]
    bt[1, 0] = w.num_blocks + 5
    pa.pa_decode(out, q, dw.kc, dw.vc, bt, sl, w.scale, mx)
    assert pa.pa_get_error_flags(reset=True) == pa.PA_EFLAG_BAD_BLOCK


@pytest.mark.parametrize("kind", ["float16", "int8", "int4"])
@pytest.mark.parametrize("part", [0, -1])
def test_skipped_block_leaves_the_rest_exact(kind, part):
    """A block id outside the pool inside a sequence: the kernel skips that block's
    16 tokens and attends over the others.  Attention has no token order, so the
    expected output is the oracle's on the table row without that block and the
    length 16 shorter; the other sequences are untouched.  Covers the blocks the
    quantised kernels consume two at a time (a skipped block beside a good one)."""
    w = W.random_case([100, 200, 37], num_q_heads=16, num_kv_heads=4, head_dim=128, dtype="float16",
                      seed=71)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    quant = kind != "float16"
    if kind == "int8":
        dw.quantize_int8()
    elif kind == "int4":
        dw.quantize_int4()
    _, q, bt, sl, mx, out = dw.steps[0][-1]
    op = w.steps[0][0]
    for skip in (2, 5):  # the first or the second block of a pair
        bt_bad = bt.clone()
        bt_bad[1, skip] = w.num_blocks + 5
        kc, vc = (dw.kc8, dw.vc8) if quant else (dw.kc, dw.vc)
        ks, vs = (dw.k_scales, dw.v_scales) if quant else (None, None)
        ws = torch.zeros(pa.pa_decode_workspace_size(q, kc, bt_bad, mx, part, ks, vs, pa.PA_ALGO_TENSOR),
                         dtype=torch.uint8, device=q.device)
        pa.pa_decode(out, q, kc, vc, bt_bad, sl, w.scale, mx, ks, vs, part, ws, pa.PA_ALGO_TENSOR)
        torch.cuda.synchronize()
        assert pa.pa_get_error_flags(reset=True) == pa.PA_EFLAG_BAD_BLOCK
        tables = op.block_tables.copy()
        row = [b for j, b in enumerate(tables[1]) if j != skip] + [tables[1][-1]]
        tables[1] = np.array(row, dtype=tables.dtype)
        lens = op.seq_lens.copy()
        lens[1] -= 16
        if quant:
            ref = oracle.decode(op.q, dw.kc8.cpu().numpy(), dw.vc8.cpu().numpy(), tables, lens, w.scale,
                                dw.k_scales.cpu().numpy(), dw.v_scales.cpu().numpy())
        else:
            ref = oracle.decode(op.q, dw.kc.cpu().numpy(), dw.vc.cpu().numpy(), tables, lens, w.scale)
        assert_close(out, ref, "float16", f"{kind} part={part} skip={skip}")


# -- the study's workloads at full size ---------------------------------------------------
def test_gqa_b8_full():
    w = W.gqa_b8()
    ref, _, _ = replay(w)
    for part in (0, -1, 128):
        got, _ = run_gpu(w, part)
        assert_close(got[0], ref[0], "float16", f"gqa_b8 part={part}")


@pytest.mark.slow
def test_long_fp16_and_int8_full():
    w = W.long()
    ref, kc, vc = replay(w, fill_nan=False)
    got, dw = run_gpu(w, 512)
    assert_close(got[0], ref[0], "float16", "long fp16")
    got8, dw = run_gpu(w, 512, int8=True, dw=runner.DeviceWorkload(w, fill_nan=False))
    kc8, ks = oracle.quantize_int8(kc)
    vc8, vs = oracle.quantize_int8(vc)
    assert np.array_equal(bits(dw.kc8), kc8.view(np.uint8)) and np.array_equal(bits(dw.k_scales), ks.view(np.uint8))
    op = w.steps[0][0]
    ref8 = oracle.decode(op.q, kc8, vc8, op.block_tables, op.seq_lens, w.scale, ks, vs)
    assert_close(got8[0], ref8, "float16", "long int8")


def test_mha_prefix_full():
    w = W.mha_prefix()
    ref, kc, vc = replay(w)
    got, dw = run_gpu(w, -1)
    assert_close(got[0], ref[0], "float16", "mha_prefix")
    # after copy-on-write the shared prefix blocks are unchanged and the caches match bit for bit
    assert np.array_equal(bits(dw.kc), kc.view(np.uint8))


@pytest.mark.slow
def test_ragged_full_trace():
    """The continuous-batching trace in the benchmark's launch configuration:
    all 128 steps on the GPU, oracle decode on 8 sampled steps, caches bit-exact."""
    w = W.ragged()
    sample = {0, 1, 2, 31, 64, 100, 126, 127}
    ref, kc, vc = replay(w, want=lambda s: s in sample)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    for i in range(len(w.steps)):
        out = dw.run_step(i, -1)
        if i in sample:
            assert_close(out, ref[i], "float16", f"ragged step {i}")
    torch.cuda.synchronize()
    assert np.array_equal(bits(dw.kc), kc.view(np.uint8))
    assert np.array_equal(bits(dw.vc), vc.view(np.uint8))


@pytest.mark.slow
def test_ragged_trace_back_to_back_inputs_ready():
    """The benchmark's exact issue pattern: all 128 steps (append, then decode)
    through the pre-marshalled C-ABI calls on one stream with no synchronisation
    in between, decodes flagged PA_DECODE_INPUTS_READY, so each kernel may start
    while the one before it finishes.  Sampled steps against the oracle, caches
    bit-exact at the end."""
    w = W.ragged()
    sample = {0, 5, 47, 90, 127}
    ref, kc, vc = replay(w, want=lambda s: s in sample)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    calls = runner.StepCalls(dw, -1, False, pa.PA_ALGO_AUTO, stream, flags=pa.PA_DECODE_INPUTS_READY)
    with torch.cuda.stream(stream):
        for i in range(len(w.steps)):
            calls.run(i)
    torch.cuda.synchronize()
    for i in sorted(sample):
        out = dw.steps[i][-1][-1]
        assert_close(out, ref[i], "float16", f"ragged step {i}")
    assert np.array_equal(bits(dw.kc), kc.view(np.uint8))
    assert np.array_equal(bits(dw.vc), vc.view(np.uint8))


@pytest.mark.slow
def test_ragged_trace_appends_overlapping_the_previous_decode():
    """The ragged trace issued back to back with every append flagged
    PA_APPEND_OVERLAP_PREVIOUS (the recipe reuses freed blocks one step late, so
    no append writes a slot the previous decode reads): each append runs while the
    previous decode finishes.  Sampled steps against the oracle, caches bit-exact."""
    w = W.ragged()
    sample = {1, 2, 33, 77, 127}
    ref, kc, vc = replay(w, want=lambda s: s in sample)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    calls = runner.StepCalls(dw, -1, False, pa.PA_ALGO_AUTO, stream, flags=pa.PA_DECODE_INPUTS_READY,
                             append_flags=pa.PA_APPEND_OVERLAP_PREVIOUS)
    with torch.cuda.stream(stream):
        for i in range(len(w.steps)):
            calls.run(i)
    torch.cuda.synchronize()
    for i in sorted(sample):
        assert_close(dw.steps[i][-1][-1], ref[i], "float16", f"ragged step {i}")
    assert np.array_equal(bits(dw.kc), kc.view(np.uint8))
    assert np.array_equal(bits(dw.vc), vc.view(np.uint8))


@pytest.mark.parametrize("hq,hkv", [(32, 1), (64, 2), (16, 1)])
@pytest.mark.parametrize("kind", ["float16", "int8"])
def test_virtual_heads_uniform_and_near_uniform_lengths(hq, hkv, kind):
    """Groups above 8 heads (virtual KV heads sharing one cache head's tiles)
    with every sequence the same length, and with one sequence a token shorter,
    on the tensor-core family's balanced schedule, fp16 and int8 caches, against
    the oracle."""
    for lens in ([1024] * 4, [1024] * 3 + [1023]):
        w = W.random_case(lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=128, dtype="float16",
                          seed=hq + hkv)
        dw = runner.DeviceWorkload(w)
        dw.run_setup()
        if kind == "int8":
            dw.quantize_int8()
        got = dw.run_step(0, -1, int8=kind == "int8", algo=pa.PA_ALGO_TENSOR)
        torch.cuda.synchronize()
        op = w.steps[0][0]
        if kind == "int8":
            ref = oracle.decode(op.q, dw.kc8.cpu().numpy(), dw.vc8.cpu().numpy(), op.block_tables, op.seq_lens,
                                w.scale, dw.k_scales.cpu().numpy(), dw.v_scales.cpu().numpy())
        else:
            ref = oracle.decode(op.q, dw.kc.cpu().numpy(), dw.vc.cpu().numpy(), op.block_tables, op.seq_lens,
                                w.scale)
        assert_close(got, ref, "float16", f"{kind} G={hq // hkv} lens={lens[-1]}")


@pytest.mark.parametrize("algo", [pa.PA_ALGO_SIMT, pa.PA_ALGO_TENSOR])
def test_inputs_ready_flag_same_result(algo):
    """The early-start flag changes when the kernel waits, not what it computes."""
    w = W.random_case([1, 16, 33, 700, 1500], num_q_heads=32, num_kv_heads=8, head_dim=128, seed=12)
    ref, _, _ = replay(w)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    _, q, bt, sl, mx, _ = dw.steps[0][-1]
    outs = []
    for flags in (0, pa.PA_DECODE_INPUTS_READY):
        out = torch.empty_like(q)
        ws = dw.workspace_for(dw.steps[0][-1], -1, algo=algo)
        pa.pa_decode(out, q, dw.kc, dw.vc, bt, sl, w.scale, mx, partition_size=-1, workspace=ws,
                     algo=algo, flags=flags)
        outs.append(out)
    torch.cuda.synchronize()
    assert np.array_equal(bits(outs[0]), bits(outs[1]))
    assert_close(outs[1], ref[0], "float16", "inputs-ready")


# -- wider shapes: MQA-style large groups, head_dim 256 ------------------------------------
@pytest.mark.parametrize("algo", [pa.PA_ALGO_SIMT, pa.PA_ALGO_TENSOR])
@pytest.mark.parametrize("hq,hkv", [(16, 1), (32, 1), (64, 1), (32, 2)])
@pytest.mark.parametrize("part", [0, 16, -1])
def test_large_groups(hq, hkv, part, algo):
    """G = 16 .. 64 (H_kv = 1 is MQA) run as 8-head groups over the same KV
    tiles; both families against the oracle, ragged tails included."""
    w = W.random_case([1, 16, 40, 300, 901], num_q_heads=hq, num_kv_heads=hkv, head_dim=128,
                      dtype="float16", seed=hq * 7 + hkv)
    ref, _, _ = replay(w)
    got, _ = run_gpu(w, part, algo)
    assert_close(got[0], ref[0], "float16", f"G={hq // hkv} part={part}")


@pytest.mark.parametrize("scale", [-0.07, 0.0, 0.5])
@pytest.mark.parametrize("hq", [32, 64])
def test_large_groups_any_scale(hq, scale):
    """The cooperative mode keeps scores unscaled and folds the scale into the
    exponent: a negative scale (flipped into q), a zero scale (uniform weights) and a
    sharp one, against the oracle."""
    w = W.random_case([3, 40, 301], num_q_heads=hq, num_kv_heads=1, head_dim=128, dtype="float16",
                      seed=hq + 5)
    w.scale = scale
    ref, _, _ = replay(w)
    got, _ = run_gpu(w, -1)
    assert_close(got[0], ref[0], "float16", f"G={hq} scale={scale}")


@pytest.mark.parametrize("qdt", ["float16", "bfloat16"])
def test_large_group_bf16_and_int8(qdt):
    w = W.random_case([7, 129, 640], num_q_heads=64, num_kv_heads=1, head_dim=128, dtype=qdt, seed=77)
    ref, _, _ = replay(w)
    got, dw = run_gpu(w, -1)
    check(got[0], ref[0], qdt, "MQA G=64", dw, -1, pa.PA_ALGO_AUTO)
    got8, dw = run_gpu(w, -1, int8=True, dw=runner.DeviceWorkload(w))
    kc8, vc8 = dw.kc8.cpu().numpy(), dw.vc8.cpu().numpy()
    ks, vs = dw.k_scales.cpu().numpy(), dw.v_scales.cpu().numpy()
    op = w.steps[0][0]
    ref8 = oracle.decode(op.q, kc8, vc8, op.block_tables, op.seq_lens, w.scale, ks, vs)
    check(got8[0], ref8, qdt, "MQA G=64 int8", dw, -1, pa.PA_ALGO_AUTO, int8=True)


@pytest.mark.parametrize("algo", [pa.PA_ALGO_SIMT, pa.PA_ALGO_TENSOR])
@pytest.mark.parametrize("qdt", ["float16", "bfloat16"])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 4), (32, 4), (32, 1), (6, 2)])
@pytest.mark.parametrize("part", [0, 32, -1])
def test_head_dim_256(qdt, hq, hkv, part, algo):
    """head_dim 256 on both families (the tensor-core family is the library's pick
    for fp16/bf16), ragged tails and partitions, padded groups (G = 3) on the
    tensor-core family only."""
    if algo == pa.PA_ALGO_SIMT and hq // hkv == 3:
        pytest.skip("the CUDA-core family takes G in 1, 2, 4, 8 and multiples of 8")
    w = W.random_case([1, 17, 200, 513], num_q_heads=hq, num_kv_heads=hkv, head_dim=256, dtype=qdt,
                      seed=hq + hkv + 256)
    ref, _, _ = replay(w)
    got, dw = run_gpu(w, part, algo)
    check(got[0], ref[0], qdt, f"d=256 G={hq // hkv} part={part} algo={algo}", dw, part, algo)


@pytest.mark.parametrize("Q", [2, 3])
def test_head_dim_256_multi_query(Q):
    """Several new tokens per sequence at head_dim 256 (tensor-core family)."""
    w = W.random_multi_case([Q, 40, 300], Q, num_q_heads=16, num_kv_heads=4, head_dim=256,
                            dtype="float16", seed=256 + Q)
    ref, _, _ = replay(w)
    got, dw = run_gpu(w, -1, pa.PA_ALGO_TENSOR)
    assert_close(got[0], ref[0], "float16", f"d=256 Q={Q}")


@pytest.mark.parametrize("algo", [pa.PA_ALGO_SIMT, pa.PA_ALGO_TENSOR])
@pytest.mark.parametrize("hq,hkv", [(16, 4), (8, 8), (32, 4), (64, 1)])
@pytest.mark.parametrize("part", [0, 16, -1])
def test_head_dim_256_int8(hq, hkv, part, algo):
    """int8 caches at head_dim 256 on both families (the tensor-core family reads
    each 256-byte row as two 128-byte boxes), against the oracle dequantising the
    same int8 values; one-pass, one-block and library-picked partitions."""
    if algo == pa.PA_ALGO_SIMT and hq // hkv > 8:
        pytest.skip("int8 on the CUDA-core family: G in 1, 2, 4, 8")
    w = W.random_case([3, 16, 100, 700], num_q_heads=hq, num_kv_heads=hkv, head_dim=256, dtype="float16",
                      seed=256 + hq + hkv)
    got, dw = run_gpu(w, part, algo, int8=True, dw=runner.DeviceWorkload(w))
    kc8, vc8 = dw.kc8.cpu().numpy(), dw.vc8.cpu().numpy()
    ks, vs = dw.k_scales.cpu().numpy(), dw.v_scales.cpu().numpy()
    op = w.steps[0][0]
    ref = oracle.decode(op.q, kc8, vc8, op.block_tables, op.seq_lens, w.scale, ks, vs)
    assert_close(got[0], ref, "float16", f"d=256 int8 G={hq // hkv} part={part} algo={algo}")


@pytest.mark.parametrize("Q", [2, 3])
def test_head_dim_256_int8_multi_query(Q):
    """Several new tokens per sequence over an int8 cache at head_dim 256."""
    w = W.random_multi_case([Q, 40, 300], Q, num_q_heads=16, num_kv_heads=4, head_dim=256,
                            dtype="float16", seed=512 + Q)
    got, dw = run_gpu(w, -1, pa.PA_ALGO_TENSOR, int8=True, dw=runner.DeviceWorkload(w))
    kc8, vc8 = dw.kc8.cpu().numpy(), dw.vc8.cpu().numpy()
    ks, vs = dw.k_scales.cpu().numpy(), dw.v_scales.cpu().numpy()
    op = w.steps[0][0]
    ref = oracle.decode_multi(op.q, kc8, vc8, op.block_tables, op.seq_lens, w.scale, ks, vs)
    assert_close(got[0], ref, "float16", f"d=256 int8 Q={Q}")


@pytest.mark.slow
@pytest.mark.parametrize("name", ["mqa", "mqa64", "d256"])
def test_wide_workloads_full_size_sampled(name):
    """The benchmark's MQA and head_dim-256 workloads at full size, in the bench's
    launch configuration (library-picked partition, inputs-ready flag), against
    the oracle on sampled (sequence, head) rows; MQA through the tcgen05 kernel as
    well (which the library itself picks for the groups of 64)."""
    w = W.NAMED[name]()
    B, Hq = w.steps[0][0].q.shape[:2]
    rng = np.random.default_rng(0)
    rows = np.array([[b, h] for b in rng.choice(B, 3, replace=False) for h in (0, Hq // 2, Hq - 1)],
                    dtype=np.int32)
    ref, _, _ = replay(w, fill_nan=False, bh=rows)
    dw = runner.DeviceWorkload(w, fill_nan=False)
    dw.run_setup()
    calls = runner.StepCalls(dw, -1, False, pa.PA_ALGO_AUTO, flags=pa.PA_DECODE_INPUTS_READY)
    calls.run(0)
    torch.cuda.synchronize()
    out = dw.steps[0][-1][-1]
    assert_close(out, ref[0], "float16", name, rows=rows)
    if name == "mqa":
        # the opt-in tcgen05 kernel, same launch configuration
        out.fill_(float("nan"))
        calls = runner.StepCalls(dw, -1, False, pa.PA_ALGO_TCGEN05, flags=pa.PA_DECODE_INPUTS_READY)
        calls.run(0)
        torch.cuda.synchronize()
        assert_close(out, ref[0], "float16", name + " tcgen05", rows=rows)


# -- several new tokens per sequence (causal among them) -----------------------------------
MULTI = [
    # (H_q, H_kv, Q): columns per KV head = Q * G
    (8, 2, 2),    # 8 columns, one row
    (32, 8, 3),   # 12 columns: a full row and a half-padded one
    (8, 8, 5),    # G = 1: 5 columns padded to 8
    (32, 1, 2),   # MQA: 64 columns, 8 rows per KV head
    (16, 8, 1),   # single token, G = 2
    (6, 2, 1),    # G = 3 padded to 4
]


@pytest.mark.parametrize("qdt", ["float16", "bfloat16"])
@pytest.mark.parametrize("hq,hkv,Q", MULTI)
@pytest.mark.parametrize("part", [0, 16, -1])
def test_multi_query(qdt, hq, hkv, Q, part):
    """Q new tokens per sequence against the oracle; lengths below 16, equal to
    Q, and ragged tails."""
    lens = [Q, Q + 3, 16, 100, 513]
    w = W.random_multi_case(lens, Q, num_q_heads=hq, num_kv_heads=hkv, head_dim=128, dtype=qdt,
                            seed=hq * 10 + hkv + Q)
    ref, _, _ = replay(w)
    got, dw = run_gpu(w, part, pa.PA_ALGO_TENSOR)
    assert got[0].shape == (len(lens), Q, hq, 128)
    check(got[0], ref[0], qdt, f"Q={Q} G={hq // hkv} part={part}", dw, part, pa.PA_ALGO_TENSOR)


def test_multi_query_int8_and_d64():
    w = W.random_multi_case([4, 90, 300], 4, num_q_heads=8, num_kv_heads=4, head_dim=128,
                            dtype="float16", seed=31)
    got, dw = run_gpu(w, -1, int8=True, dw=runner.DeviceWorkload(w))
    kc8, vc8 = dw.kc8.cpu().numpy(), dw.vc8.cpu().numpy()
    ks, vs = dw.k_scales.cpu().numpy(), dw.v_scales.cpu().numpy()
    op = w.steps[0][0]
    ref = oracle.decode_multi(op.q, kc8, vc8, op.block_tables, op.seq_lens, w.scale, ks, vs)
    assert_close(got[0], ref, "float16", "multi int8")
    w = W.random_multi_case([7, 64, 129], 3, num_q_heads=4, num_kv_heads=2, head_dim=64,
                            dtype="bfloat16", seed=32)
    ref, _, _ = replay(w)
    got, dw = run_gpu(w, 16)
    check(got[0], ref[0], "bfloat16", "multi d=64", dw, 16, pa.PA_ALGO_AUTO)


@pytest.mark.slow
def test_specdec_trace_back_to_back():
    """The speculative-verification workload in the bench's issue pattern: 16
    steps of (append 2 tokens per sequence, decode both) back to back with the
    inputs-ready flag; sampled steps against the oracle."""
    w = W.specdec()
    sample = {0, 7, 15}
    ref, kc, vc = replay(w, want=lambda s: s in sample, fill_nan=False)
    dw = runner.DeviceWorkload(w, fill_nan=False)
    dw.run_setup()
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    calls = runner.StepCalls(dw, -1, False, pa.PA_ALGO_AUTO, stream, flags=pa.PA_DECODE_INPUTS_READY)
    with torch.cuda.stream(stream):
        for i in range(len(w.steps)):
            calls.run(i)
    torch.cuda.synchronize()
    for i in sorted(sample):
        assert_close(dw.steps[i][-1][-1], ref[i], "float16", f"specdec step {i}")
    assert np.array_equal(bits(dw.kc), kc.view(np.uint8))


# -- 4-bit caches ---------------------------------------------------------------------------
def _int4_ref(w, dw, multi=False):
    kc4, vc4 = dw.kc8.cpu().numpy(), dw.vc8.cpu().numpy()
    ks, vs = dw.k_scales.cpu().numpy(), dw.v_scales.cpu().numpy()
    op = w.steps[0][0]
    fn = oracle.decode_multi if multi else oracle.decode
    return fn(op.q, kc4, vc4, op.block_tables, op.seq_lens, w.scale, ks, vs)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (64, 8), (32, 1)])
@pytest.mark.parametrize("part", [0, 16, -1])
def test_int4_decode(hq, hkv, part):
    """4-bit caches on the tensor-core family against the oracle decoding the very
    same packed bytes and scales (device-quantised, bit-exact with the oracle's
    quantiser per test_gpu_cache_ops)."""
    w = W.random_case([1, 15, 16, 33, 250, 777], num_q_heads=hq, num_kv_heads=hkv, head_dim=128,
                      dtype="float16", seed=hq + 2 * hkv)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    dw.quantize_int4()
    got = dw.run_step(0, part, int8=True, algo=pa.PA_ALGO_TENSOR)
    torch.cuda.synchronize()
    assert_close(got, _int4_ref(w, dw), "float16", f"int4 G={hq // hkv} part={part}")


def test_int4_multi_query_and_auto():
    w = W.random_multi_case([3, 64, 500], 2, num_q_heads=16, num_kv_heads=4, head_dim=128,
                            dtype="float16", seed=44)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    dw.quantize_int4()
    got = dw.run_step(0, -1, int8=True, algo=pa.PA_ALGO_AUTO)
    torch.cuda.synchronize()
    assert_close(got, _int4_ref(w, dw, multi=True), "float16", "int4 multi-query")


def test_int4_rejected_off_its_path():
    """4-bit caches need fp16 q and head_dim 128 on the tensor-core family."""
    w = W.random_case([40], num_q_heads=8, num_kv_heads=2, head_dim=128, dtype="float16", seed=45)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    dw.quantize_int4()
    _, q, bt, sl, mx, out = dw.steps[0][-1]
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode(out, q, dw.kc8, dw.vc8, bt, sl, w.scale, mx, dw.k_scales, dw.v_scales,
                     algo=pa.PA_ALGO_SIMT)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED


# -- one workspace across calls of any shape; the failure path of the bounded waits ---------
def _oracle_ref(w, dw, int8=False):
    op = w.steps[0][0]
    if int8:
        return oracle.decode(op.q, dw.kc8.cpu().numpy(), dw.vc8.cpu().numpy(), op.block_tables,
                             op.seq_lens, w.scale, dw.k_scales.cpu().numpy(), dw.v_scales.cpu().numpy())
    return oracle.decode(op.q, dw.kc.cpu().numpy(), dw.vc.cpu().numpy(), op.block_tables, op.seq_lens,
                         w.scale)


def test_workspace_shared_across_parameter_sets():
    """One workspace, never initialised (filled with 0xff garbage once), serves
    calls whose parameters differ: a 6-sequence batch split into 16-token
    partitions, a 3-sequence batch with 256-token partitions, the CUDA-core
    family's split, MQA rows (the cooperative mode), and the first call again;
    each against the oracle."""
    wa = W.random_case([1, 40, 300, 777, 1500, 2047], num_q_heads=32, num_kv_heads=8, head_dim=128, seed=81)
    wb = W.random_case([900, 3000, 20], num_q_heads=16, num_kv_heads=2, head_dim=128, seed=82)
    wc = W.random_case([64, 1000, 513, 2], num_q_heads=32, num_kv_heads=1, head_dim=128, seed=83)
    runs = []
    for w in (wa, wb, wc):
        dw = runner.DeviceWorkload(w)
        dw.run_setup()
        runs.append((w, dw, _oracle_ref(w, dw)))
    calls = [(0, 16, pa.PA_ALGO_TENSOR), (1, 256, pa.PA_ALGO_TENSOR), (0, 32, pa.PA_ALGO_SIMT),
             (1, 16, pa.PA_ALGO_TENSOR), (2, -1, pa.PA_ALGO_TENSOR), (1, 64, pa.PA_ALGO_SIMT),
             (0, 16, pa.PA_ALGO_TENSOR), (2, 16, pa.PA_ALGO_TENSOR), (0, -1, pa.PA_ALGO_AUTO)]
    need = 0
    for k, part, algo in calls:
        w, dw, _ = runs[k]
        _, q, bt, _, mx, _ = dw.steps[0][-1]
        need = max(need, pa.pa_decode_workspace_size(q, dw.kc, bt, mx, part, algo=algo))
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    for n, (k, part, algo) in enumerate(calls):
        w, dw, ref = runs[k]
        _, q, bt, sl, mx, _ = dw.steps[0][-1]
        out = torch.full_like(q, float("nan"))
        pa.pa_decode(out, q, dw.kc, dw.vc, bt, sl, w.scale, mx, partition_size=part, workspace=ws, algo=algo)
        assert_close(out, ref, "float16", f"call {n}: case {k} part={part} algo={algo}")


@pytest.mark.parametrize("stall_at", [0, 3])
def test_wait_timeout_reported_and_workspace_left_ready(stall_at):
    """The failure path of the bounded waits on a working GPU, without a fault:
    the first worker of the tensor-core family leaves one of its copies
    unissued, so its wait for that stage runs out after 5 ms.  The call returns,
    the host reads PA_EFLAG_WAIT_TIMEOUT, every row the worker did not touch still
    matches the oracle (the worker's partials are written empty, so the merge
    kernel reads no stale slot: the workspace starts as 0xff garbage), and the
    next decode on the same workspace matches the oracle on every row."""
    lens = [1000, 3000, 500]
    w = W.random_case(lens, num_q_heads=32, num_kv_heads=8, head_dim=128, seed=91)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    ref = _oracle_ref(w, dw)
    _, q, bt, sl, mx, _ = dw.steps[0][-1]
    ws = dw.workspace_for(dw.steps[0][-1], -1, algo=pa.PA_ALGO_TENSOR)
    ws.fill_(0xFF)
    out = torch.full_like(q, float("nan"))
    pa.pa_get_error_flags(reset=True)
    limit_ns = 5_000_000
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    pa.pa_decode_stall_selftest(out, q, dw.kc, dw.vc, bt, sl, w.scale, mx, stall_at, limit_ns,
                                partition_size=-1, workspace=ws)
    b.record()
    torch.cuda.synchronize()
    assert a.elapsed_time(b) >= limit_ns / 1e6  # the wait ran its whole limit, then gave up
    assert pa.pa_get_error_flags(reset=True) == pa.PA_EFLAG_WAIT_TIMEOUT
    # the stream's first 8-block chunk (the first worker's) lies in sequence 0, KV head 0:
    # query heads 0-3 of sequence 0; every other row is untouched by the failure
    got = out.double().cpu().numpy()
    keep = np.ones(got.shape[:2], dtype=bool)
    keep[0, 0:4] = False
    assert np.all(np.isfinite(got))
    rows = np.argwhere(keep)
    assert_close(out, ref, "float16", "rows away from the stalled worker", rows=rows)
    # the workspace serves the next call unchanged
    out2 = torch.full_like(q, float("nan"))
    pa.pa_decode(out2, q, dw.kc, dw.vc, bt, sl, w.scale, mx, partition_size=-1, workspace=ws,
                 algo=pa.PA_ALGO_TENSOR)
    assert_close(out2, ref, "float16", "next call")


# -- the tcgen05 kernel (PA_ALGO_TCGEN05, groups of 32 or 64 heads per KV head) ----------
@pytest.mark.parametrize("qdt", ["float16", "bfloat16"])
@pytest.mark.parametrize("hq,hkv", [(32, 1), (64, 1), (64, 2), (128, 4)])
@pytest.mark.parametrize("part", [16, 48, -1])
def test_tcgen05_large_groups(hq, hkv, part, qdt):
    """The tcgen05 kernel against the oracle: lengths of 1 token, a block, a block plus
    one, ragged tails; one-block, three-block and library-picked partitions (groups of
    1-4 blocks, rows cut anywhere); bf16 through its fp32 result."""
    w = W.random_case([1, 16, 17, 40, 300, 901], num_q_heads=hq, num_kv_heads=hkv, head_dim=128, dtype=qdt,
                      seed=hq * 3 + hkv + part)
    ref, _, _ = replay(w)
    got, dw = run_gpu(w, part, pa.PA_ALGO_TCGEN05)
    check(got[0], ref[0], qdt, f"tcgen05 G={hq // hkv} part={part}", dw, part, pa.PA_ALGO_TCGEN05)


@pytest.mark.parametrize("q_scale", [1.0, 6.0])
@pytest.mark.parametrize("part", [-1, 128, 256])
def test_tcgen05_edge_lengths(part, q_scale):
    """Empty sequences (zero rows), rows of exactly one and two 8-block groups and one
    token past them, rows spanning many groups, chunks of one or two groups (128, 256
    tokens); a sharpened softmax (q scaled by 6) moves the running maximum past the lazy
    threshold mid-row, so O is rescaled in tensor memory."""
    lens = [0, 128, 129, 255, 256, 2049, 0, 5, 1500]
    w = W.random_case(lens, num_q_heads=64, num_kv_heads=2, head_dim=128, dtype="float16",
                      seed=17 + part + int(q_scale), q_scale=q_scale)
    ref, _, _ = replay(w)
    got, dw = run_gpu(w, part, pa.PA_ALGO_TCGEN05)
    check(got[0], ref[0], "float16", f"tcgen05 edges part={part} q_scale={q_scale}", dw, part, pa.PA_ALGO_TCGEN05)


@pytest.mark.parametrize("scale", [-0.07, 0.0, 0.5])
def test_tcgen05_any_scale(scale):
    w = W.random_case([3, 40, 301], num_q_heads=64, num_kv_heads=1, head_dim=128, dtype="float16", seed=71)
    w.scale = scale
    ref, _, _ = replay(w)
    got, _ = run_gpu(w, -1, pa.PA_ALGO_TCGEN05)
    assert_close(got[0], ref[0], "float16", f"tcgen05 scale={scale}")


def test_tcgen05_skips_blocks_outside_the_pool():
    """A table entry outside the pool: PA_EFLAG_BAD_BLOCK; the block's scores are masked
    and its V rows zeroed, every other token counts.  Expected: dense fp64 attention over
    the workload's own K/V without that block's tokens."""
    w = W.random_case([40, 300], num_q_heads=32, num_kv_heads=1, head_dim=128, seed=72)
    op = w.steps[0][0]
    op.block_tables[1, 3] = w.num_blocks + 5
    got, _ = run_gpu(w, -1, pa.PA_ALGO_TCGEN05)
    assert pa.pa_get_error_flags(reset=True) == pa.PA_EFLAG_BAD_BLOCK
    for b in (0, 1):
        k, v = (x.astype(np.float64)[:, 0] for x in w.logical[b])
        keep = [t for t in range(int(op.seq_lens[b])) if b == 0 or t // 16 != 3]
        s_ = op.q[b].astype(np.float64) @ k[keep].T * w.scale
        p_ = np.exp(s_ - s_.max(axis=1, keepdims=True))
        ref = (p_ / p_.sum(axis=1, keepdims=True)) @ v[keep]
        g = got[0][b].double().cpu().numpy()
        assert np.all(np.abs(g - ref) <= 2e-3 + 2e-3 * np.abs(ref)), b


@pytest.mark.parametrize("stall_at", [0, 2])
def test_tcgen05_wait_timeout(stall_at):
    """The tcgen05 kernel's failure path: the first CTA leaves one group's copies
    unissued; its producer, MMA and softmax warps give up after 5 ms, write empty
    results and release the tensor memory.  The flag is raised, the other sequences
    match the oracle, and the next call on the same workspace matches everywhere."""
    # long enough that every CTA's chunk spans more than three groups of 8 blocks
    lens = [40000, 30000, 8000]
    w = W.random_case(lens, num_q_heads=32, num_kv_heads=1, head_dim=128, seed=93)
    dw = runner.DeviceWorkload(w)
    dw.run_setup()
    ref, _, _ = replay(w)
    _, q, bt, sl, mx, _ = dw.steps[0][-1]
    ws = dw.workspace_for(dw.steps[0][-1], -1, algo=pa.PA_ALGO_TCGEN05)
    ws.fill_(0xFF)
    out = torch.full_like(q, float("nan"))
    pa.pa_get_error_flags(reset=True)
    pa.pa_decode_stall_selftest(out, q, dw.kc, dw.vc, bt, sl, w.scale, mx, stall_at, 5_000_000,
                                partition_size=-1, workspace=ws, algo=pa.PA_ALGO_TCGEN05)
    torch.cuda.synchronize()
    assert pa.pa_get_error_flags(reset=True) == pa.PA_EFLAG_WAIT_TIMEOUT
    got = out.double().cpu().numpy()
    assert np.all(np.isfinite(got))
    # the first CTA's chunk lies in sequence 0; sequences 1 and 2 are untouched
    rows = [(b, h) for b in (1, 2) for h in range(32)]
    assert_close(out, ref[0], "float16", "sequences away from the stalled CTA", rows=rows)
    out2 = torch.full_like(q, float("nan"))
    pa.pa_decode(out2, q, dw.kc, dw.vc, bt, sl, w.scale, mx, partition_size=-1, workspace=ws,
                 algo=pa.PA_ALGO_TCGEN05)
    assert_close(out2, ref[0], "float16", "next call")
