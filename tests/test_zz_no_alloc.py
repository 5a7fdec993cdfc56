"""pa_decode_fixed_scratch (split-K decode on the library's fixed scratch area)
against pa_decode with a caller-allocated workspace, and against the oracle.

The file name sorts last so that, in a full run, these calls come after every
other test has used the device; the tests also pass when run alone.  Two calls
in a row check that a call leaves the fixed area ready for the next one, and
calls with different parameters in a row that nothing one call leaves there
matters to the next.
"""
import numpy as np
import pytest
import torch

from paged_kv_cache_395_b200 import pa, runner, workloads as W

from .gpu_util import TOL, assert_close, gpu_f64
from .oracle_replay import replay

pytestmark = pytest.mark.gpu


def _close(got, ref, dtype, what):
    atol, rtol = TOL[dtype]
    g, r = gpu_f64(got), gpu_f64(ref)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    bad = np.abs(g - r) > atol + rtol * np.abs(r)
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside tolerance"


def _decode_pair(w, partition_size, algo, int8=False):
    dw = runner.DeviceWorkload(w, fill_nan=False)
    dw.run_setup()
    dw.run_step(0, decode=False)  # the step's append, if it has one
    if int8:
        dw.quantize_int8()
    op = dw.steps[0][-1]
    _, q, bt, sl, mx, _ = op
    kc, vc = (dw.kc8, dw.vc8) if int8 else (dw.kc, dw.vc)
    ks, vs = (dw.k_scales, dw.v_scales) if int8 else (None, None)
    ws = dw.workspace_for(op, partition_size, int8, algo)
    ref = torch.empty_like(q)
    pa.pa_decode(ref, q, kc, vc, bt, sl, w.scale, mx, ks, vs, partition_size, ws, algo)
    outs = []
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        pa.pa_decode_fixed_scratch(o, q, kc, vc, bt, sl, w.scale, mx, ks, vs, partition_size, algo)
        outs.append(o)
    torch.cuda.synchronize()
    return ref, outs


CASES = [
    # (lengths, H_q, H_kv, d, dtype, partition_size, algo, int8)
    ([1, 16, 17, 100, 513, 1000, 2047], 32, 8, 128, "float16", -1, pa.PA_ALGO_AUTO, False),
    ([5, 300, 1500, 64], 32, 8, 128, "bfloat16", 256, pa.PA_ALGO_TENSOR, False),
    ([33, 700, 1200], 16, 2, 64, "float16", 128, pa.PA_ALGO_SIMT, False),
    ([17, 900, 2000], 32, 8, 128, "float16", 512, pa.PA_ALGO_SIMT, True),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_fixed_scratch_matches_caller_workspace(case):
    lens, hq, hkv, d, dt, part, algo, int8 = CASES[case]
    w = W.random_case(lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, dtype=dt, seed=40 + case)
    pa.pa_get_error_flags(reset=True)
    ref, outs = _decode_pair(w, part, algo, int8)
    for i, o in enumerate(outs):
        _close(o, ref, dt, f"call {i + 1}")
    assert pa.pa_get_error_flags(reset=True) == 0


def test_fixed_scratch_ragged_step():
    """One step of the 64-sequence ragged trace (lengths up to 4096), library-picked partition."""
    w = W.ragged(num_steps=1)
    ref, outs = _decode_pair(w, -1, pa.PA_ALGO_AUTO)
    for i, o in enumerate(outs):
        _close(o, ref, "float16", f"call {i + 1}")


def test_fixed_scratch_rejects_oversized_request():
    """Parameters whose workspace exceeds the fixed area are refused before any launch."""
    B, hq, hkv, d, L = 256, 32, 32, 128, 4096
    q = torch.zeros((B, hq, d), dtype=torch.float16, device="cuda")
    kc = torch.zeros((1, hkv, 16, d), dtype=torch.float16, device="cuda")
    bt = torch.zeros((B, L // 16), dtype=torch.int32, device="cuda")
    sl = torch.ones(B, dtype=torch.int32, device="cuda")
    need = pa.pa_decode_workspace_size(q, kc, bt, L, 16, algo=pa.PA_ALGO_SIMT)
    assert need > pa.FIXED_SCRATCH_BYTES
    out = torch.zeros_like(q)
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_fixed_scratch(out, q, kc, kc, bt, sl, 0.1, L, partition_size=16,
                                   algo=pa.PA_ALGO_SIMT)
    assert e.value.status == pa.PA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0


def test_fixed_scratch_alternating_parameter_sets():
    """Calls with different parameters in a row share the fixed area: a ragged
    7-sequence batch split into 16-token partitions, then a 3-sequence batch with
    256-token partitions, the CUDA-core family's split (its partial results start
    at the same offset as the tensor-core family's), and the first case again.
    Each call against pa_decode with a fresh workspace and against the oracle."""
    cases = [
        (W.random_case([1, 16, 17, 100, 513, 1000, 2047], num_q_heads=32, num_kv_heads=8, head_dim=128,
                       dtype="float16", seed=60), 16, pa.PA_ALGO_TENSOR),
        (W.random_case([900, 3000, 20], num_q_heads=16, num_kv_heads=2, head_dim=128, dtype="float16",
                       seed=61), 256, pa.PA_ALGO_TENSOR),
        (W.random_case([700, 64, 1500], num_q_heads=8, num_kv_heads=2, head_dim=128, dtype="float16",
                       seed=62), 128, pa.PA_ALGO_SIMT),
    ]
    prepared = []
    for w, part, algo in cases:
        dw = runner.DeviceWorkload(w)
        dw.run_setup()
        ref, _, _ = replay(w)
        prepared.append((w, dw, ref[0], part, algo))
    torch.cuda.synchronize()
    for n, k in enumerate([0, 1, 2, 0, 1, 0]):
        w, dw, ref, part, algo = prepared[k]
        _, q, bt, sl, mx, _ = dw.steps[0][-1]
        fresh = torch.empty_like(q)
        ws = dw.workspace_for(dw.steps[0][-1], part, algo=algo)
        pa.pa_decode(fresh, q, dw.kc, dw.vc, bt, sl, w.scale, mx, None, None, part, ws, algo)
        o = torch.full_like(q, float("nan"))
        pa.pa_decode_fixed_scratch(o, q, dw.kc, dw.vc, bt, sl, w.scale, mx, None, None, part, algo)
        torch.cuda.synchronize()
        _close(o, fresh, "float16", f"call {n} (case {k}) vs pa_decode")
        assert_close(o, ref, "float16", f"call {n} (case {k}) vs oracle")
    assert pa.pa_get_error_flags(reset=True) == 0
