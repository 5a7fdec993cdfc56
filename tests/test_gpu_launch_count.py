"""The kernel launches of one pa_decode call, as the profiler records them, against
pa_decode_launches (the count the benchmark's gpu_launches is built from)."""
import pytest
import torch

from paged_kv_cache_395_b200 import pa, runner, workloads as W

pytestmark = pytest.mark.gpu


def _library_kernels(fn):
    """Names of the kernels of this library (namespace pa::) that fn launches."""
    torch.cuda.synchronize()
    with torch.profiler.profile(activities=[torch.profiler.ProfilerActivity.CUDA]) as prof:
        fn()
        torch.cuda.synchronize()
    cuda = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    if not cuda:
        pytest.skip("the profiler recorded no device activity here")
    return [n for n in cuda if "pa::" in n]


@pytest.mark.parametrize("case", [
    dict(hq=32, hkv=8, part=0, algo=pa.PA_ALGO_AUTO),       # one pass
    dict(hq=32, hkv=8, part=-1, algo=pa.PA_ALGO_AUTO),      # split, per-warp kernel + merge
    dict(hq=32, hkv=1, part=-1, algo=pa.PA_ALGO_AUTO),      # cooperative kernel + merge
    dict(hq=32, hkv=1, part=-1, algo=pa.PA_ALGO_TCGEN05),   # tcgen05 kernel + merge
    dict(hq=32, hkv=8, part=64, algo=pa.PA_ALGO_SIMT),      # CUDA-core family, split + merge
    dict(hq=32, hkv=8, part=0, algo=pa.PA_ALGO_SIMT),       # CUDA-core family, one pass
])
def test_launches_match_the_profiler(case):
    w = W.random_case([40, 700, 3000], num_q_heads=case["hq"], num_kv_heads=case["hkv"], head_dim=128,
                      dtype="float16", seed=5)
    dw = runner.DeviceWorkload(w, fill_nan=False)
    dw.run_setup()
    _, q, bt, sl, mx, out = dw.steps[0][-1]
    want = pa.pa_decode_launches(q, dw.kc, bt, mx, case["part"], algo=case["algo"])
    ws = dw.workspace_for(dw.steps[0][-1], case["part"], algo=case["algo"])

    def call():
        pa.pa_decode(out, q, dw.kc, dw.vc, bt, sl, w.scale, mx, partition_size=case["part"], workspace=ws,
                     algo=case["algo"])
    call()  # first call: one-time setup (attributes, tensor maps) outside the profile
    names = _library_kernels(call)
    assert len(names) == want, (names, want)
    assert 1 <= want <= 2
    if want == 2:
        assert any("merge" in n for n in names), names


def test_bench_step_launch_count_matches_the_profiler():
    """The benchmark's ragged step (admitted prompts, then pa_decode_append fused with
    its merge): the runner's per-step launch count, which gpu_launches sums, equals the
    library kernels the profiler records, on steps with and without admitted prompts."""
    w = W.ragged()
    dw = runner.DeviceWorkload(w, fill_nan=False)
    dw.run_setup()
    stream = torch.cuda.current_stream()
    calls = runner.StepCalls(dw, -1, False, pa.PA_ALGO_AUTO, stream, flags=pa.PA_DECODE_INPUTS_READY, fused=True,
                             prompt_flags=pa.PA_APPEND_OVERLAP_PREVIOUS)
    assert calls.fused_steps == len(w.steps)
    seen = set()
    for i in range(len(w.steps)):  # every step once, in order (the recipe's block reuse needs it)
        has_prompts = any(n == "reshape" for n, _, _ in calls.calls[i])
        if i >= 2 and has_prompts not in seen:
            names = _library_kernels(lambda: calls.run(i))
            assert len(names) == calls.launches[i], (i, names, calls.launches[i])
            seen.add(has_prompts)
            if len(seen) == 2:
                break
        else:
            calls.run(i)
    assert seen == {True, False}
