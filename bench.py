"""Benchmark: paged decode attention KV-read GB/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ragged]
                    [--impl ours|reference] [--partition -1] [--algo auto|simt|tensor]

One step = one decode step of one attention layer over the whole batch: the
append of the step's new tokens (pa_reshape_and_cache, plus copy-on-write
copies where the workload has them) followed by pa_decode (split-K +
log-sum-exp merge where partitions apply).  The default workload is the
continuous-batching ragged trace: 7B-GQA heads (32 q / 8 KV, head_dim 128),
fp16 KV, batch 64, lengths U[16, 4096] growing by one per step for 128 steps,
sequences finishing with p = 0.02 and being replaced by new ones of
U[16, 512] tokens.  Steps beyond 128 replay the trace from its start (same
kernels, same byte counts).

value = algorithmic KV-read bytes of the timed decode steps / device time of
those steps (CUDA events around the whole step: append + decode + merge),
inputs resident in HBM.  On the ragged trace the KV pool (1.1 GB) and the
bytes read per step (140-566 MB) are larger than the 126 MB L2, so the steps
run back to back with no flush; a workload whose steps read less than twice
the L2 size is timed step by step with the L2 flushed in between (outside the
events).  e2e = the same metric through the C ABI with the per-step inputs in
pinned host memory copied in and the outputs copied out inside the timed
region, the copies on their own streams overlapping other steps' kernels as a
serving loop would.  For N > 1 (torchrun) every rank runs an independent replica on its
own GPU (the decode path has no exchange step); value = bytes of all ranks /
max over ranks of the device time.

--impl reference times the CPU oracle (the fp64 C reference of the same
computation) on a bounded sample of the same workload, on rank 0 only.
"""
import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV-read GB/s (% of B200 HBM peak); decode tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic of the decode kernel from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum of the two captured launches, trace steps 8 and 9 of the
# ragged workload, the kernel of pa_decode_append that the bench's step runs), per
# algorithmic byte.
# It holds only for the kernel code it was taken on (hash of the source without
# comments); after any code change the bench reports null until it is taken again.
NCU_TRAFFIC = {
    "ragged": {"source": ["paged_kv_cache_395_b200/csrc/pa_decode_tc.cu",
                          "paged_kv_cache_395_b200/csrc/pa_tc_shared.cuh"], "code": "e113e6a303473e88",
               "per_alg_byte": (475231488 + 7520256 + 462311424 + 6604800) / (472969728 + 459894508)},
}


def code_hash(paths):
    s = "\n".join(open(os.path.join(ROOT, p)).read() for p in paths)
    s = re.sub(r"/\*.*?\*/", " ", s, flags=re.S)
    s = re.sub(r"//[^\n]*", " ", s)
    return hashlib.sha256(" ".join(s.split()).encode()).hexdigest()[:16]


def traffic_per_launch(workload, algo, partition, mean_alg_bytes, fused=True):
    t = NCU_TRAFFIC.get(workload)
    if t is None or algo == "simt" or partition != -1 or not fused or \
            code_hash(t["source"]) != t["code"]:
        return None
    return t["per_alg_byte"] * mean_alg_bytes


WORKLOADS = {
    "ragged": "continuous-batching ragged decode: 7B-GQA 32 q / 8 KV heads, head_dim 128, fp16 KV, "
              "batch 64, lengths U[16,4096], 128 steps of +1 token, finish p=0.02, "
              "new sequences U[16,512]",
    "gqa_b8": "7B-GQA decode: 32 q / 8 KV heads, head_dim 128, fp16, batch 8, all lengths 1024",
    "long": "long context: 7B-GQA heads, fp16, batch 16, all lengths 8192, split-K 512",
    "long_int4": "long context: 7B-GQA heads, 4-bit KV (per-(block, KV head) scales), fp16 q/out, "
                 "batch 16, all lengths 8192, split-K 512",
    "long_int8": "long context: 7B-GQA heads, int8 KV (per-(block, KV head) scales), fp16 q/out, "
                 "batch 16, all lengths 8192, split-K 512",
    "mha_prefix": "MHA 32/32 heads, head_dim 128, fp16, batch 16, shared 1000-token prefix with "
                  "copy-on-write + private suffix U[64,1048]",
    "mqa": "MQA: 32 q heads / 1 KV head, head_dim 128, fp16, batch 128, all lengths 4096",
    "mqa64": "MQA, groups of 64: 64 q heads / 1 KV head, head_dim 128, fp16, batch 128, all lengths 4096",
    "d256": "head_dim 256: 16 q / 8 KV heads, fp16, batch 16, all lengths 4096",
    "d256_int8": "head_dim 256: 16 q / 8 KV heads, int8 KV (per-(block, KV head) scales), fp16 q/out, "
                 "batch 16, all lengths 4096",
    "specdec": "speculative verification: 7B-GQA 32 q / 8 KV heads, head_dim 128, fp16, batch 64, "
               "lengths U[512,4096], 2 new tokens per sequence per step (causal), 16 steps",
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=512)
    ap.add_argument("--warmup", type=int, default=16)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="ragged")
    ap.add_argument("--partition", type=int, default=-1)
    ap.add_argument("--algo", choices=["auto", "simt", "tensor", "tcgen05"], default="auto")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--append", choices=["fused", "plain"], default="fused",
                    help="fused: a step's new tokens go through pa_decode_append (one kernel with "
                         "the decode where the library fuses them); plain: pa_reshape_and_cache "
                         "then pa_decode")
    return ap.parse_args(argv)


def load_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def make_workload(name):
    from paged_kv_cache_395_b200 import workloads as W
    if name == "ragged":
        return W.ragged(), False, 256
    if name == "gqa_b8":
        return W.gqa_b8(), False, 256
    if name == "long":
        return W.long(), False, 512
    if name == "long_int8":
        return W.long(), "i8", 512
    if name == "long_int4":
        return W.long(), "i4", 512
    if name == "mha_prefix":
        return W.mha_prefix(), False, 256
    if name == "mqa":
        return W.mqa(), False, -1
    if name == "mqa64":
        return W.mqa64(), False, -1
    if name == "d256":
        return W.d256(), False, -1
    if name == "d256_int8":
        return W.d256(), "i8", -1
    if name == "specdec":
        return W.specdec(), False, -1
    raise ValueError(name)


def kv_elem_bytes(int8):
    """Bytes per cached value of a quantised pool ("i8": 1, "i4": 0.5), None if not."""
    return {"i8": 1, "i4": 0.5}.get(int8) if int8 else None


def quantize_host(kc, int8):
    """The oracle's quantiser for the pool kind ("i8" or "i4")."""
    import oracle
    return oracle.quantize_int4(kc) if int8 == "i4" else oracle.quantize_int8(kc)


def step_bytes(w, int8):
    from paged_kv_cache_395_b200 import workloads as W
    out = []
    for ops in w.steps:
        dec = [o for o in ops if isinstance(o, W.Decode)][0]
        out.append(W.decode_kv_bytes(dec, w, kv_elem_bytes(int8)))
    return out


def step_tokens(w):
    from paged_kv_cache_395_b200 import workloads as W
    out = []
    for ops in w.steps:
        q = [o for o in ops if isinstance(o, W.Decode)][0].q
        out.append(int(q.shape[0] * (q.shape[1] if q.ndim == 4 else 1)))  # query tokens decoded
    return out


class ClockSampler:
    """Poll NVML (the data nvidia-smi prints) during the timed region."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index, period=0.001):
        self.samples, self.reasons, self.max_mhz, self.ok = [], 0, None, False
        self.period = period
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report it, do not guess
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def report(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.err}
        names = [n for n, b in self.REASONS.items() if self.reasons & b]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def max_over_ranks(ms, dist, device="cuda"):
    """Device time of the slowest rank: every rank times its own replica, and
    the job's time is the largest of them (one all-reduce; identity without a
    process group)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([float(ms)], device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(bytes_rank, ms, dist, device="cuda"):
    """(GB/s of the whole job, max-over-ranks ms): the ranks run identical
    replicas, so the job moves bytes_rank x world bytes in the slowest rank's time."""
    world = 1 if dist is None else dist.get_world_size()
    ms_max = max_over_ranks(ms, dist, device)
    return bytes_rank * world / (ms_max * 1e-3) / 1e9, ms_max


def dist_setup(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def cpu_model():
    """The host CPU's model name (as lscpu prints it), or the platform string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def cpu_baseline(w, int8, seconds, host_caches=None):
    """The oracle as it stands, on this host's cores, over whole decode steps
    of the workload replayed in order until ``seconds`` of work are done."""
    import oracle
    from paged_kv_cache_395_b200 import workloads as W
    N, H, bs, d = w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim
    kc = np.zeros((N, H, bs, d), dtype=w.storage_dtype())
    vc = np.zeros_like(kc)
    for op in w.setup:
        oracle.reshape_and_cache(op.k, op.v, kc, vc, op.slot_mapping)
    ks = vs = None
    if int8:
        kc, ks = quantize_host(kc, int8)
        vc, vs = quantize_host(vc, int8)
    threads = oracle.nthreads_default()
    done_bytes, t_work, nsteps, ntok = 0, 0.0, 0, 0
    for si, ops in enumerate(w.steps):
        for op in ops:
            if isinstance(op, W.Reshape) and not int8:
                oracle.reshape_and_cache(op.k, op.v, kc, vc, op.slot_mapping)
            elif isinstance(op, W.Copy) and op.pairs.size and not int8:
                oracle.block_copy(kc, vc, op.pairs)
            elif isinstance(op, W.Decode):
                t0 = time.perf_counter()
                if op.q.ndim == 4:
                    oracle.decode_multi(op.q, kc, vc, op.block_tables, op.seq_lens, w.scale, ks, vs,
                                        nthreads=threads)
                else:
                    oracle.decode(op.q, kc, vc, op.block_tables, op.seq_lens, w.scale, ks, vs,
                                  nthreads=threads)
                t_work += time.perf_counter() - t0
                done_bytes += W.decode_kv_bytes(op, w, kv_elem_bytes(int8))
                ntok += op.q.shape[0] * (op.q.shape[1] if op.q.ndim == 4 else 1)
                nsteps += 1
        if t_work >= seconds:
            break
    # the same oracle on one thread, over the first four sequences of the first decode
    first = next(op for ops in w.steps for op in ops if isinstance(op, W.Decode))
    n1 = min(4, first.q.shape[0])
    sub = W.Decode(first.q[:n1], first.block_tables[:n1], first.seq_lens[:n1], first.max_seq_len)
    t0 = time.perf_counter()
    if sub.q.ndim == 4:
        oracle.decode_multi(sub.q, kc, vc, sub.block_tables, sub.seq_lens, w.scale, ks, vs, nthreads=1)
    else:
        oracle.decode(sub.q, kc, vc, sub.block_tables, sub.seq_lens, w.scale, ks, vs, nthreads=1)
    t1 = time.perf_counter() - t0
    return {"value": done_bytes / t_work / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{nsteps} whole decode step(s) of the workload in trace order "
                      f"({ntok} sequence decodes, all heads), fp64 C oracle, {t_work:.2f} s",
            "tokens_per_s": ntok / t_work,
            "value_1_thread": W.decode_kv_bytes(sub, w, kv_elem_bytes(int8)) / t1 / 1e9,
            "sample_1_thread": f"the first {n1} sequences of the first decode step on one thread, {t1:.2f} s",
            "cpu_model": cpu_model()}


def reference_arm(args, rank, world):
    if rank != 0:
        return 0
    import oracle
    from paged_kv_cache_395_b200 import workloads as W
    w, int8, _ = make_workload(args.workload)
    N, H, bs, d = w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim
    kc = np.zeros((N, H, bs, d), dtype=w.storage_dtype())
    vc = np.zeros_like(kc)
    for op in w.setup:
        oracle.reshape_and_cache(op.k, op.v, kc, vc, op.slot_mapping)
    ks = vs = None
    if int8:
        kc, ks = quantize_host(kc, int8)
        vc, vs = quantize_host(vc, int8)
    threads = oracle.nthreads_default()
    # each step: the trace's step i % T, a bounded sample of one sequence (all heads)
    decs = [[o for o in ops if isinstance(o, W.Decode)][0] for ops in w.steps]
    T = len(decs)

    def one(i):
        op = decs[i % T]
        b = i % op.q.shape[0]
        if op.q.ndim == 4:
            oracle.decode_multi(op.q[b:b + 1], kc, vc, op.block_tables[b:b + 1], op.seq_lens[b:b + 1],
                                w.scale, ks, vs, nthreads=threads)
        else:
            bh = np.array([[b, h] for h in range(w.num_q_heads)], dtype=np.int32)
            oracle.decode(op.q, kc, vc, op.block_tables, op.seq_lens, w.scale, ks, vs, bh=bh,
                          nthreads=threads)
        L = int(max(op.seq_lens[b], 0))
        E = kv_elem_bytes(int8) if int8 else w.elem_size
        return L * w.num_kv_heads * w.head_dim * 2 * E

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    nbytes = sum(one(args.warmup + i) for i in range(args.steps))
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOADS[args.workload], "name": args.workload},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": "per step: one sequence (all query heads) of trace step "
                                   "i mod T, fp64 C oracle", "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    rank, world, local = dist_setup(args)
    if args.impl == "reference":
        return reference_arm(args, rank, world)

    import torch
    from paged_kv_cache_395_b200 import pa, runner

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    algo = {"auto": pa.PA_ALGO_AUTO, "simt": pa.PA_ALGO_SIMT, "tensor": pa.PA_ALGO_TENSOR,
            "tcgen05": pa.PA_ALGO_TCGEN05}[args.algo]
    w, int8, default_part = make_workload(args.workload)
    part = args.partition
    dw = runner.DeviceWorkload(w, fill_nan=False)
    dw.run_setup()
    if int8 == "i4":
        dw.quantize_int4()
    elif int8:
        dw.quantize_int8()
    stream = torch.cuda.Stream()
    # each decode follows this library's own reshape, decode or merge kernel, which
    # writes none of q, the tables, the lengths or the new tokens: the decode may read
    # those before it finishes
    fused = args.append == "fused"
    # the prompts of admitted sequences were computed earlier (a prefill): where the
    # recipe reuses freed blocks one step late, their append may overlap the kernel
    # before it
    pflags = pa.PA_APPEND_OVERLAP_PREVIOUS if getattr(w, "appends_overlap_previous", False) else 0
    calls = runner.StepCalls(dw, part, int8, algo, stream, flags=pa.PA_DECODE_INPUTS_READY, fused=fused,
                             prompt_flags=pflags)
    plain_calls = runner.StepCalls(dw, part, int8, algo, stream, flags=pa.PA_DECODE_INPUTS_READY) \
        if calls.fused_steps else None
    T = len(w.steps)
    sbytes = step_bytes(w, int8)
    stoks = step_tokens(w)
    torch.cuda.synchronize()

    # ---- device-resident timing ----------------------------------------------------------
    # Every step reads more than the L2 holds, and the largest more than twice that:
    # one event pair around the K timed steps issued back to back (the host enqueues
    # a step in well under the step's device time, so the device never waits), then a
    # second loop of only the decode calls of the same steps for the dominant kernel.
    # Otherwise each step is timed by its own event pair, with the L2 flushed (a
    # write of twice its size) before it, outside the events.
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    per_step = min(sbytes) <= l2 or max(sbytes) < 2 * l2
    flush = torch.empty(2 * l2, dtype=torch.uint8, device="cuda") if per_step else None
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            calls.run(i % T)
    torch.cuda.synchronize()
    K = args.steps
    idx = [(args.warmup + j) % T for j in range(K)]

    def timed(run_one):
        """(device ms, host enqueue ms) of run_one(i) over idx; the device time
        is the sum of per-step event pairs when the L2 is flushed between steps."""
        if not per_step:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            h0 = time.perf_counter()
            a.record(stream)
            for i in idx:
                run_one(i)
            b.record(stream)
            host = (time.perf_counter() - h0) * 1e3
            torch.cuda.synchronize()
            return a.elapsed_time(b), host
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in idx]
        h0 = time.perf_counter()
        with torch.cuda.stream(stream):
            for n, i in enumerate(idx):
                flush.fill_(n & 0xff)
                evs[n][0].record(stream)
                run_one(i)
                evs[n][1].record(stream)
        host = (time.perf_counter() - h0) * 1e3
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs), host

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms, host_ms = timed(calls.run)
        if dist is not None:
            dist.barrier()
        dec_ms, _ = timed(calls.run_decode_only)
        # The same K-step window repeated (at least 5 times and ~60 ms of device
        # time, so the clock sampler sees the GPU under load), then one full lap of
        # the trace: every step once, in order, right after the window.
        reps = []
        n_rep = max(5, min(200, int(np.ceil(60.0 / max(ms, 1e-3)))))
        for _ in range(n_rep):
            reps.append(timed(calls.run)[0])
        idx_window = idx
        idx = [(args.warmup + K + j) % T for j in range(T)]
        lap_ms, _ = timed(calls.run)
        lap_dec_ms, _ = timed(calls.run_decode_only)
        lap_bytes = sum(sbytes[i] for i in idx)
        idx = idx_window
        # the same window with the plain calls (append kernel, then decode)
        plain_ms = timed(plain_calls.run)[0] if plain_calls is not None else None
    bytes_rank = sum(sbytes[i] for i in idx)
    toks_rank = sum(stoks[i] for i in idx)
    launches = sum(calls.launches[i] for i in idx)
    value, ms_max = replica_throughput(bytes_rank, ms, dist)
    peak, peak_kind = load_peak()
    achieved = bytes_rank / (dec_ms * 1e-3) / 1e9
    rep_vals = [replica_throughput(bytes_rank, r, dist)[0] for r in reps]
    lap_value, lap_ms_max = replica_throughput(lap_bytes, lap_ms, dist)
    lap_dec_value, _ = replica_throughput(lap_bytes, lap_dec_ms, dist)

    # ---- end to end through the C ABI with host buffers ------------------------------------------
    e2e = None
    if not args.no_e2e:
        e2e = time_e2e(dw, w, int8, part, algo, args, T, sbytes, stream, dist)

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_max / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": int8 if int8 else "f16", "data": "synthetic",
        "config": {"workload": WORKLOADS[args.workload], "name": args.workload,
                   "partition_size": "library picks (-1)" if part == -1 else part, "algo": args.algo,
                   "l2": ("L2 flushed before every timed step (write of twice the L2 size, "
                          "outside the events)" if per_step else
                          f"inputs larger than L2: every step reads {min(sbytes) / 1e6:.0f}-"
                          f"{max(sbytes) / 1e6:.0f} MB against {l2 / 1e6:.0f} MB of L2, no flush"),
                   "timing": ("one CUDA event pair per step, summed" if per_step else
                              "CUDA events around the K steps issued back to back"),
                   "decode_flags": "PA_DECODE_INPUTS_READY",
                   "step_calls": (("pa_block_copy where a step copies, pa_reshape_and_cache_ex of the "
                                   "admitted prompts" + (" (PA_APPEND_OVERLAP_PREVIOUS)" if pflags else "") +
                                   ", pa_decode_append of the new tokens and the decode "
                                   f"(one kernel in {calls.fused_steps} of {T} steps, plus the merge "
                                   "where it splits)") if calls.fused_steps else
                                  "the workload's own calls (pa_block_copy, pa_reshape_and_cache, pa_decode)"),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "decode_tokens_per_s": toks_rank * world / (ms_max * 1e-3),
        # the same step repeated for 32 layers: attention-only context for a 7B-class model
        "decode_tokens_per_s_32_layers": toks_rank * world / (ms_max * 1e-3) / 32,
        "hbm_frac_nominal_8tbs": value / world / NOMINAL_HBM_GBS,
        "hbm_frac_of_" + peak_kind: value / world / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": traffic_per_launch(args.workload, args.algo, part, bytes_rank / K,
                                                   calls.fused_steps > 0),
                     "traffic_unit": "bytes per decode launch (ncu DRAM read + write, scaled)",
                     "kernel": ("pa_decode_append (new tokens + decode, one kernel) and its merge: the K "
                                "steps' calls issued back to back" if calls.fused_steps else
                                "pa_decode: the K steps' decode calls issued back to back"),
                     "peak_kind": peak_kind},
        "gpu_launches": launches,
        "host_enqueue_ms": host_ms,
        # the K-step window timed again, n times back to back
        "value_repeats": {"median": statistics.median(rep_vals), "min": min(rep_vals),
                          "max": max(rep_vals), "n": len(rep_vals), "unit": "GB/s"},
        # one full lap of the trace (all T steps once, in trace order), timed after the
        # window: the sum of its algorithmic bytes over its device time, whole steps and
        # the decode calls alone
        "value_full_trace": lap_value,
        # the K-step window with the plain calls: pa_reshape_and_cache of all the
        # step's tokens, then pa_decode
        "value_plain_append": (replica_throughput(bytes_rank, plain_ms, dist)[0]
                               if plain_ms is not None else None),
        "decode_full_trace": lap_dec_value,
        "full_trace": {"steps": T, "ms_per_step": lap_ms_max / T, "bytes": lap_bytes * world,
                       "decode_frac_of_" + peak_kind: lap_dec_value / world / peak},
        "clocks": clk.report(),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, int8, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def time_e2e(dw, w, int8, part, algo, args, T, sbytes, stream, dist):
    """Per step: one pinned host -> device copy of the step's inputs (new k/v,
    slots, copy pairs, q, block tables, seq_lens, packed in one buffer), the
    library calls, and one device -> host copy of the decode output; the copies
    of one step overlap the computation of others."""
    import torch
    from paged_kv_cache_395_b200 import pa, runner

    packs, h2d, d2h = [], [], []
    for i in range(T):
        tensors = [t for op in dw.steps[i] for t in op[1:] if isinstance(t, torch.Tensor)]
        outs = [op[-1] for op in dw.steps[i] if op[0] == "decode"]
        ins = [t for t in tensors if not any(t is o for o in outs)]
        offs, n = [], 0
        for t in ins:
            offs.append(n)
            n += (t.numel() * t.element_size() + 255) // 256 * 256
        host = torch.empty(n, dtype=torch.uint8, pin_memory=True)
        for t, o in zip(ins, offs):
            nb = t.numel() * t.element_size()
            host[o:o + nb].copy_(t.contiguous().view(torch.uint8).view(-1).cpu())
        dev = torch.empty(n, dtype=torch.uint8, device="cuda")
        views = {}
        for t, o in zip(ins, offs):
            nb = t.numel() * t.element_size()
            views[id(t)] = dev[o:o + nb].view(t.dtype).view(t.shape)
        out = outs[0]
        host_out = torch.empty(out.numel() * out.element_size(), dtype=torch.uint8, pin_memory=True)
        packs.append((host, dev, views, out, host_out))
        h2d.append(n)
        d2h.append(host_out.numel())
    # library calls that read the staging buffers
    staged = runner.DeviceWorkload.__new__(runner.DeviceWorkload)
    staged.__dict__.update(dw.__dict__)
    staged.steps = {}
    for i in range(T):
        views = packs[i][2]
        staged.steps[i] = [tuple(views.get(id(x), x) if isinstance(x, torch.Tensor) else x
                                 for x in op) for op in dw.steps[i]]
    pflags = pa.PA_APPEND_OVERLAP_PREVIOUS if getattr(w, "appends_overlap_previous", False) else 0
    calls = runner.StepCalls(staged, part, int8, algo, stream, flags=pa.PA_DECODE_INPUTS_READY,
                             fused=args.append == "fused", prompt_flags=pflags)
    K = args.steps
    # Pipelined like a serving loop: step j's inputs are copied in on one copy
    # stream while earlier steps compute on `stream`, and each step's output is
    # copied out on another; events order copy -> compute -> copy per step, and
    # a staging buffer is refilled only after the step that used it T steps
    # earlier has finished with it.
    h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
    ring = 2 * T
    ev_h2d = [torch.cuda.Event() for _ in range(ring)]
    ev_comp = [torch.cuda.Event() for _ in range(ring)]
    ev_d2h = [torch.cuda.Event() for _ in range(ring)]

    def issue(j):
        i = j % T
        host, dev, _, out, host_out = packs[i]
        if j >= T:
            h2d_s.wait_event(ev_comp[(j - T) % ring])
        with torch.cuda.stream(h2d_s):
            dev.copy_(host, non_blocking=True)
        ev_h2d[j % ring].record(h2d_s)
        stream.wait_event(ev_h2d[j % ring])
        if j >= T:
            stream.wait_event(ev_d2h[(j - T) % ring])
        calls.run(i)
        ev_comp[j % ring].record(stream)
        d2h_s.wait_event(ev_comp[j % ring])
        with torch.cuda.stream(d2h_s):
            host_out.copy_(out.view(torch.uint8).view(-1), non_blocking=True)
        ev_d2h[j % ring].record(d2h_s)
        return i

    for j in range(args.warmup):
        issue(j)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(h2d_s)
    stream.wait_event(start)
    d2h_s.wait_event(start)
    nbytes, hb, db = 0, 0, 0
    for j in range(args.warmup, args.warmup + K):
        i = issue(j)
        nbytes += sbytes[i]
        hb += h2d[i]
        db += d2h[i]
    d2h_s.wait_stream(stream)
    d2h_s.wait_stream(h2d_s)
    end.record(d2h_s)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    value, ms = replica_throughput(nbytes, ms, dist)
    return {"value": value, "unit": "GB/s",
            "h2d_bytes_per_step": hb // K, "d2h_bytes_per_step": db // K, "ms_per_step": ms / K}


if __name__ == "__main__":
    sys.exit(main())
