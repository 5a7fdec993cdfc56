"""Host-side accounting behind the bench line: the algorithmic bytes of a decode
(the roofline numerator) and the ncu traffic record that scales them.  No GPU."""
import numpy as np
import pytest

import bench
from paged_kv_cache_395_b200 import workloads as W


def _by_hand(lens, hq, hkv, d, elem, kv_elem=None):
    """Count the bytes one decode must move, element by element."""
    E = elem if kv_elem is None else kv_elem
    total = 0
    for L in lens:
        if L <= 0:
            continue
        blocks = -(-L // 16)
        total += L * hkv * d * 2 * E  # every K and V element of every token once
        if kv_elem is not None:
            total += blocks * hkv * 2 * 4  # one fp32 scale per (block, KV head), K and V
        total += blocks * 4  # table entries read
    total += len(lens) * hq * d * elem * 2  # q in, out out
    total += len(lens) * 4  # seq_lens
    return int(total)


@pytest.mark.parametrize("lens,hq,hkv,d,dtype", [([5, 17, 33], 4, 2, 64, "float32"),
                                                ([1, 16, 4000, 0], 32, 8, 128, "float16"),
                                                ([300, 77], 64, 1, 128, "bfloat16")])
def test_decode_bytes_match_a_count_by_hand(lens, hq, hkv, d, dtype):
    w = W.random_case(lens, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, dtype=dtype, seed=3)
    op = w.steps[0][-1]
    elem = np.dtype(np.float32 if dtype == "float32" else np.float16).itemsize
    assert W.decode_kv_bytes(op, w) == _by_hand(lens, hq, hkv, d, elem)
    for kv_elem in (1, 0.5):  # int8, 4-bit pools
        assert W.decode_kv_bytes(op, w, kv_elem) == _by_hand(lens, hq, hkv, d, elem, kv_elem)


def test_kv_part_is_the_pages_per_token_size():
    """The K/V part of a decode is seq_len x (2 * H_kv * d * bytes) per layer: the
    pages' 128 KB per token for 32 layers x 8 KV heads x 128 x fp16 is 4 KB per layer."""
    w = W.random_case([1000], num_q_heads=32, num_kv_heads=8, head_dim=128, dtype="float16", seed=1)
    op = w.steps[0][-1]
    rest = _by_hand([1000], 32, 8, 128, 2) - 1000 * 8 * 128 * 2 * 2
    assert W.decode_kv_bytes(op, w) - rest == 1000 * 131072 // 32


def test_ragged_trace_steps_exceed_l2():
    """The headline trace is timed without L2 flushes because every step reads
    more than the B200's L2 (126 MiB) and the largest more than twice that."""
    w, int8, _ = bench.make_workload("ragged")
    b = bench.step_bytes(w, int8)
    l2 = 126 * 2**20
    assert min(b) > l2 and max(b) > 2 * l2


def test_code_hash_ignores_comments_and_layout(tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    a.write_text("int f(int x) {\n  // one\n  return x + 1; /* two */\n}\n")
    b.write_text("int f(int x) { /* changed\n comment */ return x + 1;   // other\n}")
    assert bench.code_hash([str(a)]) == bench.code_hash([str(b)])
    b.write_text("int f(int x) { return x + 2; }")
    assert bench.code_hash([str(a)]) != bench.code_hash([str(b)])
    # every listed source counts
    assert bench.code_hash([str(a), str(a)]) != bench.code_hash([str(a), str(b)])


def test_traffic_is_reported_only_for_the_captured_kernel(monkeypatch):
    rec = dict(bench.NCU_TRAFFIC["ragged"])
    monkeypatch.setitem(bench.NCU_TRAFFIC, "ragged", rec)
    monkeypatch.setattr(bench, "code_hash", lambda paths: rec["code"])
    t = bench.traffic_per_launch("ragged", "auto", -1, 2.0e8)
    assert t == pytest.approx(rec["per_alg_byte"] * 2.0e8)
    assert 1.0 <= rec["per_alg_byte"] < 1.1  # the capture read about the algorithmic bytes
    # another code, the CUDA-core family, a fixed partition or another workload: no figure
    monkeypatch.setattr(bench, "code_hash", lambda paths: "0" * 16)
    assert bench.traffic_per_launch("ragged", "auto", -1, 2.0e8) is None
    monkeypatch.setattr(bench, "code_hash", lambda paths: rec["code"])
    assert bench.traffic_per_launch("ragged", "simt", -1, 2.0e8) is None
    assert bench.traffic_per_launch("ragged", "auto", 512, 2.0e8) is None
    assert bench.traffic_per_launch("long", "auto", -1, 2.0e8) is None


@pytest.mark.parametrize("int8", [False, "i8", "i4"])
def test_cpu_baseline_reports_its_sample(int8):
    """The oracle leg of the bench line: GB/s over whole decode steps on all host
    threads, a one-thread figure on a named sample, and the CPU model."""
    w = W.random_case([40, 300, 17, 64, 5], num_q_heads=8, num_kv_heads=2, head_dim=128, dtype="float16",
                      seed=4)
    cb = bench.cpu_baseline(w, int8, 0.01)
    assert cb["kind"] == "oracle" and cb["unit"] == "GB/s" and cb["cores"] >= 1
    assert cb["value"] > 0 and cb["value_1_thread"] > 0 and cb["tokens_per_s"] > 0
    assert "1 whole decode step" in cb["sample"] and "first 4 sequences" in cb["sample_1_thread"]
    assert isinstance(cb["cpu_model"], str) and cb["cpu_model"]
