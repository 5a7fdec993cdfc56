"""Pins of the CPU oracle to things other than itself.

Each ``pin_*`` function raises AssertionError on a mismatch.  They check the
oracle against: the pages' printed numbers (KV-size closed form and table,
``golden/kv_size_table.txt``), an independent NumPy brute force on unpaged K/V
(``oracle/dense.py``), a library routine (torch's scaled_dot_product_attention
in fp64), closed forms (one token, equal keys, zero query, one dominant
logit), invariants (physical-block permutation, GQA = MHA on an expanded
cache, partition order), exhaustive format conversions against numpy/torch,
and crafted round-half-even cases for the int8 quantiser.
``test_oracle_mutations`` plants mistakes in the oracle and checks that at
least one pin fails for each.
"""
import os

import numpy as np
import torch

import oracle
from oracle.dense import dense_attention
from paged_kv_cache_395_b200 import workloads as W
from paged_kv_cache_395_b200.block_manager import BlockManager

from .oracle_replay import replay, to_f64

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _close(a, b, tol, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert a.shape == b.shape and np.all(np.isfinite(a)) and err <= tol, \
        f"{what}: max err {err} > {tol}"


# -- format conversions -----------------------------------------------------
def pin_half_exhaustive():
    """Every fp16 bit pattern converts like numpy's float16 -> float64."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), f"fp16 conversion differs at {np.nonzero(~same)[0][:5]}"


def pin_bf16_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_double(int(b)) for b in bits])
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), "bf16 conversion differs"


# -- decode against an independent dense computation -------------------------------
def _dense_of(w, out_step=0):
    op = [o for o in w.steps[out_step] if isinstance(o, W.Decode)][0]
    q = to_f64(op.q, w.dtype)
    ref = np.zeros(q.shape)
    for b in range(q.shape[0]):
        K, V = w.logical[b]
        ref[b] = dense_attention(q[b], to_f64(K, w.dtype), to_f64(V, w.dtype), w.scale, w.group)
    return ref


def pin_tiny_dense():
    w = W.tiny()
    outs, _, _ = replay(w)
    _close(outs[0], _dense_of(w), 1e-12, "tiny vs dense")


RANDOM_CASES = [
    dict(lens=[1, 15, 16, 17, 40], num_q_heads=8, num_kv_heads=2, head_dim=64, dtype="float16"),
    dict(lens=[33, 2, 64], num_q_heads=4, num_kv_heads=4, head_dim=128, dtype="float32"),
    dict(lens=[31, 48, 7], num_q_heads=8, num_kv_heads=1, head_dim=64, dtype="bfloat16"),
    dict(lens=[100, 5], num_q_heads=16, num_kv_heads=2, head_dim=128, dtype="float16", seed=7),
]


def pin_random_dense():
    for case in RANDOM_CASES:
        w = W.random_case(**case)
        outs, _, _ = replay(w)
        _close(outs[0], _dense_of(w), 1e-12, f"random {case}")


def pin_sdpa_library():
    """torch's scaled_dot_product_attention (fp64, CPU) on the logical K/V."""
    for case in RANDOM_CASES[:2]:
        w = W.random_case(**case)
        outs, _, _ = replay(w)
        op = w.steps[0][0]
        q = to_f64(op.q, w.dtype)
        for b in range(q.shape[0]):
            K, V = (torch.from_numpy(to_f64(x, w.dtype)) for x in w.logical[b])
            K = K.permute(1, 0, 2).repeat_interleave(w.group, dim=0)  # [H_q][L][d]
            V = V.permute(1, 0, 2).repeat_interleave(w.group, dim=0)
            qq = torch.from_numpy(q[b]).unsqueeze(1)  # [H_q][1][d]
            ref = torch.nn.functional.scaled_dot_product_attention(qq, K, V, scale=w.scale)
            _close(outs[0][b], ref.squeeze(1).numpy(), 1e-12, "sdpa")


# -- paging invariants --------------------------------------------------------------
def pin_permutation_invariance():
    """Moving physical blocks (and rewriting the tables) changes nothing, bit for bit."""
    w = W.random_case([37, 16, 70], num_q_heads=4, num_kv_heads=2, head_dim=64, seed=3)
    outs, kc, vc = replay(w)
    op = w.steps[0][0]
    rng = np.random.default_rng(11)
    sigma = rng.permutation(w.num_blocks)  # new location of block b is sigma[b]
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[sigma] = kc
    vc2[sigma] = vc
    bt = op.block_tables.copy()
    valid = bt >= 0
    bt[valid] = sigma[bt[valid]]
    out2 = oracle.decode(op.q, kc2, vc2, bt, op.seq_lens, w.scale)
    assert np.array_equal(outs[0], out2), "output depends on physical placement"


def pin_gqa_expand():
    """GQA with head h -> KV head h // G equals MHA over a cache whose KV heads
    are repeated G times, bit for bit."""
    w = W.random_case([29, 50], num_q_heads=8, num_kv_heads=2, head_dim=64, seed=5)
    outs, kc, vc = replay(w)
    op = w.steps[0][0]
    G = w.group
    kc_e = np.repeat(kc, G, axis=1)
    vc_e = np.repeat(vc, G, axis=1)
    out_mha = oracle.decode(op.q, kc_e, vc_e, op.block_tables, op.seq_lens, w.scale)
    assert np.array_equal(outs[0], out_mha), "GQA head mapping differs from h // G"


def _single_seq_cache(K, V, perm_seed=0):
    """Paged cache holding one sequence with the given logical K/V [L][1][d]."""
    L, H, d = K.shape
    nb = -(-L // 16)
    bm = BlockManager(nb + 2, 16, free_order=np.random.default_rng(perm_seed).permutation(nb + 2))
    slots = bm.add_sequence(0, L)
    kc = np.full((nb + 2, H, 16, d), np.nan)
    vc = np.full((nb + 2, H, 16, d), np.nan)
    kc, vc = kc.astype(np.float32), vc.astype(np.float32)
    oracle.reshape_and_cache(K.astype(np.float32), V.astype(np.float32), kc, vc, slots)
    return kc, vc, bm.block_table([0], nb), np.array([L], np.int32)


# -- closed forms -------------------------------------------------------------------
def pin_closed_forms():
    rng = np.random.default_rng(21)
    d = 64
    # one token: softmax weight 1, out = V_0 exactly (the appended token attends to itself)
    K = rng.standard_normal((1, 1, d))
    V = rng.standard_normal((1, 1, d))
    kc, vc, bt, sl = _single_seq_cache(K, V)
    q = rng.standard_normal((1, 1, d))
    out = oracle.decode(q, kc, vc, bt, sl, 0.125)
    assert np.array_equal(out[0, 0], V[0, 0].astype(np.float32).astype(np.float64)), "L=1"
    # all keys equal -> uniform weights -> mean of V
    L = 45
    K = np.repeat(rng.standard_normal((1, 1, d)), L, axis=0)
    V = rng.standard_normal((L, 1, d))
    kc, vc, bt, sl = _single_seq_cache(K, V, 1)
    out = oracle.decode(q, kc, vc, bt, sl, 0.125)
    _close(out[0, 0], V.astype(np.float32).astype(np.float64)[:, 0].mean(0), 1e-14, "equal keys")
    # zero query -> mean of V whatever the keys
    K = rng.standard_normal((L, 1, d))
    kc, vc, bt, sl = _single_seq_cache(K, V, 2)
    out = oracle.decode(np.zeros((1, 1, d)), kc, vc, bt, sl, 0.125)
    _close(out[0, 0], V.astype(np.float32).astype(np.float64)[:, 0].mean(0), 1e-14, "q = 0")
    # one dominant logit: K_t* = 4 e_0, others 0, q = 100 e_0 -> scores 50 vs 0;
    # weight of the rest is (L-1) e^-50 ~ 1e-20
    K = np.zeros((L, 1, d))
    K[17, 0, 0] = 4.0
    kc, vc, bt, sl = _single_seq_cache(K, V, 3)
    qd = np.zeros((1, 1, d))
    qd[0, 0, 0] = 100.0
    out = oracle.decode(qd, kc, vc, bt, sl, 0.125)
    _close(out[0, 0], V.astype(np.float32).astype(np.float64)[17, 0], 1e-15, "dominant")
    # output is a convex combination of the V rows
    K = rng.standard_normal((L, 1, d))
    kc, vc, bt, sl = _single_seq_cache(K, V, 4)
    out = oracle.decode(q, kc, vc, bt, sl, 0.125)[0, 0]
    V64 = V.astype(np.float32).astype(np.float64)[:, 0]
    assert np.all(out <= V64.max(0) + 1e-15) and np.all(out >= V64.min(0) - 1e-15), "hull"
    # seq_len 0 gives zeros
    out = oracle.decode(q, kc, vc, bt, np.array([0], np.int32), 0.125)
    assert np.array_equal(out[0, 0], np.zeros(d)), "L=0"


# -- split form ------------------------------------------------------------------------
def pin_split_merge():
    w = W.random_case([1, 17, 64, 200, 129], num_q_heads=4, num_kv_heads=2, head_dim=64, seed=9)
    outs, kc, vc = replay(w)
    op = w.steps[0][0]
    for P in (16, 32, 48, 512):
        mp = -(-int(op.seq_lens.max()) // P)
        o, lse = oracle.decode_partials(op.q, kc, vc, op.block_tables, op.seq_lens, w.scale, P, mp)
        merged = oracle.merge(o, lse)
        _close(merged, outs[0], 1e-12, f"merge P={P}")
        # partition order does not matter
        rng = np.random.default_rng(P)
        perm = rng.permutation(mp)
        _close(oracle.merge(o[:, :, perm], lse[:, :, perm]), outs[0], 1e-12, "merge order")
        if P == 512:  # one partition: the partial is the output itself
            assert np.array_equal(o[:, :, 0], outs[0]), "single partition"
    # a one-token partition has lse = its score (sum of one exp(0) is 1)
    o, lse = oracle.decode_partials(op.q, kc, vc, op.block_tables, op.seq_lens, w.scale, 16, 13)
    q64 = to_f64(op.q, w.dtype)
    b, h = 0, 3
    blk = op.block_tables[b, 0]
    k0 = kc[blk, h // w.group, 0].astype(np.float64)
    s = w.scale * float(np.dot(q64[b, h], k0))
    assert abs(lse[b, h, 0] - s) <= 1e-12 * max(1.0, abs(s)), "lse of one token"
    assert np.array_equal(o[b, h, 0], vc[blk, h // w.group, 0].astype(np.float64)), "o of one token"
    assert np.all(np.isneginf(lse[b, h, 1:])), "empty partitions"


# -- KV size closed form, the pages' numbers ---------------------------------------------------
def load_kv_golden():
    rows = []
    with open(os.path.join(GOLDEN, "kv_size_table.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            parts = [p.strip() for p in line.split("|")]
            rows.append((parts[0], *[int(x) for x in parts[1:7]], float(parts[7]), parts[8]))
    return rows


def pin_kv_size_golden():
    rows = load_kv_golden()
    assert len(rows) == 7
    for name, layers, kvh, d, E, L, B, expect, src in rows:
        per_tok = oracle.kv_bytes_per_token(layers, kvh, d, E)
        if name.startswith("gqa_ratio"):
            mha = oracle.kv_bytes_per_token(layers, 32, d, E)
            assert per_tok / mha == expect, name
        else:
            assert per_tok * L * B == expect, (name, per_tok * L * B, expect, src)
    # the study's pools are these closed forms times their token counts
    assert oracle.kv_bytes_per_token(1, 8, 128, 2) * 1024 * 8 == 32 * 2 ** 20  # 1/32 of 1 GB
    assert oracle.kv_bytes_per_token(1, 8, 128, 2) * 8192 * 16 == 512 * 2 ** 20  # 1/32 of 16 GB


# -- cache operations ----------------------------------------------------------------------------
def pin_reshape():
    rng = np.random.default_rng(31)
    N, H, d, T = 6, 3, 64, 20
    kc = np.full((N, H, 16, d), np.nan, dtype=np.float16)
    vc = kc.copy()
    slots = rng.choice(N * 16, size=T, replace=False).astype(np.int64)
    slots[[3, 11]] = -1  # padding tokens
    k = rng.standard_normal((T, H, d)).astype(np.float16)
    v = rng.standard_normal((T, H, d)).astype(np.float16)
    oracle.reshape_and_cache(k, v, kc, vc, slots)
    ek = np.full_like(kc, np.nan)
    ev = np.full_like(vc, np.nan)
    m = slots >= 0
    ek[slots[m] // 16, :, slots[m] % 16] = k[m]
    ev[slots[m] // 16, :, slots[m] % 16] = v[m]
    assert np.array_equal(kc.view(np.uint16), ek.view(np.uint16)), "reshape K"
    assert np.array_equal(vc.view(np.uint16), ev.view(np.uint16)), "reshape V"


def pin_block_copy():
    rng = np.random.default_rng(41)
    N, H, d = 8, 2, 64
    kc = rng.standard_normal((N, H, 16, d)).astype(np.float32)
    vc = rng.standard_normal((N, H, 16, d)).astype(np.float32)
    ks = rng.random((N, H)).astype(np.float32)
    vs = rng.random((N, H)).astype(np.float32)
    ek, ev, eks, evs = kc.copy(), vc.copy(), ks.copy(), vs.copy()
    pairs = np.array([[1, 5], [1, 6], [3, 0]], dtype=np.int64)
    for s, t in pairs:
        ek[t], ev[t], eks[t], evs[t] = ek[s], ev[s], eks[s], evs[s]
    oracle.block_copy(kc, vc, pairs, ks, vs)
    for got, exp, n in ((kc, ek, "K"), (vc, ev, "V"), (ks, eks, "k scales"), (vs, evs, "v scales")):
        assert np.array_equal(got.view(np.uint32), exp.view(np.uint32)), f"block copy {n}"


def pin_quantize():
    rng = np.random.default_rng(51)
    N, H, d = 5, 2, 64
    src = (rng.standard_normal((N, H, 16, d)) * 3).astype(np.float16)
    src[2, 1] = 0  # all-zero tile
    q, s = oracle.quantize_int8(src)
    x = src.astype(np.float64)
    deq = q.astype(np.float64) * s.astype(np.float64)[:, :, None, None]
    err = np.abs(deq - x)
    bound = s.astype(np.float64)[:, :, None, None] * (0.5 + 1e-6)
    assert np.all(err <= bound), "dequantisation error above s/2"
    assert s[2, 1] == 0 and not q[2, 1].any(), "zero tile"
    amax = np.abs(x).reshape(N, H, -1).max(-1)
    for n in range(N):
        for h in range(H):
            if amax[n, h] == 0:
                continue
            t = x[n, h].reshape(-1)
            i = int(np.argmax(np.abs(t)))
            assert abs(int(q[n, h].reshape(-1)[i])) == 127, "absmax maps to +-127"
            assert s[n, h] == np.float32(np.float32(amax[n, h]) / np.float32(127)), "scale"
    # crafted tile: absmax 127 gives s = 1, so q = round-half-even(x)
    t = np.zeros((1, 1, 16, d), dtype=np.float32)
    vals = [127.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.49, -126.5, 126.5]
    t.reshape(-1)[: len(vals)] = vals
    q, s = oracle.quantize_int8(t)
    assert s[0, 0] == 1.0
    assert q.reshape(-1)[: len(vals)].tolist() == [127, 0, 2, 2, 0, -2, -2, 3, -126, 126], \
        q.reshape(-1)[: len(vals)].tolist()


# -- appending into an int8 cache -----------------------------------------------------
def pin_append_int8():
    """Appending single tokens into int8 tiles: (1) into an empty tile it equals
    quantising a tile that holds only that token (the pinned quantiser); (2) a
    token that fits the tile's scale leaves every other code and the scale as they
    were; (3) a token that raises the scale re-rounds the other codes within half
    the new scale of their old values, and its own values within half the new
    scale of the inputs; (4) after any sequence of appends every stored value is
    within the sum of the half-scales it went through of the original input."""
    rng = np.random.default_rng(61)
    N, H, d, bs = 6, 2, 64, 16
    # (1) empty tiles: scale 0, codes 0
    kc = np.zeros((N, H, bs, d), dtype=np.int8)
    vc = np.zeros_like(kc)
    ks = np.zeros((N, H), dtype=np.float32)
    vs = np.zeros_like(ks)
    k = (rng.standard_normal((2, H, d)) * 3).astype(np.float16)
    v = (rng.standard_normal((2, H, d)) * 3).astype(np.float16)
    slots = np.array([1 * bs + 5, 4 * bs + 0], dtype=np.int64)
    oracle.append_int8(k, v, kc, vc, ks, vs, slots)
    for i, s in enumerate(slots):
        b, o = divmod(int(s), bs)
        for src, cache, sc in ((k, kc, ks), (v, vc, vs)):
            tile = np.zeros((1, H, bs, d), dtype=np.float16)
            tile[0, :, o] = src[i]
            q, qs = oracle.quantize_int8(tile)
            assert np.array_equal(cache[b], q[0]) and np.array_equal(sc[b], qs[0]), "empty tile"
    # a quantised pool to append into
    src = (rng.standard_normal((N, H, bs, d)) * 2).astype(np.float16)
    kc, ks = oracle.quantize_int8(src)
    vc, vs = oracle.quantize_int8(src[::-1].copy())
    # (2) a small token: nothing else changes
    kc0, ks0 = kc.copy(), ks.copy()
    small = (rng.standard_normal((1, H, d)) * 0.1).astype(np.float16)
    oracle.append_int8(small, small, kc, vc, ks, vs, np.array([2 * bs + 7], dtype=np.int64))
    assert np.array_equal(ks, ks0), "scale changed without need"
    keep = np.ones((N, H, bs), dtype=bool)
    keep[2, :, 7] = False
    assert np.array_equal(kc[keep], kc0[keep]), "codes changed without need"
    x = small.astype(np.float64)[0]
    got = kc[2, :, 7].astype(np.float64) * ks[2].astype(np.float64)[:, None]
    assert np.all(np.abs(got - x) <= ks[2].astype(np.float64)[:, None] * (0.5 + 1e-6)), "small token"
    # (3) a large token raises the scale and re-rounds the rest
    kc0, ks0 = kc.copy(), ks.copy()
    big = (rng.standard_normal((1, H, d)) * 20).astype(np.float16)
    oracle.append_int8(big, big, kc, vc, ks, vs, np.array([3 * bs + 2], dtype=np.int64))
    s_new = ks[3].astype(np.float64)
    amax = np.abs(big.astype(np.float64)[0]).max(-1)
    assert np.all(ks[3] == (amax.astype(np.float32) / np.float32(127))), "raised scale = absmax / 127"
    assert np.all(ks[3] > ks0[3])
    old = kc0[3].astype(np.float64) * ks0[3].astype(np.float64)[:, None, None]
    new = kc[3].astype(np.float64) * s_new[:, None, None]
    others = np.ones((H, bs), dtype=bool)
    others[:, 2] = False
    bound = s_new[:, None, None] * (0.5 + 1e-6)
    assert np.all((np.abs(new - old) <= bound)[others]), "re-rounding moved a value by more than s/2"
    tok = kc[3, :, 2].astype(np.float64) * s_new[:, None]
    assert np.all(np.abs(tok - big.astype(np.float64)[0]) <= s_new[:, None] * (0.5 + 1e-6)), "large token"
    unchanged = np.ones(N, dtype=bool)
    unchanged[[2, 3]] = False
    assert np.array_equal(kc[unchanged], kc0[unchanged]) and np.array_equal(ks[unchanged], ks0[unchanged])
    # (4) a sequence of appends into one tile: error stays within the accumulated half-scales
    kc = np.zeros((1, 1, bs, d), dtype=np.int8)
    ks = np.zeros((1, 1), dtype=np.float32)
    vc, vs = kc.copy(), ks.copy()
    x = np.zeros((bs, d))
    budget = np.zeros(bs)
    for o in range(bs):
        t = (rng.standard_normal((1, 1, d)) * (1 + o)).astype(np.float32)
        oracle.append_int8(t, t, kc, vc, ks, vs, np.array([o], dtype=np.int64))
        x[o] = t[0, 0]
        budget[: o + 1] += float(ks[0, 0]) * 0.5 * (1 + 1e-6)
        err = np.abs(kc[0, 0, : o + 1].astype(np.float64) * float(ks[0, 0]) - x[: o + 1]).max(-1)
        assert np.all(err <= budget[: o + 1]), "accumulated re-rounding error"


# -- 4-bit KV -------------------------------------------------------------------------
def unpack_int4(packed):
    """Independent statement of the 4-bit layout: element 2k is the low four bits
    of byte k, element 2k+1 the high four, each holding q + 8."""
    lo = (packed & 15).astype(np.int64) - 8
    hi = (packed >> 4).astype(np.int64) - 8
    out = np.empty(packed.shape[:-1] + (2 * packed.shape[-1],), dtype=np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def pin_quantize_int4():
    rng = np.random.default_rng(52)
    N, H, d = 5, 2, 64
    src = (rng.standard_normal((N, H, 16, d)) * 2).astype(np.float16)
    src[3, 0] = 0  # all-zero tile
    packed, s = oracle.quantize_int4(src)
    assert packed.shape == (N, H, 16, d // 2) and packed.dtype == np.uint8
    q = unpack_int4(packed)
    assert q.min() >= -7 and q.max() <= 7
    x = src.astype(np.float64)
    deq = q * s.astype(np.float64)[:, :, None, None]
    bound = s.astype(np.float64)[:, :, None, None] * (0.5 + 1e-6)
    assert np.all(np.abs(deq - x) <= bound), "int4 dequantisation error above s/2"
    assert s[3, 0] == 0 and np.all(packed[3, 0] == 0x88), "zero tile: q = 0 stored as 8"
    amax = np.abs(x).reshape(N, H, -1).max(-1)
    for n in range(N):
        for h in range(H):
            if amax[n, h] == 0:
                continue
            i = int(np.argmax(np.abs(x[n, h]).reshape(-1)))
            assert abs(int(q[n, h].reshape(-1)[i])) == 7, "absmax maps to +-7"
            assert s[n, h] == np.float32(np.float32(amax[n, h]) / np.float32(7)), "scale"
    # crafted tile: absmax 7 gives s = 1, so q = round-half-even(x), clamped to +-7
    t = np.zeros((1, 1, 16, d), dtype=np.float32)
    vals = [7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.49, -6.5, 6.5, -7.0]
    t.reshape(-1)[: len(vals)] = vals
    packed, s = oracle.quantize_int4(t)
    assert s[0, 0] == 1.0
    assert unpack_int4(packed).reshape(-1)[: len(vals)].tolist() == [7, 0, 2, 2, 0, -2, -2, 3, -6, 6, -7]


def pin_int4_decode_dense():
    """Decode over packed 4-bit caches equals dense attention on the values the
    NumPy unpacker gives, scaled, in logical order."""
    w = W.random_case([1, 17, 40, 64], num_q_heads=8, num_kv_heads=2, head_dim=64, dtype="float16", seed=8)
    _, kc, vc = replay(w, fill_nan=False)
    k4, ks = oracle.quantize_int4(kc)
    v4, vs = oracle.quantize_int4(vc)
    op = w.steps[0][0]
    out = oracle.decode(op.q, k4, v4, op.block_tables, op.seq_lens, w.scale, ks, vs)
    kd = unpack_int4(k4) * ks.astype(np.float64)[:, :, None, None]
    vd = unpack_int4(v4) * vs.astype(np.float64)[:, :, None, None]
    q = to_f64(op.q, w.dtype)
    for b, L in enumerate(op.seq_lens):
        blocks = op.block_tables[b, : -(-int(L) // 16)]
        K = np.concatenate([kd[blk].transpose(1, 0, 2) for blk in blocks])[:L]  # [L][H_kv][d]
        V = np.concatenate([vd[blk].transpose(1, 0, 2) for blk in blocks])[:L]
        _close(out[b], dense_attention(q[b], K, V, w.scale, w.group), 1e-12, f"int4 b={b}")


# -- multi-query decode (query_len new tokens, causal among them) ---------------------
MULTI_CASES = [
    dict(lens=[2, 17, 40], query_len=2, num_q_heads=8, num_kv_heads=2, head_dim=64, dtype="float16"),
    dict(lens=[5, 33, 16], query_len=5, num_q_heads=4, num_kv_heads=4, head_dim=64, dtype="bfloat16"),
    dict(lens=[3, 70], query_len=3, num_q_heads=16, num_kv_heads=1, head_dim=128, dtype="float32"),
]


def pin_multi_dense():
    """Query token i of a sequence of L tokens equals dense attention over the
    unpaged first L - Q + i + 1 tokens (NumPy brute force, no paging)."""
    for case in MULTI_CASES:
        w = W.random_multi_case(seed=3, **case)
        outs, _, _ = replay(w)
        op = w.steps[0][0]
        q = to_f64(op.q, w.dtype)
        B, Q = q.shape[:2]
        for b in range(B):
            K, V = (to_f64(x, w.dtype) for x in w.logical[b])
            L = int(op.seq_lens[b])
            for i in range(Q):
                n = L - Q + i + 1
                ref = dense_attention(q[b, i], K[:n], V[:n], w.scale, w.group)
                _close(outs[0][b, i], ref, 1e-12, f"multi {case} b={b} i={i}")


def pin_multi_sdpa_causal_mask():
    """torch's scaled_dot_product_attention (fp64) with an explicit mask letting
    query i see keys 0 .. L - Q + i."""
    case = MULTI_CASES[0]
    w = W.random_multi_case(seed=4, **case)
    outs, _, _ = replay(w)
    op = w.steps[0][0]
    q = to_f64(op.q, w.dtype)
    B, Q, Hq, _ = q.shape
    for b in range(B):
        K, V = (torch.from_numpy(to_f64(x, w.dtype)) for x in w.logical[b])
        L = K.shape[0]
        K = K.permute(1, 0, 2).repeat_interleave(w.group, dim=0)  # [H_q][L][d]
        V = V.permute(1, 0, 2).repeat_interleave(w.group, dim=0)
        qq = torch.from_numpy(q[b]).permute(1, 0, 2)  # [H_q][Q][d]
        mask = torch.arange(L)[None, :] <= (L - Q + torch.arange(Q))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, K, V, attn_mask=mask, scale=w.scale)
        _close(outs[0][b], ref.permute(1, 0, 2).numpy(), 1e-12, "multi sdpa")


def pin_multi_single_token_is_decode():
    """Q = 1 gives the single-token decode, bit for bit."""
    w = W.random_multi_case([9, 40], 1, seed=5)
    outs, kc, vc = replay(w)
    op = w.steps[0][0]
    single = oracle.decode(op.q[:, 0], kc, vc, op.block_tables, op.seq_lens, w.scale)
    assert np.array_equal(outs[0][:, 0], single)


ALL_PINS = [pin_half_exhaustive, pin_bf16_exhaustive, pin_tiny_dense, pin_random_dense,
            pin_sdpa_library, pin_permutation_invariance, pin_gqa_expand, pin_closed_forms,
            pin_split_merge, pin_kv_size_golden, pin_reshape, pin_block_copy, pin_quantize,
            pin_multi_dense, pin_multi_sdpa_causal_mask, pin_multi_single_token_is_decode,
            pin_quantize_int4, pin_int4_decode_dense, pin_append_int8]
