"""Seeded synthetic workloads for paged decode attention.

This module draws inputs and builds the paging structure; it holds none of the
attention arithmetic.  The same arrays feed the GPU path and, in the tests,
the CPU oracle.  Every value is N(0, 1) from ``numpy.random.default_rng(seed)``
drawn in fp64 and rounded to the storage dtype (round to nearest even); the
order of the draws is part of each recipe and is written in its docstring.

A workload is a list of operations in program order:

* ``Reshape(k, v, slot_mapping)``: append tokens to the paged cache;
* ``Copy(pairs)``: copy-on-write block copies (src, dst);
* ``Decode(q, block_tables, seq_lens, max_seq_len)``: one decode of every
  sequence, with ``seq_lens`` counting the token just appended
  (lqnn.cn/news/235768 section 2.2: append, then attend).

``setup`` runs once; ``steps`` is a list of per-step operation lists.  The
named workloads are the five configurations of the paged decode study:
``tiny`` (fp32 oracle check), ``gqa_b8`` (7B-GQA, batch 8, 1024 tokens),
``ragged`` (continuous batching, batch 64, 16..4096 tokens, 128 steps),
``long`` (batch 16, 8192 tokens, split-K) and ``mha_prefix`` (32/32 heads,
1000-token shared prefix with copy-on-write).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .block_manager import BlockManager

BLOCK_SIZE = 16


@dataclass
class Reshape:
    k: np.ndarray             # [T][H_kv][d] storage dtype
    v: np.ndarray
    slot_mapping: np.ndarray  # int64 [T], -1 = padding


@dataclass
class Copy:
    pairs: np.ndarray         # int64 [n][2] (src, dst)


@dataclass
class Decode:
    q: np.ndarray             # [B][H_q][d] storage dtype, or [B][Q][H_q][d] for Q new tokens
    block_tables: np.ndarray  # int32 [B][max_blocks_per_seq]
    seq_lens: np.ndarray      # int32 [B]
    max_seq_len: int


@dataclass
class Workload:
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    num_blocks: int
    dtype: str                # 'float32' | 'float16' | 'bfloat16' (bf16 held as uint16 bits)
    scale: float
    max_blocks_per_seq: int
    partition_size: int       # split-K partition in tokens used for this workload, 0 = one pass
    setup: list = field(default_factory=list)
    steps: list = field(default_factory=list)
    block_size: int = BLOCK_SIZE
    logical: dict | None = None  # seq -> (K [L][H_kv][d], V) for small workloads
    notes: str = ""
    # a step's appends never write a slot that the previous step's decode reads
    # (blocks of finished sequences are reused one step late), so the library may
    # run them while that decode finishes (PA_APPEND_OVERLAP_PREVIOUS)
    appends_overlap_previous: bool = False

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def elem_size(self) -> int:
        return 4 if self.dtype == "float32" else 2

    def storage_dtype(self):
        return np.uint16 if self.dtype == "bfloat16" else np.dtype(self.dtype)

    def decodes(self):
        for ops in [self.setup] + list(self.steps):
            for op in ops:
                if isinstance(op, Decode):
                    yield op


def normal(rng, shape, dtype: str) -> np.ndarray:
    """N(0,1) in fp64 rounded to the storage dtype."""
    x = rng.standard_normal(shape)
    if dtype == "bfloat16":
        import torch
        t = torch.from_numpy(x).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16)
    return x.astype(dtype)


def _normal_tokens(rng, n, H, d, dtype):
    return normal(rng, (n, H, d), dtype), normal(rng, (n, H, d), dtype)


def tiny() -> Workload:
    """Tiny fp32 oracle check: batch 3, post-append lengths {5, 17, 33}, 4 query
    heads / 2 KV heads, head_dim 64, pool of 16 blocks, scale 1/8.

    Draws, seed 0: q [3][4][64]; for each sequence in order its prompt K then V
    ([L-1][2][64] each); then the appended k [3][2][64] and v [3][2][64].
    Seed 1: ``permutation(16)`` is the free-list order, so blocks are handed
    out in the order prompts, then appends, sequence by sequence.  The appended
    tokens land at offset 4 of block 0, offset 0 of logical block 1 and offset 0
    of logical block 2: the append crosses a block boundary twice.
    """
    B, Hq, Hkv, d = 3, 4, 2, 64
    lens = [5, 17, 33]
    rng = np.random.default_rng(0)
    q = normal(rng, (B, Hq, d), "float32")
    prompts = [_normal_tokens(rng, L - 1, Hkv, d, "float32") for L in lens]
    new_k = normal(rng, (B, Hkv, d), "float32")
    new_v = normal(rng, (B, Hkv, d), "float32")
    perm = np.random.default_rng(1).permutation(16)
    bm = BlockManager(16, BLOCK_SIZE, free_order=perm)
    slots = [bm.add_sequence(b, lens[b] - 1) for b in range(B)]
    pk = np.concatenate([p[0] for p in prompts])
    pv = np.concatenate([p[1] for p in prompts])
    setup = [Reshape(pk, pv, np.concatenate(slots))]
    new_slots = np.array([bm.append_slot(b)[0] for b in range(B)], dtype=np.int64)
    mb = 3
    step = [Reshape(new_k, new_v, new_slots),
            Decode(q, bm.block_table(range(B), mb), np.array(lens, np.int32), max(lens))]
    logical = {b: (np.concatenate([prompts[b][0], new_k[b:b + 1]]),
                   np.concatenate([prompts[b][1], new_v[b:b + 1]])) for b in range(B)}
    return Workload("tiny", Hq, Hkv, d, 16, "float32", 1.0 / 8.0, mb, 0, setup, [step],
                    logical=logical)


def gqa_b8(dtype: str = "float16") -> Workload:
    """7B-GQA decode: 32 query / 8 KV heads, head_dim 128, batch 8, every
    sequence 1024 tokens, pool of 512 blocks.

    Draws, seed 2: ``permutation(512)`` (free-list order), then for each
    sequence K [1024][8][128] then V, then q [8][32][128].  The whole cache is
    written by one append of all 8192 tokens."""
    B, Hq, Hkv, d, L, N = 8, 32, 8, 128, 1024, 512
    rng = np.random.default_rng(2)
    bm = BlockManager(N, BLOCK_SIZE, free_order=rng.permutation(N))
    ks, vs, slots = [], [], []
    for b in range(B):
        k, v = _normal_tokens(rng, L, Hkv, d, dtype)
        ks.append(k)
        vs.append(v)
        slots.append(bm.add_sequence(b, L))
    q = normal(rng, (B, Hq, d), dtype)
    mb = L // BLOCK_SIZE
    setup = [Reshape(np.concatenate(ks), np.concatenate(vs), np.concatenate(slots))]
    step = [Decode(q, bm.block_table(range(B), mb), np.full(B, L, np.int32), L)]
    return Workload("gqa_b8", Hq, Hkv, d, N, dtype, 1.0 / np.sqrt(d), mb, 256, setup, [step])


def ragged(num_steps: int = 128, dtype: str = "float16", batch: int = 64,
           finish_p: float = 0.02) -> Workload:
    """Continuous-batching ragged decode: 32/8 heads, head_dim 128, batch 64.

    Draws, seed 3: ``permutation(16896)`` (free-list order); initial cached
    lengths ``integers(16, 4097, size=64)``; for each sequence its K then V.
    Then per step: k [64][8][128], v, q [64][32][128]; every sequence appends
    one token (one append op that also carries the prompts of sequences
    admitted at the end of the previous step) and is decoded with length
    cached + 1; then ``random(64) < 0.02`` marks finished sequences, which free
    their blocks and are replaced, in batch order, by new sequences of
    ``integers(16, 513)`` tokens whose K then V are drawn at once.
    Pool: 64 x ceil(4224 / 16) = 16896 blocks, enough for the worst case.

    Blocks freed by the sequences that finish after step i's decode go back on
    the free list just before the admissions of step i + 1 (deferred reuse), so
    neither step i + 1's token appends nor the prompts admitted with them (both
    written by step i + 1's append) land in a block step i's decode reads."""
    B, Hq, Hkv, d = batch, 32, 8, 128
    max_len = 4096 + num_steps
    mb = -(-max_len // BLOCK_SIZE)
    N = B * mb
    rng = np.random.default_rng(3)
    bm = BlockManager(N, BLOCK_SIZE, free_order=rng.permutation(N))
    init = rng.integers(16, 4097, size=B)
    ks, vs, slots = [], [], []
    for b in range(B):
        k, v = _normal_tokens(rng, int(init[b]), Hkv, d, dtype)
        ks.append(k)
        vs.append(v)
        slots.append(bm.add_sequence(b, int(init[b])))
    setup = [Reshape(np.concatenate(ks), np.concatenate(vs), np.concatenate(slots))]
    seq_ids = list(range(B))
    next_id = B
    pending = ([], [], [])  # admitted prompts not yet written
    steps = []
    for _ in range(num_steps):
        k_new = normal(rng, (B, Hkv, d), dtype)
        v_new = normal(rng, (B, Hkv, d), dtype)
        q = normal(rng, (B, Hq, d), dtype)
        new_slots = np.array([bm.append_slot(s)[0] for s in seq_ids], dtype=np.int64)
        k_all = np.concatenate(pending[0] + [k_new])
        v_all = np.concatenate(pending[1] + [v_new])
        s_all = np.concatenate(pending[2] + [new_slots])
        lens = np.array([bm.lens[s] for s in seq_ids], dtype=np.int32)
        steps.append([Reshape(k_all, v_all, s_all),
                      Decode(q, bm.block_table(seq_ids, mb), lens, int(lens.max()))])
        finished = rng.random(B) < finish_p
        pending = ([], [], [])
        bm.release_deferred()  # freed after the previous step's decode
        for i in np.nonzero(finished)[0]:
            bm.free_sequence(seq_ids[i], defer=True)
            L = int(rng.integers(16, 513))
            k, v = _normal_tokens(rng, L, Hkv, d, dtype)
            seq_ids[i] = next_id
            pending[0].append(k)
            pending[1].append(v)
            pending[2].append(bm.add_sequence(next_id, L))
            next_id += 1
    return Workload("ragged", Hq, Hkv, d, N, dtype, 1.0 / np.sqrt(d), mb, 256, setup, steps,
                    appends_overlap_previous=True)


def long(dtype: str = "float16", batch: int = 16, seq_len: int = 8192) -> Workload:
    """Long context: 32/8 heads, head_dim 128, batch 16, every sequence 8192
    tokens, split-K partitions of 512 tokens; pool of 8192 blocks.

    Draws, seed 5: ``permutation(8192)`` (free-list order), then for each
    sequence K [8192][8][128] then V, then q [16][32][128].  The int8 run
    quantises this fp16 cache (one scale per (block, KV head) for K and for V)."""
    B, Hq, Hkv, d, L = batch, 32, 8, 128, seq_len
    mb = L // BLOCK_SIZE
    N = B * mb
    rng = np.random.default_rng(5)
    bm = BlockManager(N, BLOCK_SIZE, free_order=rng.permutation(N))
    ks, vs, slots = [], [], []
    for b in range(B):
        k, v = _normal_tokens(rng, L, Hkv, d, dtype)
        ks.append(k)
        vs.append(v)
        slots.append(bm.add_sequence(b, L))
    q = normal(rng, (B, Hq, d), dtype)
    setup = [Reshape(np.concatenate(ks), np.concatenate(vs), np.concatenate(slots))]
    step = [Decode(q, bm.block_table(range(B), mb), np.full(B, L, np.int32), L)]
    return Workload("long", Hq, Hkv, d, N, dtype, 1.0 / np.sqrt(d), mb, 512, setup, [step])


def uniform(name: str, seed: int, batch: int, seq_len: int, num_q_heads: int, num_kv_heads: int,
            head_dim: int, dtype: str = "float16") -> Workload:
    """A batch of equal-length sequences in a shuffled pool, the cache written by
    one append of all tokens.  Draws: ``permutation(N)`` (free-list order), then
    for each sequence K [L][H_kv][d] then V, then q [B][H_q][d]."""
    B, L = batch, seq_len
    mb = -(-L // BLOCK_SIZE)
    N = B * mb
    rng = np.random.default_rng(seed)
    bm = BlockManager(N, BLOCK_SIZE, free_order=rng.permutation(N))
    ks, vs, slots = [], [], []
    for b in range(B):
        k, v = _normal_tokens(rng, L, num_kv_heads, head_dim, dtype)
        ks.append(k)
        vs.append(v)
        slots.append(bm.add_sequence(b, L))
    q = normal(rng, (B, num_q_heads, head_dim), dtype)
    setup = [Reshape(np.concatenate(ks), np.concatenate(vs), np.concatenate(slots))]
    step = [Decode(q, bm.block_table(range(B), mb), np.full(B, L, np.int32), L)]
    return Workload(name, num_q_heads, num_kv_heads, head_dim, N, dtype, 1.0 / np.sqrt(head_dim), mb, -1,
                    setup, [step])


def mqa() -> Workload:
    """MQA decode: 32 query heads sharing one KV head, head_dim 128, fp16,
    batch 128, every sequence 4096 tokens (seed 6)."""
    return uniform("mqa", 6, 128, 4096, 32, 1, 128)


def mqa64() -> Workload:
    """Groups of 64: 64 query heads sharing one KV head, head_dim 128, fp16, batch 128,
    every sequence 4096 tokens (seed 12)."""
    return uniform("mqa64", 12, 128, 4096, 64, 1, 128)


def d256() -> Workload:
    """head_dim 256 decode: 16 query / 8 KV heads, fp16, batch 16, every
    sequence 4096 tokens (seed 7)."""
    return uniform("d256", 7, 16, 4096, 16, 8, 256)


def specdec(num_steps: int = 16, query_len: int = 2, dtype: str = "float16", batch: int = 64) -> Workload:
    """Speculative-decoding verification: 7B-GQA heads (32 q / 8 KV, head_dim
    128), batch 64, initial lengths U[512, 4096], and per step every sequence
    appends query_len tokens and decodes them together (causal among them).

    Draws, seed 8: ``permutation(N)`` (free-list order); initial lengths
    ``integers(512, 4097, size=64)``; for each sequence its K then V; then per
    step k, v [64 * Q][8][128] and q [64][Q][32][128]."""
    B, Hq, Hkv, d, Q = batch, 32, 8, 128, query_len
    max_len = 4096 + num_steps * Q
    mb = -(-max_len // BLOCK_SIZE)
    N = B * mb
    rng = np.random.default_rng(8)
    bm = BlockManager(N, BLOCK_SIZE, free_order=rng.permutation(N))
    init = rng.integers(512, 4097, size=B)
    ks, vs, slots = [], [], []
    for b in range(B):
        k, v = _normal_tokens(rng, int(init[b]), Hkv, d, dtype)
        ks.append(k)
        vs.append(v)
        slots.append(bm.add_sequence(b, int(init[b])))
    setup = [Reshape(np.concatenate(ks), np.concatenate(vs), np.concatenate(slots))]
    steps = []
    for _ in range(num_steps):
        k_new = normal(rng, (B * Q, Hkv, d), dtype)
        v_new = normal(rng, (B * Q, Hkv, d), dtype)
        q = normal(rng, (B, Q, Hq, d), dtype)
        new_slots = np.array([bm.append_slot(b)[0] for b in range(B) for _ in range(Q)], dtype=np.int64)
        lens = np.array([bm.lens[b] for b in range(B)], dtype=np.int32)
        steps.append([Reshape(k_new, v_new, new_slots),
                      Decode(q, bm.block_table(range(B), mb), lens, int(lens.max()))])
    # no sequence ends: every appended slot lies past the lengths of every earlier decode
    return Workload("specdec", Hq, Hkv, d, N, dtype, 1.0 / np.sqrt(d), mb, -1, setup, steps,
                    appends_overlap_previous=True)


def mha_prefix(dtype: str = "float16") -> Workload:
    """MHA with prefix sharing: 32 query / 32 KV heads, head_dim 128, batch 16.

    Draws, seed 4: ``permutation(2048)`` (free-list order); prefix K then V
    [1000][32][128]; suffix lengths ``integers(64, 1049, size=16)``; for each
    sequence its suffix K then V; then q [16][32][128].

    Sequence 0 holds the 1000-token prefix (62 full blocks + 8 tokens of a
    63rd); sequences 1..15 fork from it (reference count 16 on each prefix
    block).  Each sequence then appends its suffix; its first append finds the
    shared partial block and copies it (copy-on-write) unless it is the last
    sharer, so 15 block copies precede the suffix writes."""
    B, H, d, P = 16, 32, 128, 1000
    N = 2048
    rng = np.random.default_rng(4)
    bm = BlockManager(N, BLOCK_SIZE, free_order=rng.permutation(N))
    pk, pv = _normal_tokens(rng, P, H, d, dtype)
    prefix_slots = bm.add_sequence(0, P)
    for b in range(1, B):
        bm.fork(0, b)
    suffix = rng.integers(64, 1049, size=B)
    ks, vs, slots, pairs = [], [], [], []
    for b in range(B):
        k, v = _normal_tokens(rng, int(suffix[b]), H, d, dtype)
        ks.append(k)
        vs.append(v)
        for _ in range(int(suffix[b])):
            s, cow = bm.append_slot(b)
            slots.append(s)
            if cow is not None:
                pairs.append(cow)
    q = normal(rng, (B, H, d), dtype)
    lens = np.array([bm.lens[b] for b in range(B)], dtype=np.int32)
    mb = int(max(len(t) for t in bm.tables.values()))
    setup = [Reshape(pk, pv, prefix_slots)]
    step = [Copy(np.array(pairs, dtype=np.int64).reshape(-1, 2)),
            Reshape(np.concatenate(ks), np.concatenate(vs), np.array(slots, dtype=np.int64)),
            Decode(q, bm.block_table(range(B), mb), lens, int(lens.max()))]
    w = Workload("mha_prefix", H, H, d, N, dtype, 1.0 / np.sqrt(d), mb, 0, setup, [step])
    w.notes = f"cow_copies={len(pairs)} unique_blocks={bm.used_blocks()}"
    return w


def random_case(lens, num_q_heads=4, num_kv_heads=2, head_dim=64, dtype="float16", seed=0,
                num_blocks=None, extra_blocks=3, partition_size=0, q_scale=1.0) -> Workload:
    """Small seeded case with arbitrary lengths (edge cases, ragged tails).

    Draws: ``permutation(num_blocks)``, then per sequence K then V, then q
    (multiplied by ``q_scale`` before rounding, to sharpen the softmax)."""
    lens = [int(x) for x in lens]
    B = len(lens)
    need = sum(-(-L // BLOCK_SIZE) for L in lens)
    N = num_blocks if num_blocks is not None else need + extra_blocks
    rng = np.random.default_rng(seed)
    bm = BlockManager(N, BLOCK_SIZE, free_order=rng.permutation(N))
    ks, vs, slots, logical = [], [], [], {}
    for b, L in enumerate(lens):
        k, v = _normal_tokens(rng, L, num_kv_heads, head_dim, dtype)
        ks.append(k)
        vs.append(v)
        slots.append(bm.add_sequence(b, L))
        logical[b] = (k, v)
    x = rng.standard_normal((B, num_q_heads, head_dim)) * q_scale
    if dtype == "bfloat16":
        import torch
        q = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    else:
        q = x.astype(dtype)
    mb = max(1, max((len(bm.tables[b]) for b in range(B)), default=1))
    setup = []
    if B and sum(lens):
        setup = [Reshape(np.concatenate(ks), np.concatenate(vs), np.concatenate(slots))]
    step = [Decode(q, bm.block_table(range(B), mb), np.array(lens, np.int32),
                   max(lens, default=0))]
    return Workload(f"random{B}", num_q_heads, num_kv_heads, head_dim, N, dtype,
                    1.0 / np.sqrt(head_dim), mb, partition_size, setup, [step], logical=logical)


def random_multi_case(lens, query_len, num_q_heads=4, num_kv_heads=2, head_dim=64, dtype="float16",
                      seed=0, extra_blocks=3) -> Workload:
    """random_case with query_len new tokens per sequence: the cache holds all
    ``lens[b]`` tokens (the last query_len of them are the new ones) and q is
    [B][query_len][H_q][d].  Draws: as random_case, then q [B][Q][H_q][d]."""
    w = random_case(lens, num_q_heads, num_kv_heads, head_dim, dtype, seed, extra_blocks=extra_blocks)
    rng = np.random.default_rng(seed + 1000)
    q = normal(rng, (len(lens), query_len, num_q_heads, head_dim), dtype)
    op = w.steps[0][0]
    w.steps = [[Decode(q, op.block_tables, op.seq_lens, op.max_seq_len)]]
    w.name = f"multi{len(lens)}x{query_len}"
    return w


NAMED = {"tiny": tiny, "gqa_b8": gqa_b8, "ragged": ragged, "long": long,
         "mha_prefix": mha_prefix, "mqa": mqa, "mqa64": mqa64, "d256": d256, "specdec": specdec}


def decode_kv_bytes(op: Decode, w: Workload, kv_elem: float | None = None) -> int:
    """Algorithmic bytes of one decode: every K and V element of every logical
    token once, int8 scales once per (block, KV head) read, q in, out out,
    table entries read and seq_lens."""
    E = w.elem_size if kv_elem is None else kv_elem  # int8 1, 4-bit 0.5
    L = op.seq_lens.astype(np.int64)
    L = L[L > 0]
    nblk = -(-L // w.block_size)
    B = op.seq_lens.shape[0]
    kv = int(int(L.sum()) * w.num_kv_heads * w.head_dim * 2 * E)
    scales = int(nblk.sum()) * w.num_kv_heads * 2 * 4 if kv_elem is not None and kv_elem <= 1 else 0
    qo = int(op.q.size) * 2 * w.elem_size  # q in, out out (Q query tokens each)
    return int(kv + scales + qo + int(nblk.sum()) * 4 + B * 4)
