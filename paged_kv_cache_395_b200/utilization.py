"""KV cache memory accounting over a decode trace: paged blocks against
contiguous preallocation.

The pages contrast two ways of holding each request's K/V
(chanyi.net.cn/article/49 section 三; lqnn.cn/news/235768 sections 3.1-3.2;
hdu-wiki.cn/courses/inference-kvcache-vllm section 9.1):

* contiguous preallocation reserves one region of the maximum length per
  request, so everything between the request's current length and that
  maximum is reserved but unused;
* paged allocation hands out fixed 16-token blocks on demand, so the only
  unused slots are the tail of each sequence's last block (under 16 per
  sequence), and blocks shared by several sequences are held once.

For every decode step of a workload this module counts the tokens the live
sequences hold and the slots each scheme keeps allocated for them, from the
step's block tables and lengths alone.  Host-side accounting; no GPU.

    python -m paged_kv_cache_395_b200.utilization [--workload ragged] [--max-len N]
"""
from __future__ import annotations

import argparse
import json
from dataclasses import dataclass

import numpy as np

from . import workloads as W


@dataclass
class StepUsage:
    step: int
    sequences: int
    tokens: int            # sum of the live sequences' lengths (logical tokens)
    paged_slots: int       # 16 x distinct physical blocks the step's tables reference
    paged_used: int        # distinct physical slots that hold a token of some sequence
    contiguous_slots: int  # sequences x max_len

    @property
    def paged_utilization(self) -> float:
        """Fraction of the allocated block slots that hold a token."""
        return self.paged_used / self.paged_slots if self.paged_slots else 1.0

    @property
    def sharing(self) -> float:
        """Logical tokens per physical token (above 1 when prefix blocks are shared)."""
        return self.tokens / self.paged_used if self.paged_used else 1.0

    @property
    def contiguous_utilization(self) -> float:
        return self.tokens / self.contiguous_slots if self.contiguous_slots else 1.0


def step_usage(op: W.Decode, block_size: int, max_len: int, step: int = 0) -> StepUsage:
    lens = op.seq_lens.astype(np.int64)
    live = lens > 0
    fill: dict[int, int] = {}  # physical block -> most slots any sequence uses in it
    for b in np.nonzero(live)[0]:
        L = int(lens[b])
        for j in range(-(-L // block_size)):
            blk = int(op.block_tables[b, j])
            fill[blk] = max(fill.get(blk, 0), min(block_size, L - j * block_size))
    return StepUsage(step=step, sequences=int(live.sum()), tokens=int(lens[live].sum()),
                     paged_slots=len(fill) * block_size, paged_used=sum(fill.values()),
                     contiguous_slots=int(live.sum()) * max_len)


def account(w: W.Workload, max_len: int | None = None) -> list[StepUsage]:
    """Per-step usage of every decode in ``w``.  max_len defaults to the longest
    sequence the workload's block tables can hold (what a contiguous scheme would
    have to reserve for every request)."""
    if max_len is None:
        max_len = w.max_blocks_per_seq * w.block_size
    out = []
    for si, ops in enumerate(w.steps):
        for op in ops:
            if isinstance(op, W.Decode):
                out.append(step_usage(op, w.block_size, max_len, si))
    return out


def summary(usage: list[StepUsage]) -> dict:
    tok = sum(u.tokens for u in usage)
    used = sum(u.paged_used for u in usage)
    paged = sum(u.paged_slots for u in usage)
    contig = sum(u.contiguous_slots for u in usage)
    return {
        "steps": len(usage),
        "tokens": tok,
        "paged_utilization": used / paged,
        "contiguous_utilization": tok / contig,
        "paged_waste": 1 - used / paged,
        "contiguous_waste": 1 - tok / contig,
        "sharing": tok / used,
        # sequences that fit in the memory the contiguous scheme needs, paged / contiguous
        "concurrency_gain": contig / paged,
        "paged_utilization_min": min(u.paged_utilization for u in usage),
        "contiguous_utilization_max": max(u.contiguous_utilization for u in usage),
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="ragged", choices=sorted(W.NAMED))
    ap.add_argument("--max-len", type=int, default=None,
                    help="tokens a contiguous scheme reserves per request (default: the table width)")
    args = ap.parse_args(argv)
    w = W.NAMED[args.workload]()
    s = summary(account(w, args.max_len))
    s["workload"] = args.workload
    s["max_len"] = args.max_len or w.max_blocks_per_seq * w.block_size
    print(json.dumps(s))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
