"""The five synthetic QSA workloads: shapes, positions and seeds only.

Each workload is a list of steps.  A step appends tokens [len_before, len_after)
to every sequence (their K/V, indexer keys already written by the caller), pools
the 4-token blocks those tokens complete, and runs one query per listed
(sequence, position).  Query ids address the generator streams, so a query's
inputs are the same wherever it is regenerated.
"""

from dataclasses import dataclass, field
from typing import List


@dataclass
class Step:
    len_before: List[int]   # per sequence: tokens present before this step
    len_after: List[int]    # per sequence: tokens present after this step
    q_seq: List[int]        # per query: sequence index
    q_pos: List[int]        # per query: 0-based token position
    query_ids: List[int]    # per query: generator id


@dataclass
class Workload:
    name: str
    cid: int
    mode: str               # "decode" or "prefill"
    batch: int
    n_q_heads: int
    n_kv_heads: int
    kv_capacity: int
    steps: List[Step] = field(default_factory=list)
    head_dim: int = 128
    n_idx_heads: int = 4
    idx_dim: int = 64
    block_size: int = 4
    top_k: int = 512

    @property
    def seed(self):
        return 1000 + self.cid

    @property
    def max_blocks(self):
        return self.kv_capacity // self.block_size

    def n_queries(self):
        return sum(len(s.q_pos) for s in self.steps)


def _decode_step(batch, t, qid0):
    return Step([t] * batch, [t + 1] * batch, list(range(batch)), [t] * batch,
                list(range(qid0, qid0 + batch)))


def _prefill_step(t0, n_q):
    return Step([t0], [t0 + n_q], [0] * n_q, list(range(t0, t0 + n_q)), list(range(n_q)))


def decode_8k():
    """1 sequence, 1 query at position 8191 (2,048 complete blocks), 8 query / 1 KV head."""
    return Workload("decode_8k_b1", 0, "decode", 1, 8, 1, 8192, [_decode_step(1, 8191, 0)])


def decode_64k():
    """16 sequences at context 65,536 (16,384 blocks), 32 query / 4 KV heads."""
    return Workload("decode_64k_b16", 1, "decode", 16, 32, 4, 65536, [_decode_step(16, 65535, 0)])


def prefill_128k():
    """4,096 queries at positions 126,976..131,071 of a 131,072-token sequence."""
    return Workload("prefill_4096_at_128k", 2, "prefill", 1, 32, 4, 131072,
                    [_prefill_step(126976, 4096)])


def decode_1m():
    """4 sequences at ~1M context; step 1 at t=1,048,574, step 2 completes block 262,143."""
    return Workload("decode_1m_b4", 3, "decode", 4, 32, 4, 1 << 20,
                    [_decode_step(4, (1 << 20) - 2, 0), _decode_step(4, (1 << 20) - 1, 4)])


def prefill_1m():
    """8,192 queries at positions 1,040,384..1,048,575 of a 1,048,576-token sequence."""
    return Workload("prefill_8192_at_1m", 4, "prefill", 1, 32, 4, 1 << 20,
                    [_prefill_step((1 << 20) - 8192, 8192)])


ALL = [decode_8k, decode_64k, prefill_128k, decode_1m, prefill_1m]


def by_id(cid):
    return ALL[cid]()
