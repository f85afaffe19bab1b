"""Seeded synthetic workloads: shapes, lengths, block tables and input tensors.

This module holds no quantization or attention arithmetic; it only draws inputs.
Both the CUDA path (tests, bench) and the CPU oracle (tests) take their inputs
from here.  The five named workloads are the synthetic stand-ins for the pages'
measurements (long agent contexts up to 64K tokens; the engine's own benchmark
text is not available): per sequence, the cache holds L_b tokens, the last
n_append_b of which are appended in the measured step, and n_q_b query tokens
(1 = decode, > 1 = draft verification) attend to it.

Data law (all workloads): K, V ~ N(0, 1) drawn in fp32 from torch.Generator seeded
with 0, K channels 0..3 of every head multiplied by 10 (outlier channels), then
cast to the workload dtype; q ~ N(0, 1).  Draw order: shared-prefix K then V,
then for each sequence its own K then V, then q.  Lengths and block permutations
come from numpy.random.default_rng(1).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

PAGE = 16


@dataclass
class Workload:
    name: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq_lens: list            # L_b: tokens in the cache after the step (incl. query tokens)
    n_q: list                 # query tokens per sequence
    n_append: list            # tokens appended in the measured step (the last n_append_b of L_b)
    shared_prefix: int = 0    # tokens (multiple of 16) shared by every sequence's block table
    dtype: str = "bf16"       # "bf16" or "f32"
    shuffle: bool = True      # physical block ids are a random permutation
    note: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def n_seqs(self) -> int:
        return len(self.seq_lens)

    @property
    def total_q(self) -> int:
        return int(sum(self.n_q))

    @property
    def max_q(self) -> int:
        return int(max(self.n_q))

    @property
    def max_seq_len(self) -> int:
        return int(max(self.seq_lens))

    def max_blocks(self) -> int:
        return (self.max_seq_len + PAGE - 1) // PAGE

    def kv_bytes_logical(self, bytes_per_token_head: int) -> int:
        return int(sum(self.seq_lens)) * self.n_kv_heads * bytes_per_token_head

    def kv_bytes_unique(self, bytes_per_token_head: int) -> int:
        own = int(sum(L - self.shared_prefix for L in self.seq_lens))
        return (self.shared_prefix + own) * self.n_kv_heads * bytes_per_token_head


# ---- the five workloads -------------------------------------------------------
def tiny(L=4096) -> Workload:
    return Workload("tiny_decode_4k", 8, 2, 128, [L], [1], [1], dtype="f32", shuffle=False,
                    note="batch 1, 8 q / 2 kv heads, D 128, 4096-token history, 1 query token, fp32 K/V/q, "
                         "contiguous block table")


def long_decode(L=65536) -> Workload:
    return Workload("long_decode_64k", 32, 8, 128, [L], [1], [1],
                    note="batch 1, 32 q / 8 kv heads (GQA 4), D 128, 65536-token history, 1 bf16 query token, "
                         "shuffled 16-token blocks")


def shared_prefix(n_sessions=8, prefix=32768, suffix_lo=1024, suffix_hi=8192) -> Workload:
    assert prefix % PAGE == 0
    rng = np.random.default_rng(1)
    suf = rng.integers(suffix_lo, suffix_hi + 1, n_sessions).tolist()
    return Workload("shared_prefix_8x32k", 32, 8, 128, [prefix + s for s in suf], [1] * n_sessions,
                    [1] * n_sessions, shared_prefix=prefix,
                    note=f"{n_sessions} sessions, 32 q / 8 kv heads, D 128, a {prefix}-token prefix on the same "
                         f"physical blocks in every block table + private suffix U[{suffix_lo}, {suffix_hi}]")


def verify(history=65536, drafts=8) -> Workload:
    return Workload("verify8_64k", 32, 8, 128, [history + drafts], [drafts], [drafts],
                    note=f"batch 1, 32 q / 8 kv heads, D 128, {history}-token history + {drafts} draft tokens "
                         "appended and verified in one launch, causal among the drafts")


def mixed_append(n_sessions=32, lo=1024, hi=65536, append=512) -> Workload:
    rng = np.random.default_rng(1)
    h = np.floor(np.exp(rng.uniform(math.log(lo), math.log(hi), n_sessions))).astype(int).tolist()
    return Workload("mixed_append_32x", 16, 4, 256, [x + append for x in h], [1] * n_sessions,
                    [append] * n_sessions,
                    note=f"{n_sessions} sessions, 16 q / 4 kv heads, D 256, history log-uniform [{lo}, {hi}], "
                         f"{append} new bf16 tokens appended per session, then one decode step per session",
                    extra={"history": h})


FULL = {"tiny": tiny, "long": long_decode, "prefix": shared_prefix, "verify": verify, "mixed": mixed_append}


def reduced(name: str) -> Workload:
    """Small versions of the five workloads: several chunks and a ragged tail, cheap
    enough for the oracle in seconds."""
    if name == "tiny":
        return tiny(L=1000)
    if name == "long":
        return long_decode(L=3001)
    if name == "prefix":
        return shared_prefix(n_sessions=3, prefix=1008, suffix_lo=100, suffix_hi=600)
    if name == "verify":
        return verify(history=1500, drafts=8)
    if name == "mixed":
        return mixed_append(n_sessions=4, lo=100, hi=2000, append=50)
    raise KeyError(name)


# ---- block tables -----------------------------------------------------------------
def block_tables(w: Workload, copies: int = 1, seed: int = 1):
    """Physical block ids for every sequence, for `copies` independent copies of the
    whole workload (copy c's tables point at disjoint blocks; used to rotate the
    caches read by successive timed steps).

    Returns (tables int32 [copies, n_seqs, max_blocks], n_blocks).  The shared
    prefix's blocks appear in every sequence's table of the same copy."""
    mb = w.max_blocks()
    pre = w.shared_prefix // PAGE
    own = [(L + PAGE - 1) // PAGE - pre for L in w.seq_lens]
    per_copy = pre + sum(own)
    n_blocks = per_copy * copies
    ids = np.arange(n_blocks, dtype=np.int64)
    if w.shuffle:
        ids = np.random.default_rng(seed).permutation(n_blocks)
    tabs = np.zeros((copies, w.n_seqs, mb), np.int32)
    for c in range(copies):
        base = c * per_copy
        pre_ids = ids[base: base + pre]
        nxt = base + pre
        for b in range(w.n_seqs):
            tabs[c, b, :pre] = pre_ids
            tabs[c, b, pre: pre + own[b]] = ids[nxt: nxt + own[b]]
            nxt += own[b]
    return tabs, int(n_blocks)


# ---- input tensors ------------------------------------------------------------------
@dataclass
class Inputs:
    prefix_k: object          # [shared_prefix, Hkv, D] or None
    prefix_v: object
    own_k: list               # per sequence [L_b - shared_prefix, Hkv, D]
    own_v: list
    q: object                 # [total_q, Hq, D]

    def seq_k(self, b):
        import torch
        return self.own_k[b] if self.prefix_k is None else torch.cat([self.prefix_k, self.own_k[b]])

    def seq_v(self, b):
        import torch
        return self.own_v[b] if self.prefix_v is None else torch.cat([self.prefix_v, self.own_v[b]])


def make_inputs(w: Workload, seed: int = 0) -> Inputs:
    import torch
    g = torch.Generator().manual_seed(seed)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    H, D = w.n_kv_heads, w.head_dim

    def draw_k(n):
        x = torch.randn((n, H, D), generator=g, dtype=torch.float32)
        x[..., :4] *= 10.0
        return x.to(dt)

    def draw_v(n):
        return torch.randn((n, H, D), generator=g, dtype=torch.float32).to(dt)

    pk = pv = None
    if w.shared_prefix:
        pk = draw_k(w.shared_prefix)
        pv = draw_v(w.shared_prefix)
    ok, ov = [], []
    for L in w.seq_lens:
        n = L - w.shared_prefix
        ok.append(draw_k(n))
        ov.append(draw_v(n))
    q = torch.randn((w.total_q, w.n_q_heads, D), generator=g, dtype=torch.float32).to(dt)
    return Inputs(pk, pv, ok, ov, q)


def shard(n_items: int, rank: int, world: int):
    """Contiguous share [lo, hi) of n_items for `rank` of `world` (sizes differ by <= 1)."""
    base, rem = divmod(n_items, world)
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0)
