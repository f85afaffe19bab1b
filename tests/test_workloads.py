"""Seeded input generators and block tables (no GPU)."""
import numpy as np
import torch

import workloads as wl


def test_inputs_are_deterministic_and_shaped():
    w = wl.reduced("prefix")
    a, b = wl.make_inputs(w), wl.make_inputs(w)
    assert torch.equal(a.q, b.q) and torch.equal(a.prefix_k, b.prefix_k)
    for x, y in zip(a.own_v, b.own_v):
        assert torch.equal(x, y)
    assert a.q.shape == (w.total_q, w.n_q_heads, w.head_dim)
    for bb in range(w.n_seqs):
        assert a.seq_k(bb).shape == (w.seq_lens[bb], w.n_kv_heads, w.head_dim)
        assert a.seq_k(bb).dtype == torch.bfloat16


def test_outlier_channels():
    w = wl.long_decode(L=4000)
    k = wl.make_inputs(w).own_k[0].float()
    s = k.std(dim=(0, 1))
    assert torch.all(s[:4] > 8) and torch.all(s[4:] < 1.3)


def test_full_workload_shapes():
    t, l, p, v, m = (wl.FULL[n]() for n in ("tiny", "long", "prefix", "verify", "mixed"))
    assert t.seq_lens == [4096] and t.dtype == "f32" and (t.n_q_heads, t.n_kv_heads) == (8, 2)
    assert l.seq_lens == [65536] and (l.n_q_heads, l.n_kv_heads, l.head_dim) == (32, 8, 128)
    assert p.n_seqs == 8 and all(32768 + 1024 <= L <= 32768 + 8192 for L in p.seq_lens)
    assert v.seq_lens == [65544] and v.n_q == [8]
    assert m.n_seqs == 32 and m.head_dim == 256 and all(1024 + 512 <= L <= 65536 + 512 for L in m.seq_lens)
    assert m.n_append == [512] * 32


def test_block_tables():
    w = wl.reduced("prefix")
    tabs, n = wl.block_tables(w, copies=3)
    pre = w.shared_prefix // 16
    used = []
    for c in range(3):
        for b in range(w.n_seqs):
            assert np.array_equal(tabs[c, b, :pre], tabs[c, 0, :pre])
            nb = (w.seq_lens[b] + 15) // 16
            used += tabs[c, b, pre:nb].tolist()
        used += tabs[c, 0, :pre].tolist()
    assert sorted(used) == list(range(n))        # every block once; copies disjoint


def test_shard_partitions():
    for n in (0, 1, 7, 32):
        for world in (1, 2, 3, 8):
            parts = [wl.shard(n, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            assert max(h - l for l, h in parts) - min(h - l for l, h in parts) <= 1
