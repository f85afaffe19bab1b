"""Drives the CUDA path through the C ABI for the GPU tests, and computes the CPU
oracle's expectations for the same seeded inputs."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import quantized_kv_decode_quantize_b200 as mq
import workloads as wl
from tests import pagelayout

DT = {"f32": mq.MQ_F32, "bf16": mq.MQ_BF16}


class GpuCase:
    """A workload populated into a device cache through mq_kv_append."""

    def __init__(self, w: wl.Workload, inputs: wl.Inputs | None = None, copies: int = 1, config=None,
                 workspace: bool = True):
        self.w = w
        self.inp = inputs if inputs is not None else wl.make_inputs(w)
        tabs, n_blocks = wl.block_tables(w, copies=copies)
        self.tabs_np = tabs
        self.tabs = torch.from_numpy(tabs).cuda()
        self.cache = mq.Cache(w.n_kv_heads, w.head_dim, n_blocks)
        if config is not None:
            for cls, cfg in config.items():
                mq.mq_set_decode_config(self.cache.handle, cls, *cfg)
        self.copies = copies
        for c in range(copies):
            self.populate(c)
        self.seq_lens = torch.tensor(w.seq_lens, dtype=torch.int32, device="cuda")
        self.n_q = torch.tensor(w.n_q, dtype=torch.int32, device="cuda")
        self.q = self.inp.q.cuda()
        if workspace:   # decode calls (prefill needs none)
            ws_bytes = mq.mq_decode_workspace_bytes(self.cache.handle, w.n_seqs, w.n_q_heads, w.max_q, w.max_seq_len)
            assert ws_bytes > 0
            self.ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
        self.out = torch.empty((w.total_q, w.n_q_heads, w.head_dim), dtype=torch.float32, device="cuda")
        self.lse = torch.empty((w.total_q, w.n_q_heads), dtype=torch.float32, device="cuda")

    def append(self, k, v, seq_ids, start_pos, copy=0):
        """Appends per-sequence token blocks: k, v lists of [n_i, Hkv, D] tensors."""
        w = self.w
        n_new = [int(x.shape[0]) for x in k]
        cu = torch.tensor(np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32), device="cuda")
        sp = torch.tensor(start_pos, dtype=torch.int32, device="cuda")
        bt = self.tabs[copy][torch.tensor(seq_ids, device="cuda")].contiguous()
        kk = torch.cat(k).cuda().contiguous()
        vv = torch.cat(v).cuda().contiguous()
        mq.mq_kv_append(self.cache.handle, kk, vv, DT[w.dtype], len(seq_ids), int(sum(n_new)), cu, sp, bt,
                        w.max_blocks())
        return kk, vv

    def populate(self, copy=0):
        w, inp = self.w, self.inp
        if w.shared_prefix:
            self.append([inp.prefix_k], [inp.prefix_v], [0], [0], copy)
        self.append(inp.own_k, inp.own_v, list(range(w.n_seqs)), [w.shared_prefix] * w.n_seqs, copy)

    def decode(self, copy=0, scale=None, with_lse=True):
        w = self.w
        scale = 1.0 / math.sqrt(w.head_dim) if scale is None else scale
        mq.mq_decode_attn(self.cache.handle, self.q, DT[w.dtype], w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                          w.max_seq_len, self.tabs[copy], w.max_blocks(), self.seq_lens, self.n_q, scale, self.out,
                          self.lse if with_lse else None, self.ws, self.ws.numel())
        return self.out, self.lse

    def decode_cascade(self, prefix_len=None, copy=0, scale=None, with_lse=True):
        """mq_decode_attn_cascade over the workload's shared prefix (or prefix_len)."""
        w = self.w
        prefix_len = w.shared_prefix if prefix_len is None else prefix_len
        scale = 1.0 / math.sqrt(w.head_dim) if scale is None else scale
        need = mq.mq_decode_cascade_workspace_bytes(self.cache.handle, w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                                                    w.max_seq_len, prefix_len)
        if self.ws.numel() < need:   # need == 0: the call itself refuses the arguments
            self.ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
        mq.mq_decode_attn_cascade(self.cache.handle, self.q, DT[w.dtype], w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                                  w.max_seq_len, self.tabs[copy], w.max_blocks(), self.seq_lens, self.n_q,
                                  prefix_len, scale, self.out, self.lse if with_lse else None, self.ws,
                                  self.ws.numel())
        return self.out, self.lse

    def status(self):
        return mq.mq_device_status(self.cache.handle)

    def read_sequence(self, b, copy=0):
        pool = self.cache.pool.cpu().numpy()
        return pagelayout.gather_sequence(pool, self.w.n_kv_heads, self.w.head_dim, self.tabs_np[copy, b],
                                          self.w.seq_lens[b])


def f32(t: torch.Tensor) -> np.ndarray:
    return t.float().numpy()


def oracle_codes(inp: wl.Inputs, b: int):
    k = f32(inp.seq_k(b))
    v = f32(inp.seq_v(b))
    kc, ks = oracle.quantize_k(k)
    vp, vs = oracle.quantize_v(v)
    return kc, ks, vp, vs


def oracle_outputs(w: wl.Workload, inp: wl.Inputs, scale=None, n_threads=None, seqs=None, unquantized=False):
    """Oracle out [total_q, Hq, D] and lse [total_q, Hq] (fp64) for the listed sequences
    (all by default; rows of other sequences are NaN)."""
    scale = 1.0 / math.sqrt(w.head_dim) if scale is None else scale
    n_threads = n_threads or oracle.max_threads()
    out = np.full((w.total_q, w.n_q_heads, w.head_dim), np.nan)
    lse = np.full((w.total_q, w.n_q_heads), np.nan)
    qoff = np.concatenate([[0], np.cumsum(w.n_q)]).astype(int)
    q = f32(inp.q).astype(np.float64)
    for b in (range(w.n_seqs) if seqs is None else seqs):
        qb = q[qoff[b]: qoff[b + 1]]
        if unquantized:
            o, l = oracle.attention(qb, f32(inp.seq_k(b)), f32(inp.seq_v(b)), scale, n_threads)
        else:
            kc, ks, vp, vs = oracle_codes(inp, b)
            o, l = oracle.attention_quant(qb, kc, ks, vp, vs, scale, n_threads)
        out[qoff[b]: qoff[b + 1]] = o
        lse[qoff[b]: qoff[b + 1]] = l
    return out, lse
