"""mq_prefill_attn (CUDA) against the CPU oracle's fp64 attention over the same
quantized cache: every checked output within max-abs 1e-3 (and lse within 1e-3).
Query token j of n sees positions 0 .. L - n + j (a whole prompt when n = L, a prompt
chunk after a cached history when n < L)."""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_kv_decode_quantize_b200 as mq
import workloads as wl
from tests.gpu_harness import DT, GpuCase, oracle_codes, oracle_outputs

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _prefill(case, with_lse=True):
    w = case.w
    mq.mq_prefill_attn(case.cache.handle, case.q, DT[w.dtype], w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                       w.max_seq_len, case.tabs[0], w.max_blocks(), case.seq_lens, case.n_q,
                       1.0 / math.sqrt(w.head_dim), case.out, case.lse if with_lse else None)
    return case.out, case.lse


def _check_all(w):
    case = GpuCase(w, workspace=False)
    out, lse = _prefill(case)
    assert case.status() == mq.MQ_OK
    eo, el = oracle_outputs(w, case.inp)
    o, l = out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o))
    err, lerr = float(np.max(np.abs(o - eo))), float(np.max(np.abs(l - el)))
    assert err <= TOL, f"max-abs error {err:.3e}"
    assert lerr <= TOL, f"lse error {lerr:.3e}"


@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 8), (16, 2)], ids=["gqa4", "mha", "gqa8"])
def test_prefill_whole_prompt(hq, hkv):
    """n = L: every position of a 1000-token prompt (several 128-row tiles and
    128-token chunks, ragged ends)."""
    _check_all(wl.Workload("prefill_1000", hq, hkv, 128, [1000], [1000], [1000]))


def test_prefill_chunk_after_history_and_mixed_batch():
    """Sequences of unequal lengths in one launch: a 300-token prompt chunk after a
    1200-token history, a whole 700-token prompt, and a single query (decode-like)."""
    _check_all(wl.Workload("prefill_mixed", 32, 8, 128, [1500, 700, 257], [300, 700, 1], [300, 700, 1]))


def test_prefill_fp16_queries():
    """F16 q (exact in the fp16 operand, like BF16)."""
    w = wl.Workload("prefill_f16", 8, 2, 128, [777], [777], [777])
    case = GpuCase(w, workspace=False)
    case.q = case.q.to(torch.float16)
    mq.mq_prefill_attn(case.cache.handle, case.q, mq.MQ_F16, w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                       w.max_seq_len, case.tabs[0], w.max_blocks(), case.seq_lens, case.n_q,
                       1.0 / math.sqrt(w.head_dim), case.out, case.lse)
    assert case.status() == mq.MQ_OK
    case.inp.q = case.q.cpu()
    eo, el = oracle_outputs(w, case.inp)
    err = float(np.max(np.abs(case.out.cpu().numpy() - eo)))
    lerr = float(np.max(np.abs(case.lse.cpu().numpy() - el)))
    assert err <= TOL and lerr <= TOL, (err, lerr)


def test_prefill_refuses_f32_queries():
    """F32 q would lose bits in the fp16 operand: refused, nothing launched."""
    w = wl.Workload("prefill_f32", 8, 2, 128, [64], [64], [64])
    w.dtype = "f32"
    case = GpuCase(w, workspace=False)
    case.out.fill_(7.0)
    with pytest.raises(mq.MQError) as e:
        _prefill(case)
    assert e.value.status == mq.MQ_ERR_UNSUPPORTED
    assert bool((case.out == 7.0).all())


def _check_sampled(w, rows, seed=3):
    """Sampled query rows of a large prefill against the oracle, one query at a time
    over the positions it sees (the oracle's causal rule with n = 1 on the truncated
    cache is the same row)."""
    case = GpuCase(w, workspace=False)
    out, lse = _prefill(case)
    assert case.status() == mq.MQ_OK
    o, l = out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o))
    kc, ks, vp, vs = oracle_codes(case.inp, 0)
    q = case.inp.q.float().numpy().astype(np.float64)
    L, n = w.seq_lens[0], w.n_q[0]
    rng = np.random.default_rng(seed)
    js = sorted(set([0, n - 1] + list(rng.choice(n, size=rows, replace=False))))
    for j in js:
        vis = L - n + j + 1
        eo, el = oracle.attention_quant(q[j:j + 1], kc[:vis], ks[:vis], vp[:vis], vs[:vis],
                                        1.0 / math.sqrt(w.head_dim), oracle.max_threads())
        err = float(np.max(np.abs(o[j] - eo[0])))
        lerr = float(np.max(np.abs(l[j] - el[0])))
        assert err <= TOL and lerr <= TOL, (j, err, lerr)


def test_prefill_4k_prompt_sampled_rows():
    _check_sampled(wl.Workload("prefill_4k", 32, 8, 128, [4096], [4096], [4096]), rows=24)


def test_prefill_64k_prompt_sampled_rows():
    """A whole 64K-token prompt (512 tiles per kv-head, up to 512 chunks each)."""
    _check_sampled(wl.Workload("prefill_64k", 32, 8, 128, [65536], [65536], [65536]), rows=6)


def test_prefill_64k_chunk_after_history_sampled_rows():
    """The last 512 tokens of a 64K context as one prompt chunk."""
    _check_sampled(wl.Workload("prefill_64k_tail", 32, 8, 128, [65536], [512], [512]), rows=8)


def test_prefill_refuses_head_dim_256_and_odd_groups():
    cache = mq.Cache(4, 256, 8)
    i32 = dict(dtype=torch.int32, device="cuda")
    q = torch.zeros((4, 16, 256), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((4, 16, 256), dtype=torch.float32, device="cuda")
    bt = torch.zeros((1, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(mq.MQError) as e:
        mq.mq_prefill_attn(cache.handle, q, mq.MQ_BF16, 1, 16, 4, 4, 4, bt, 8, torch.tensor([4], **i32),
                           torch.tensor([4], **i32), 0.1, out, None)
    assert e.value.status == mq.MQ_ERR_UNSUPPORTED
    cache3 = mq.Cache(1, 128, 8)
    q3 = torch.zeros((4, 3, 128), dtype=torch.bfloat16, device="cuda")
    out3 = torch.zeros((4, 3, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(mq.MQError) as e:
        mq.mq_prefill_attn(cache3.handle, q3, mq.MQ_BF16, 1, 3, 4, 4, 4, bt, 8, torch.tensor([4], **i32),
                           torch.tensor([4], **i32), 0.1, out3, None)
    assert e.value.status == mq.MQ_ERR_UNSUPPORTED
