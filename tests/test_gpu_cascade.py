"""mq_decode_attn_cascade on the device: sessions sharing a cached prefix, the prefix
read once for every session's queries, merged with each session's own pages by
log-sum-exp.  Compared with the fp64 oracle over each session's whole cache (the
oracle knows nothing of the cascade: attention over the concatenated token set) and
with the plain decode."""
import numpy as np
import pytest
import torch

import quantized_kv_decode_quantize_b200 as mq
import workloads as wl
from tests.gpu_harness import GpuCase, oracle_outputs

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _check_oracle(case, out, lse):
    eo, el = oracle_outputs(case.w, case.inp)
    o, l = out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o))
    err = np.max(np.abs(o - eo))
    lerr = np.max(np.abs(l - el))
    assert err <= TOL, f"max-abs error {err:.3e}"
    assert lerr <= TOL, f"lse error {lerr:.3e}"
    assert case.status() == mq.MQ_OK
    return err


def test_cascade_reduced_prefix_workload():
    case = GpuCase(wl.reduced("prefix"))
    out, lse = case.decode_cascade()
    _check_oracle(case, out.clone(), lse.clone())


def test_cascade_full_size_prefix_workload():
    """8 sessions x (32768-token shared prefix + private suffix), every row checked."""
    case = GpuCase(wl.FULL["prefix"]())
    out, lse = case.decode_cascade()
    _check_oracle(case, out.clone(), lse.clone())


def test_cascade_close_to_plain_decode():
    case = GpuCase(wl.reduced("prefix"))
    o1, l1 = [t.clone() for t in case.decode()]
    o2, l2 = [t.clone() for t in case.decode_cascade()]
    assert (o1 - o2).abs().max().item() <= 1e-4
    assert (l1 - l2).abs().max().item() <= 1e-4


@pytest.mark.parametrize("prefix_len", [16, 512, 1008])
def test_cascade_any_page_aligned_split(prefix_len):
    """The cascade may split the cache at any page boundary inside the shared prefix;
    each split gives the whole-cache attention."""
    case = GpuCase(wl.reduced("prefix"))
    out, lse = case.decode_cascade(prefix_len=prefix_len)
    _check_oracle(case, out.clone(), lse.clone())


def test_cascade_with_drafts():
    """Sessions verifying drafts after a shared prefix: every draft sees the whole
    prefix, the drafts stay causal among themselves in the suffix pass."""
    pre = 1024
    lens = [pre + 300, pre + 901, pre + 57]
    nq = [3, 1, 4]
    w = wl.Workload("prefix_drafts", 16, 4, 128, lens, nq, nq, shared_prefix=pre)
    case = GpuCase(w)
    out, lse = case.decode_cascade()
    _check_oracle(case, out.clone(), lse.clone())


def test_cascade_without_lse_and_d256():
    w = wl.Workload("prefix_d256", 8, 2, 256, [512 + 200, 512 + 33], [1, 1], [1, 1], shared_prefix=512)
    case = GpuCase(w)
    ref_out, _ = [t.clone() for t in case.decode()]
    out, _ = case.decode_cascade(with_lse=False)
    assert (out - ref_out).abs().max().item() <= 1e-4
    assert case.status() == mq.MQ_OK


def test_cascade_argument_checks():
    case = GpuCase(wl.reduced("prefix"))
    w = case.w
    for bad in (0, 24, w.max_seq_len):
        assert mq.mq_decode_cascade_workspace_bytes(case.cache.handle, w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                                                    w.max_seq_len, bad) == 0
        with pytest.raises(mq.MQError) as e:
            case.decode_cascade(prefix_len=bad)
        assert e.value.status == mq.MQ_ERR_INVALID_ARG


def test_cascade_flags_a_session_shorter_than_the_prefix():
    """prefix_len beyond one session's queries: that session is skipped and reported;
    the call itself launches (the lengths live on the device)."""
    pre = 512
    w = wl.Workload("prefix_short", 16, 4, 128, [pre + 100, pre + 200], [1, 1], [1, 1], shared_prefix=pre)
    case = GpuCase(w)
    case.decode_cascade(prefix_len=pre + 112)   # session 0 has only pre + 100 tokens
    assert case.status() == mq.MQ_ERR_DEVICE
    assert case.status() == mq.MQ_OK            # the error word was cleared
