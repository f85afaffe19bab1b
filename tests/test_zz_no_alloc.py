"""mq_decode_attn_static (library-owned scratch) against mq_decode_attn (caller
workspace): two calls in a row through the C ABI.  Both entry points run the same
launch plan over the same pages, so each output must equal the workspace entry
point's bit for bit (a scratch offset or aliasing fault that moved a partial would
show); on the reduced shapes the outputs are also within the decode tolerance of the
CPU oracle.  Collected last, so it also runs after every other GPU test has used the
library on the same device."""
import math

import numpy as np
import pytest
import torch

import quantized_kv_decode_quantize_b200 as mq
import workloads as wl
from tests.gpu_harness import DT, GpuCase, oracle_outputs

pytestmark = pytest.mark.gpu

TOL = 1e-3


def _static(case, out, lse):
    w = case.w
    mq.mq_decode_attn_static(case.cache.handle, case.q, DT[w.dtype], w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                             w.max_seq_len, case.tabs[0], w.max_blocks(), case.seq_lens, case.n_q,
                             1.0 / math.sqrt(w.head_dim), out, lse)


@pytest.mark.parametrize("w,small", [(wl.reduced("long"), True), (wl.reduced("mixed"), True),
                                     (wl.FULL["long"](), False), (wl.FULL["verify"](), False)],
                         ids=["long_reduced", "mixed_reduced", "long_64k", "verify8_64k"])
def test_static_scratch_twice_equals_workspace_entry(w, small):
    case = GpuCase(w)
    ref_out, ref_lse = (t.clone() for t in case.decode())
    outs = []
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        _static(case, out, lse)
        outs.append((out, lse))
    torch.cuda.synchronize()
    assert case.status() == mq.MQ_OK
    for out, lse in outs:
        assert torch.isfinite(out).all()
        assert torch.equal(out, ref_out), f"max-abs difference {(out - ref_out).abs().max().item():.3e}"
        assert torch.equal(lse, ref_lse), f"lse difference {(lse - ref_lse).abs().max().item():.3e}"
    if small:
        eo, el = oracle_outputs(w, case.inp)
        err = float(np.max(np.abs(outs[1][0].cpu().numpy() - eo)))
        lerr = float(np.max(np.abs(outs[1][1].cpu().numpy() - el)))
        assert err <= TOL and lerr <= TOL, (err, lerr)


def test_static_scratch_refuses_a_shape_beyond_its_size():
    cache = mq.Cache(8, 128, 64)
    n_seqs = 4096
    assert mq.mq_decode_workspace_bytes(cache.handle, n_seqs, 32, 1, 1024) > 16 << 20
    q = torch.zeros((n_seqs, 32, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((n_seqs, 32, 128), dtype=torch.float32, device="cuda")
    bt = torch.zeros((n_seqs, 64), dtype=torch.int32, device="cuda")
    lens = torch.full((n_seqs,), 1024, dtype=torch.int32, device="cuda")
    nq = torch.ones(n_seqs, dtype=torch.int32, device="cuda")
    with pytest.raises(mq.MQError) as ei:
        mq.mq_decode_attn_static(cache.handle, q, mq.MQ_BF16, n_seqs, 32, n_seqs, 1, 1024, bt, 64, lens, nq,
                                 1.0 / math.sqrt(128), out, None)
    assert ei.value.status == mq.MQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert np.count_nonzero(out.cpu().numpy()) == 0
