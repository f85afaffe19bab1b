"""mq_decode_attn (CUDA) against the CPU oracle's fp64 attention over the same
quantized cache: every output within max-abs 1e-3 (and lse within 1e-3)."""
import math

import numpy as np
import pytest
import torch

import oracle
import quantized_kv_decode_quantize_b200 as mq
import workloads as wl
from tests.gpu_harness import GpuCase, oracle_outputs

pytestmark = pytest.mark.gpu

TOL = 1e-3          # max-abs on out (the stated tolerance)
TOL_LSE = 1e-3


def _check(case, seqs=None):
    out, lse = case.decode()
    assert case.status() == mq.MQ_OK
    eo, el = oracle_outputs(case.w, case.inp, seqs=seqs)
    o, l = out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    mask = ~np.isnan(el)
    err = np.max(np.abs(o[mask] - eo[mask])) if mask.any() else 0.0
    lerr = np.max(np.abs(l[mask] - el[mask])) if mask.any() else 0.0
    assert np.all(np.isfinite(o[mask]))
    assert err <= TOL, f"max-abs error {err:.3e}"
    assert lerr <= TOL_LSE, f"lse error {lerr:.3e}"
    return err


@pytest.mark.parametrize("name", ["tiny", "long", "prefix", "verify", "mixed"])
def test_decode_reduced_workloads(name):
    _check(GpuCase(wl.reduced(name)))


@pytest.mark.parametrize("name", ["tiny", "long", "prefix", "verify", "mixed"])
def test_decode_full_size_workloads(name):
    """Full sizes (64K history etc.), default launch configuration, every output row
    compared (the C oracle with OpenMP computes them all)."""
    _check(GpuCase(wl.FULL[name]()))


@pytest.mark.parametrize("L", [1, 2, 15, 16, 17, 127, 128, 129, 255, 1025])
def test_decode_lengths(L):
    w = wl.long_decode(L=L)
    _check(GpuCase(w))


@pytest.mark.parametrize("Hq,Hkv,D,L,n", [(8, 2, 128, 262152, 8), (4, 1, 256, 524288, 4)])
def test_decode_long_history_row_class_fallback(Hq, Hkv, D, L, n):
    """Histories whose per-warp partial stacks outgrow shared memory in the natural
    row class (32 rows at D 128, 16 rows at D 256) run in a smaller class with more
    row blocks; every row stays within tolerance."""
    _check(GpuCase(wl.Workload("long_fallback", Hq, Hkv, D, [L], [n], [n], shuffle=False)))


def test_workspace_reused_across_shapes():
    """One workspace, sized for the largest shape and passed with the same size on
    every call, serves calls of different shapes back to back (few units with many
    splits, then many units): each output is bit-identical to the same call with a
    fresh zero-filled workspace of its own."""
    cases = [GpuCase(wl.FULL["long"]()),
             GpuCase(wl.Workload("many_units", 32, 8, 128, [600 + 37 * i for i in range(40)], [1] * 40, [1] * 40)),
             GpuCase(wl.reduced("verify")),
             GpuCase(wl.reduced("mixed"))]
    fresh = [c.decode()[0].clone() for c in cases]
    shared = torch.zeros(max(c.ws.numel() for c in cases), dtype=torch.uint8, device="cuda")
    for c in cases:
        c.ws = shared
    for i in [0, 1, 2, 3, 0, 1, 3, 2, 0]:
        out = cases[i].decode()[0]
        assert torch.equal(out, fresh[i]), f"case {i}"
        assert cases[i].status() == mq.MQ_OK


def test_single_token_cache_returns_its_value():
    """L = 1: the weight is exactly 1, so out equals the dequantized v_0 exactly."""
    w = wl.long_decode(L=1)
    case = GpuCase(w)
    out, _ = case.decode()
    vp, vs = oracle.quantize_v(case.inp.seq_v(0).float().numpy())
    v0 = oracle.dequantize_v(vp, vs)[0]                     # [Hkv, D]
    G = w.n_q_heads // w.n_kv_heads
    exp = np.repeat(v0, G, axis=0)
    assert np.array_equal(out.cpu().numpy()[0].astype(np.float64), exp)


@pytest.mark.parametrize("Hq,Hkv,n,D", [(8, 8, 1, 128), (16, 2, 1, 128), (4, 2, 8, 128), (32, 8, 8, 128),
                                         (64, 8, 8, 128), (16, 4, 8, 256), (8, 4, 3, 256), (12, 4, 5, 128)])
def test_decode_gqa_and_draft_shapes(Hq, Hkv, n, D):
    """Every row class (8, 16, 32 rows per kv-head) and several row blocks."""
    w = wl.Workload("shape", Hq, Hkv, D, [700, 1300], [n, max(1, n - 1)], [n, max(1, n - 1)])
    _check(GpuCase(w))


def test_drafts_equal_cache_length():
    """n_q = L: the first draft sees one token."""
    w = wl.Workload("all_drafts", 32, 8, 128, [8, 3], [8, 3], [8, 3])
    _check(GpuCase(w))


def test_f16_queries():
    w = wl.reduced("long")
    inp = wl.make_inputs(w)
    case = GpuCase(w, inp)
    q16 = inp.q.to(torch.float16)
    mq.mq_decode_attn(case.cache.handle, q16.cuda(), mq.MQ_F16, w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                      w.max_seq_len, case.tabs[0], w.max_blocks(), case.seq_lens, case.n_q,
                      1 / math.sqrt(w.head_dim), case.out, case.lse, case.ws, case.ws.numel())
    inp.q = q16
    eo, _ = oracle_outputs(w, inp)
    assert np.max(np.abs(case.out.cpu().numpy() - eo)) <= TOL


def test_ragged_grid_and_null_lse():
    """max_seq_len far above the actual lengths (empty CTAs exit), lse = NULL."""
    w = wl.reduced("mixed")
    case = GpuCase(w)
    mq.mq_decode_attn(case.cache.handle, case.q, mq.MQ_BF16, w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                      w.max_seq_len, case.tabs[0], w.max_blocks(), case.seq_lens, case.n_q,
                      1 / math.sqrt(w.head_dim), case.out, None, case.ws, case.ws.numel())
    assert case.status() == mq.MQ_OK
    eo, _ = oracle_outputs(w, case.inp)
    assert np.max(np.abs(case.out.cpu().numpy() - eo)) <= TOL


def test_shared_prefix_equals_private_copies():
    """Sessions that alias the same physical prefix blocks get bit-identical outputs
    to the same sessions holding private copies of the prefix."""
    w = wl.reduced("prefix")
    inp = wl.make_inputs(w)
    shared = GpuCase(w, inp)
    o1 = shared.decode()[0].clone()
    wp = wl.Workload("private", w.n_q_heads, w.n_kv_heads, w.head_dim, list(w.seq_lens), list(w.n_q),
                     list(w.n_append), shared_prefix=0)
    inp2 = wl.Inputs(None, None, [inp.seq_k(b) for b in range(w.n_seqs)], [inp.seq_v(b) for b in range(w.n_seqs)],
                     inp.q)
    private = GpuCase(wp, inp2)
    o2 = private.decode()[0]
    assert torch.equal(o1, o2)


RING_STAGES = (2, 3, 4)
SPLITS_PER_SM = (1, 2, 4)


@pytest.mark.parametrize("name", ["long", "verify", "mixed"])
def test_ring_depth_bit_identical(name):
    """The ring depth never changes the output bytes."""
    w = wl.reduced(name)
    if name == "long":
        w = wl.long_decode(L=20000)
    case = GpuCase(w)
    ref = [t.clone() for t in case.decode()]
    for sps in SPLITS_PER_SM:
        for k in range(3):
            mq.mq_set_decode_config(case.cache.handle, k, 4, sps)
        base = [t.clone() for t in case.decode()]
        for r in RING_STAGES:
            for k in range(3):
                mq.mq_set_decode_config(case.cache.handle, k, r, sps)
            out, lse = case.decode()
            assert case.status() == mq.MQ_OK
            assert torch.equal(out, base[0]) and torch.equal(lse, base[1]), (r, sps)
        if sps == 1:
            assert torch.equal(base[0], ref[0]) and torch.equal(base[1], ref[1])


@pytest.mark.parametrize("shape", ["long", "tiny", "mixed", "gqa8", "ragged"])
def test_split_count_bit_identical_for_decode_classes(shape):
    """One query token per sequence at GQA <= 8 (row classes of 4 and 8 rows): every split
    count and ring depth gives the same output bytes, because the merge-tree leaves are
    fixed runs of chunks that do not depend on the split count."""
    if shape == "long":
        w = wl.long_decode(L=20000)
    elif shape == "tiny":
        w = wl.tiny(L=4096)
    elif shape == "mixed":
        w = wl.reduced("mixed")
    elif shape == "gqa8":
        w = wl.Workload("gqa8", 32, 4, 128, [33000, 5000], [1, 1], [1, 1])
    else:
        w = wl.Workload("ragged", 8, 2, 256, [70000, 129, 16385], [1, 1, 1], [1, 1, 1])
    case = GpuCase(w)
    ref = [t.clone() for t in case.decode()]
    assert case.status() == mq.MQ_OK
    for sps in SPLITS_PER_SM:
        for r in RING_STAGES:
            mq.mq_set_decode_config(case.cache.handle, 0, r, sps)
            out, lse = case.decode()
            assert case.status() == mq.MQ_OK
            assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1]), (sps, r)
    _check(case)


def test_flat_grid_many_sequences_of_very_different_lengths():
    """36 sequences (more than one warp's worth: the device planner reads their lengths in
    two rounds) from 1 token to 40000: the units take CTAs in proportion to their own
    lengths, chosen on the device; every split budget and ring depth gives the same bytes,
    within tolerance of the oracle."""
    rng = np.random.default_rng(5)
    lens = [1, 40000, 16, 17, 2048] + np.floor(np.exp(rng.uniform(0.0, math.log(40000), 31))).astype(int).tolist()
    w = wl.Workload("flat_many", 32, 8, 128, lens, [1] * len(lens), [1] * len(lens))
    case = GpuCase(w)
    ref = [t.clone() for t in case.decode()]
    assert case.status() == mq.MQ_OK
    for sps in SPLITS_PER_SM:
        for r in (2, 4):
            mq.mq_set_decode_config(case.cache.handle, 0, r, sps)
            out, lse = case.decode()
            assert case.status() == mq.MQ_OK
            assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1]), (sps, r)
    _check(case)


def test_batch_past_the_flat_grid_limit():
    """80 sequences (more than a flat grid takes: the (split, unit) grid sized by the
    longest): bit-identical for every split budget, within tolerance of the oracle."""
    rng = np.random.default_rng(8)
    lens = [9000, 1] + rng.integers(16, 3000, 78).tolist()
    w = wl.Workload("past_flat", 16, 4, 128, lens, [1] * len(lens), [1] * len(lens))
    case = GpuCase(w)
    ref = [t.clone() for t in case.decode()]
    assert case.status() == mq.MQ_OK
    for sps in SPLITS_PER_SM:
        mq.mq_set_decode_config(case.cache.handle, 0, 3, sps)
        out, lse = case.decode()
        assert case.status() == mq.MQ_OK
        assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1]), sps
    _check(case)


def test_flat_grid_bad_sequence_is_flagged_and_the_others_unchanged():
    """A sequence with an out-of-range length in a batch: the device error word is set, the
    sequence takes no CTA, and every other sequence's output keeps its bytes."""
    w = wl.Workload("flat_bad", 32, 8, 128, [20000, 3000, 9000, 500], [1] * 4, [1] * 4)
    case = GpuCase(w)
    ref = [t.clone() for t in case.decode()]
    assert case.status() == mq.MQ_OK
    bad = case.seq_lens.clone()
    bad[1] = w.max_blocks() * 16 + 5
    mq.mq_decode_attn(case.cache.handle, case.q, mq.MQ_BF16, w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                      w.max_seq_len, case.tabs[0], w.max_blocks(), bad, case.n_q, 1.0 / math.sqrt(w.head_dim),
                      case.out, case.lse, case.ws, case.ws.numel())
    assert case.status() == mq.MQ_ERR_DEVICE
    keep = [0, 2, 3]   # one query row per sequence
    assert torch.equal(case.out[keep], ref[0][keep]) and torch.equal(case.lse[keep], ref[1][keep])


@pytest.mark.parametrize("shape", ["gqa8", "drafts4", "d256_gqa8", "d256_drafts4"])
def test_softmax_warps_bit_identical(shape):
    """Splitting a row block over two groups of softmax warps never changes the output."""
    w = {"gqa8": wl.Workload("gqa8", 32, 4, 128, [20000, 3000], [1, 1], [1, 1]),
         "drafts4": wl.Workload("drafts4", 16, 4, 128, [9000, 700], [4, 3], [4, 3]),
         "d256_gqa8": wl.Workload("d256_gqa8", 16, 2, 256, [12000], [1], [1]),
         "d256_drafts4": wl.Workload("d256_drafts4", 16, 4, 256, [5000, 300], [4, 2], [4, 2])}[shape]
    case = GpuCase(w)
    cls = 0 if max(w.n_q) * w.n_q_heads // w.n_kv_heads <= 8 else 1
    mq.mq_set_decode_config(case.cache.handle, cls, 4, 1, 4)
    ref = [t.clone() for t in case.decode()]
    assert case.status() == mq.MQ_OK
    for r, sps in ((4, 1), (3, 2)):
        mq.mq_set_decode_config(case.cache.handle, cls, r, sps, 8)
        out, lse = case.decode()
        assert case.status() == mq.MQ_OK
        if sps == 1 or cls == 0 and shape != "d256_gqa8":
            assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1]), (r, sps)
    _check(case)


@pytest.mark.parametrize("sps", SPLITS_PER_SM)
def test_every_split_count_within_tolerance(sps):
    """Every split count the tuner may try stays within the tolerance of the oracle."""
    w = wl.long_decode(L=20000)
    case = GpuCase(w)
    for k in range(3):
        mq.mq_set_decode_config(case.cache.handle, k, 3, sps)
    _check(case)


def test_workspace_needs_no_initialization():
    """A workspace full of garbage gives the same bytes as a zeroed one, call after call."""
    case = GpuCase(wl.reduced("verify"))
    ref = case.decode()[0].clone()
    case.ws.fill_(0xFF)
    for _ in range(5):
        assert torch.equal(case.decode()[0], ref)
    assert case.status() == mq.MQ_OK


def test_bad_sequence_is_flagged_not_faulted():
    w = wl.reduced("long")
    case = GpuCase(w)
    bad_len = torch.tensor([w.max_blocks() * 16 + 5], dtype=torch.int32, device="cuda")
    mq.mq_decode_attn(case.cache.handle, case.q, mq.MQ_BF16, 1, w.n_q_heads, 1, 1, w.max_seq_len, case.tabs[0],
                      w.max_blocks(), bad_len, case.n_q, 0.1, case.out, case.lse, case.ws, case.ws.numel())
    assert case.status() == mq.MQ_ERR_DEVICE
    bad_tab = case.tabs[0].clone()
    bad_tab[0, 3] = 10 ** 8
    case.ws.zero_()
    mq.mq_decode_attn(case.cache.handle, case.q, mq.MQ_BF16, 1, w.n_q_heads, 1, 1, w.max_seq_len, bad_tab,
                      w.max_blocks(), case.seq_lens, case.n_q, 0.1, case.out, case.lse, case.ws, case.ws.numel())
    assert case.status() == mq.MQ_ERR_DEVICE


def test_error_against_unquantized_is_reported():
    """Reported, not gated: error of the quantized path against fp64 attention over
    the original (unquantized) K/V on the long workload shape (parity unpinned)."""
    w = wl.long_decode(L=4096)
    case = GpuCase(w)
    out, _ = case.decode()
    eo, _ = oracle_outputs(w, case.inp, unquantized=True)
    o = out.cpu().numpy()
    err = float(np.max(np.abs(o - eo)))
    rel = float(np.linalg.norm(o - eo) / np.linalg.norm(eo))
    print(f"\nvs unquantized fp64 attention: max-abs {err:.3e}, relative L2 {rel:.3e}")
    assert np.isfinite(err)


@pytest.mark.parametrize("vmax", [1e4, 3e4, 1e5, 4.5e5])
@pytest.mark.parametrize("name", ["long", "verify"])
def test_large_values_up_to_the_codec_domain(name, vmax):
    """Values whose V scales reach the top of fp16 (a scale is max|x| / 7, so |V| up to
    65504 * 7 = 458,528 is inside the codec's domain).  The weights p * s_v are fp16
    operands of the value MMAs; the running max is raised where they could overflow.
    Attention is linear in V, so the bar is the unit-scale bar on out / vmax (here
    |V| <= vmax, against |V| of about 5 in the unit workloads); lse does not depend on
    V and keeps the absolute bar.  Mixed magnitudes: every 7th token is unscaled and
    every 5th at a third of the rest."""
    w = wl.reduced(name)
    inp = wl.make_inputs(w)
    v = inp.own_v[0].float()
    f = torch.full((v.shape[0], 1, 1), 1.0)
    f[::5] = 1.0 / 3.0
    f[::7] = 1.0 / vmax
    inp.own_v[0] = (v / v.abs().amax() * vmax * f).to(inp.own_v[0].dtype)
    case = GpuCase(w, inputs=inp)
    out, lse = case.decode()
    assert case.status() == mq.MQ_OK
    eo, el = oracle_outputs(w, inp)
    o, l = out.cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o)), "non-finite output: a weight overflowed fp16"
    err = float(np.max(np.abs(o - eo))) / vmax
    lerr = float(np.max(np.abs(l - el)))
    assert err <= TOL, f"max-abs error / vmax {err:.3e}"
    assert lerr <= TOL_LSE, f"lse error {lerr:.3e}"
