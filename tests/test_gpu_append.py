"""mq_kv_append (CUDA) against the CPU oracle: codes and scales must match bit for bit,
and so must the packed V bytes in the codec's canonical packing (read back through
mq_kv_export)."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_decode_quantize_b200 as mq
import workloads as wl
from tests import oracle_pins, pagelayout
from tests.gpu_harness import GpuCase, oracle_codes

pytestmark = pytest.mark.gpu


def _assert_seq_equal(case, b):
    kc, ks, vp, vs = case.read_sequence(b)
    ekc, eks, evp, evs = oracle_codes(case.inp, b)
    assert np.array_equal(kc, ekc), "K codes differ"
    assert np.array_equal(ks, eks), "K scales differ"
    assert np.array_equal(vp, evp), "V codes differ"
    assert np.array_equal(vs, evs), "V scales differ"


def export_sequence(case, b, copy=0):
    """Every token of sequence b through mq_kv_export (one call, one sequence)."""
    w = case.w
    L = w.seq_lens[b]
    H, D = w.n_kv_heads, w.head_dim
    i32 = dict(dtype=torch.int32, device="cuda")
    kc = torch.empty((L, H, D), dtype=torch.int8, device="cuda")
    ks = torch.empty((L, H), dtype=torch.int16, device="cuda")
    vp = torch.empty((L, H, D // 2), dtype=torch.uint8, device="cuda")
    vs = torch.empty((L, H, D // 32), dtype=torch.int16, device="cuda")
    mq.mq_kv_export(case.cache.handle, 1, L, torch.tensor([0, L], **i32), torch.tensor([0], **i32),
                    case.tabs[copy][b:b + 1].contiguous(), w.max_blocks(), kc, ks, vp, vs)
    return (kc.cpu().numpy(), ks.cpu().numpy().view(np.uint16), vp.cpu().numpy(),
            vs.cpu().numpy().view(np.uint16))


def _assert_export_equal(case, b):
    kc, ks, vp, vs = export_sequence(case, b)
    ekc, eks, evp, evs = oracle_codes(case.inp, b)
    assert np.array_equal(kc, ekc), "exported K codes differ"
    assert np.array_equal(ks, eks), "exported K scales differ"
    assert np.array_equal(vp, evp), "exported packed V bytes differ from the oracle's packing"
    assert np.array_equal(vs, evs), "exported V scales differ"


@pytest.mark.parametrize("name", ["tiny", "long", "prefix", "verify", "mixed"])
def test_export_packed_bytes_bit_exact(name):
    """The codec's byte contract end to end: quantize-on-append, then the packed bytes
    read back in the canonical packing equal the oracle's packed bytes."""
    w = wl.reduced(name)
    case = GpuCase(w)
    for b in range(w.n_seqs):
        _assert_export_equal(case, b)
    assert case.status() == mq.MQ_OK


def test_export_bad_position_is_flagged_and_zeroed():
    w = wl.reduced("long")
    case = GpuCase(w)
    i32 = dict(dtype=torch.int32, device="cuda")
    H, D = w.n_kv_heads, w.head_dim
    kc = torch.full((2, H, D), 7, dtype=torch.int8, device="cuda")
    ks = torch.full((2, H), 7, dtype=torch.int16, device="cuda")
    vp = torch.full((2, H, D // 2), 7, dtype=torch.uint8, device="cuda")
    vs = torch.full((2, H, D // 32), 7, dtype=torch.int16, device="cuda")
    mq.mq_kv_export(case.cache.handle, 1, 2, torch.tensor([0, 2], **i32),
                    torch.tensor([w.max_blocks() * 16 - 1], **i32), case.tabs[0][:1].contiguous(), w.max_blocks(),
                    kc, ks, vp, vs)
    assert case.status() == mq.MQ_ERR_DEVICE
    # the first token is in range, the second is not: zeros there
    assert int(kc[1].abs().sum()) == 0 and int(vp[1].sum()) == 0 and int(ks[1].abs().sum()) == 0
    assert int(vs[1].abs().sum()) == 0


@pytest.mark.parametrize("name", ["tiny", "long", "prefix", "verify", "mixed"])
def test_append_reduced_workloads_bit_exact(name):
    w = wl.reduced(name)
    case = GpuCase(w)
    assert case.status() == mq.MQ_OK
    for b in range(w.n_seqs):
        _assert_seq_equal(case, b)


@pytest.mark.parametrize("name", ["long", "mixed"])
def test_append_full_size_bit_exact(name):
    """Full-size workloads: the 64K-token cache, and the 32-session D=256 batch whose
    step appends 512 tokens per session (checked on every session)."""
    w = wl.FULL[name]()
    case = GpuCase(w)
    assert case.status() == mq.MQ_OK
    seqs = range(w.n_seqs) if name == "long" else range(0, w.n_seqs, 3)
    for b in seqs:
        _assert_seq_equal(case, b)
        _assert_export_equal(case, b)


@pytest.mark.parametrize("D", [128, 256])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
def test_append_edge_vectors(D, dtype):
    """Zero vectors, constant vectors, exact ties, subnormal and underflowing scales,
    fp16-overflowing scales and NaN entries, in every input dtype."""
    rng = np.random.default_rng(4)
    n = 48
    x = rng.standard_normal((n, 2, D)).astype(np.float32)
    x[0] = 0.0                                       # all zero
    x[1] = 0.37                                      # constant
    x[2, 0, :] = (np.arange(D) % 9 - 4 + 0.5) * 2.0 ** -6
    x[2, 0, 0] = 127 * 2.0 ** -6                     # scale 2^-6 exactly: ties on K
    x[3] *= 1e-6                                     # K scale underflows to 0 in fp16
    x[4] *= 3e-6                                     # subnormal scales
    x[5] *= 2e5                                      # scales overflow fp16 (and f16 inputs hold inf)
    x[6, 1, 5] = np.nan                              # NaN element
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    xt = torch.from_numpy(x).to(tdt)
    yt = torch.from_numpy(x[::-1].copy()).to(tdt)
    xf, yf = xt.float().numpy(), yt.float().numpy()
    cache = mq.Cache(2, D, 4)
    tab = torch.tensor([[2, 0, 3, 1]], dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, n], dtype=torch.int32, device="cuda")
    sp = torch.tensor([0], dtype=torch.int32, device="cuda")
    mq.mq_kv_append(cache.handle, xt.cuda(), yt.cuda(), {"f32": 0, "bf16": 1, "f16": 2}[dtype], 1, n, cu, sp, tab, 4)
    assert mq.mq_device_status(cache.handle) == mq.MQ_OK
    kc, ks, vp, vs = pagelayout.gather_sequence(cache.pool.cpu().numpy(), 2, D, tab.cpu().numpy()[0], n)
    ekc, eks = oracle.quantize_k(xf)
    evp, evs = oracle.quantize_v(yf)
    assert np.array_equal(kc, ekc) and np.array_equal(ks, eks)
    assert np.array_equal(vp, evp) and np.array_equal(vs, evs)


def _near_ties(rng, n_tok, D, group, div, n_lo, n_hi):
    """Tokens whose elements sit at and a few ulps around (n + 1/2) * s, s the scale the
    token's (or group's) first element sets: every code is decided next to a tie."""
    x = np.zeros((n_tok, D), dtype=np.float32)
    for t in range(n_tok):
        for g0 in range(0, D, group):
            m = np.float32(10.0 ** rng.uniform(-3, 3))
            s = np.float32(np.float16(m / np.float32(div)))
            n = rng.integers(n_lo, n_hi + 1, group).astype(np.float32)
            v = ((n + np.float32(0.5)) * s).astype(np.float32)
            k = rng.integers(-3, 4, group)
            for _ in range(3):
                step = np.where(k > 0, np.float32(np.inf), np.float32(-np.inf))
                v = np.where(k != 0, np.nextafter(v, step), v).astype(np.float32)
                k = k - np.sign(k)
            v[0] = m
            x[t, g0:g0 + group] = v
    return x


@pytest.mark.parametrize("D", [128, 256])
def test_append_codes_next_to_ties_bit_exact(D):
    """Every K and V element at, or up to 3 ulps from, a half-integer multiple of its
    scale: the codes equal the oracle's IEEE-division codes bit for bit."""
    rng = np.random.default_rng(11)
    n = 64
    xk = _near_ties(rng, n, D, D, 127.0, -126, 125)
    xv = _near_ties(rng, n, D, 32, 7.0, -7, 5)
    kt = torch.from_numpy(np.stack([xk, xk[::-1]], 1).copy())
    vt = torch.from_numpy(np.stack([xv, xv[::-1]], 1).copy())
    cache = mq.Cache(2, D, 4)
    tab = torch.tensor([[1, 3, 0, 2]], dtype=torch.int32, device="cuda")
    cu = torch.tensor([0, n], dtype=torch.int32, device="cuda")
    sp = torch.tensor([0], dtype=torch.int32, device="cuda")
    mq.mq_kv_append(cache.handle, kt.cuda(), vt.cuda(), 0, 1, n, cu, sp, tab, 4)
    assert mq.mq_device_status(cache.handle) == mq.MQ_OK
    kc, ks, vp, vs = pagelayout.gather_sequence(cache.pool.cpu().numpy(), 2, D, tab.cpu().numpy()[0], n)
    ekc, eks = oracle.quantize_k(kt.numpy())
    evp, evs = oracle.quantize_v(vt.numpy())
    assert np.array_equal(ks, eks) and np.array_equal(vs, evs)
    assert np.array_equal(kc, ekc), f"K codes differ at {np.argwhere(kc != ekc)[:4].tolist()}"
    assert np.array_equal(vp, evp), f"V codes differ at {np.argwhere(vp != evp)[:4].tolist()}"


def test_append_hand_worked_cases():
    """The hand-derived cases of tests/golden/quant_hand_cases.json, through the GPU."""
    g = oracle_pins.golden()
    D = 128
    rows_k = [oracle_pins._pad(c["x"], D) for c in g["k"]]
    rows_v = []
    for c in g["v"]:
        if "x_by_group" in c:
            v = np.zeros(D, np.float32)
            for gi, vals in enumerate(c["x_by_group"]):
                v[32 * gi: 32 * gi + len(vals)] = vals
            rows_v.append(v)
        else:
            rows_v.append(oracle_pins._pad(c["x"], D))
    n = max(len(rows_k), len(rows_v))
    k = np.zeros((n, 1, D), np.float32)
    v = np.zeros((n, 1, D), np.float32)
    k[: len(rows_k), 0] = rows_k
    v[: len(rows_v), 0] = rows_v
    cache = mq.Cache(1, D, 1)
    tab = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    mq.mq_kv_append(cache.handle, torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), mq.MQ_F32, 1, n,
                    torch.tensor([0, n], dtype=torch.int32, device="cuda"),
                    torch.tensor([0], dtype=torch.int32, device="cuda"), tab, 1)
    kc, ks, vp, vs = pagelayout.gather_sequence(cache.pool.cpu().numpy(), 1, D, np.zeros(1, np.int32), n)
    for i, c in enumerate(g["k"]):
        assert int(ks[i, 0]) == int(c["scale_bits"], 16), c["why"]
        exp = np.zeros(D, np.int32)
        exp[: len(c["codes"])] = c["codes"]
        assert np.array_equal(kc[i, 0].astype(np.int32), exp), c["why"]
    for i, c in enumerate(g["v"]):
        assert [int(s) for s in vs[i, 0]] == [int(s, 16) for s in c["scale_bits"]], c["why"]
        if "bytes" in c:
            exp = np.zeros(D // 2, np.uint8)
            exp[: len(c["bytes"])] = [int(b, 16) for b in c["bytes"]]
            assert np.array_equal(vp[i, 0], exp), c["why"]
        else:
            assert [int(vp[i, 0, 16 * gi]) for gi in range(4)] == [int(b, 16) for b in c["first_bytes_by_group"]]


def test_append_incremental_equals_bulk():
    """Appending token by token at increasing positions writes the same pages as one bulk append."""
    w = wl.reduced("long")
    w.seq_lens = [77]
    inp = wl.make_inputs(w)
    bulk = GpuCase(w, inp)
    inc = mq.Cache(w.n_kv_heads, w.head_dim, bulk.cache.n_blocks)
    for pos in range(77):
        mq.mq_kv_append(inc.handle, inp.own_k[0][pos: pos + 1].cuda(), inp.own_v[0][pos: pos + 1].cuda(), mq.MQ_BF16,
                        1, 1, torch.tensor([0, 1], dtype=torch.int32, device="cuda"),
                        torch.tensor([pos], dtype=torch.int32, device="cuda"), bulk.tabs[0], w.max_blocks())
    a = pagelayout.gather_sequence(bulk.cache.pool.cpu().numpy(), w.n_kv_heads, w.head_dim, bulk.tabs_np[0, 0], 77)
    b = pagelayout.gather_sequence(inc.pool.cpu().numpy(), w.n_kv_heads, w.head_dim, bulk.tabs_np[0, 0], 77)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_append_bad_position_and_block_are_flagged():
    cache = mq.Cache(1, 128, 2)
    k = torch.zeros((2, 1, 128), dtype=torch.bfloat16, device="cuda")
    tab = torch.tensor([[0, 7]], dtype=torch.int32, device="cuda")     # block 7 is out of range
    cu = torch.tensor([0, 2], dtype=torch.int32, device="cuda")
    mq.mq_kv_append(cache.handle, k, k, mq.MQ_BF16, 1, 2, cu, torch.tensor([16], dtype=torch.int32, device="cuda"),
                    tab, 2)
    assert mq.mq_device_status(cache.handle) == mq.MQ_ERR_DEVICE
    mq.mq_kv_append(cache.handle, k, k, mq.MQ_BF16, 1, 2, cu, torch.tensor([31], dtype=torch.int32, device="cuda"),
                    tab[:, :1].contiguous(), 1)
    assert mq.mq_device_status(cache.handle) == mq.MQ_ERR_DEVICE
    assert mq.mq_device_status(cache.handle) == mq.MQ_OK     # the word was cleared


@pytest.mark.parametrize("cuts", [[13, 40, 41, 77], [1, 2, 8, 9, 24, 77], [77]])
def test_append_split_launches_equal_bulk(cuts):
    """Appends cut at arbitrary positions (records completed across launches, partly
    with whole-record stores, partly with atomic nibble updates) write the same pages as
    one bulk append."""
    w = wl.reduced("long")
    w.seq_lens = [77]
    inp = wl.make_inputs(w)
    bulk = GpuCase(w, inp)
    inc = mq.Cache(w.n_kv_heads, w.head_dim, bulk.cache.n_blocks)
    lo = 0
    for hi in cuts:
        mq.mq_kv_append(inc.handle, inp.own_k[0][lo:hi].cuda(), inp.own_v[0][lo:hi].cuda(), mq.MQ_BF16, 1, hi - lo,
                        torch.tensor([0, hi - lo], dtype=torch.int32, device="cuda"),
                        torch.tensor([lo], dtype=torch.int32, device="cuda"), bulk.tabs[0], w.max_blocks())
        lo = hi
    assert mq.mq_device_status(inc.handle) == mq.MQ_OK
    a = pagelayout.gather_sequence(bulk.cache.pool.cpu().numpy(), w.n_kv_heads, w.head_dim, bulk.tabs_np[0, 0], 77)
    b = pagelayout.gather_sequence(inc.pool.cpu().numpy(), w.n_kv_heads, w.head_dim, bulk.tabs_np[0, 0], 77)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_append_inconsistent_cu_new_and_negative_position_are_flagged():
    cache = mq.Cache(1, 128, 2)
    k = torch.zeros((2, 1, 128), dtype=torch.bfloat16, device="cuda")
    tab = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    # cu_new claims 5 tokens where the launch has 2: refused before any K/V is read
    mq.mq_kv_append(cache.handle, k, k, mq.MQ_BF16, 1, 2, torch.tensor([0, 5], dtype=torch.int32, device="cuda"),
                    torch.tensor([0], dtype=torch.int32, device="cuda"), tab, 2)
    assert mq.mq_device_status(cache.handle) == mq.MQ_ERR_DEVICE
    # positions -1 and 0: the first is flagged, the second written
    mq.mq_kv_append(cache.handle, k, k, mq.MQ_BF16, 1, 2, torch.tensor([0, 2], dtype=torch.int32, device="cuda"),
                    torch.tensor([-1], dtype=torch.int32, device="cuda"), tab, 2)
    assert mq.mq_device_status(cache.handle) == mq.MQ_ERR_DEVICE
    assert mq.mq_device_status(cache.handle) == mq.MQ_OK
