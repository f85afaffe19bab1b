"""mq_draft_ngram on the device against the oracle's definition (token ids and counts
must match exactly)."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_decode_quantize_b200 as mq

pytestmark = pytest.mark.gpu


def _run(hist, n, k, max_len=None):
    max_len = max_len or max(1, max(len(h) for h in hist))
    tok = np.zeros((len(hist), max_len), np.int32)
    for b, h in enumerate(hist):
        tok[b, :len(h)] = h
    lens = torch.tensor([len(h) for h in hist], dtype=torch.int32, device="cuda")
    drafts = torch.full((len(hist), k), -7, dtype=torch.int32, device="cuda")
    nd = torch.empty(len(hist), dtype=torch.int32, device="cuda")
    mq.mq_draft_ngram(torch.from_numpy(tok).cuda(), max_len, lens, len(hist), n, k, drafts, nd)
    torch.cuda.synchronize()
    return drafts.cpu().numpy(), nd.cpu().numpy()


def _check(hist, n, k):
    d, nd = _run(hist, n, k)
    for b, h in enumerate(hist):
        want = oracle.draft_ngram(np.array(h, np.int32), n, k).tolist()
        assert nd[b] == len(want), (b, nd[b], want)
        assert d[b, :nd[b]].tolist() == want
        assert np.all(d[b, nd[b]:] == -7)   # nothing written past the count


@pytest.mark.parametrize("n,k", [(1, 1), (2, 4), (3, 8), (5, 3), (8, 16)])
def test_draft_random_histories(n, k):
    rng = np.random.default_rng(100 + n)
    hist = [rng.integers(0, int(rng.integers(2, 6)), int(rng.integers(0, 3000))).tolist() for _ in range(37)]
    _check(hist, n, k)


def test_draft_long_history_planted_repeat():
    rng = np.random.default_rng(7)
    h = rng.integers(0, 1 << 30, 65536).astype(np.int64)
    h[1000:1006] = h[-6:]          # the last 6 tokens also sit at 1000 .. 1005
    h[50000:50006] = h[-6:]        # and, later, at 50000 .. 50005
    _check([h.astype(np.int32).tolist()], 6, 5)
    d, nd = _run([h.astype(np.int32).tolist()], 6, 5)
    assert nd[0] == 5 and d[0].tolist() == h[50006:50011].astype(np.int32).tolist()


def test_draft_edge_lengths():
    _check([[], [3], [3, 3], [1, 2], [9, 9, 9, 9, 9]], 1, 4)
    _check([[1, 2, 1, 2, 1, 2], [4, 8, 4, 8, 4]], 2, 2)


def test_draft_length_beyond_max_len_is_marked():
    tok = torch.zeros((2, 8), dtype=torch.int32, device="cuda")
    lens = torch.tensor([9, -1], dtype=torch.int32, device="cuda")
    drafts = torch.zeros((2, 2), dtype=torch.int32, device="cuda")
    nd = torch.zeros(2, dtype=torch.int32, device="cuda")
    mq.mq_draft_ngram(tok, 8, lens, 2, 2, 2, drafts, nd)
    assert nd.cpu().tolist() == [-1, -1]
