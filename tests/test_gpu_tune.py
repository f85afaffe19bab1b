"""mq_tune on the device: budget handling, bit-identical admission, evidence log."""
import json
import os

import pytest
import torch

import quantized_kv_decode_quantize_b200 as mq
from quantized_kv_decode_quantize_b200 import workloads as wl
from tests.gpu_harness import GpuCase

pytestmark = pytest.mark.gpu


def test_tune_zero_budget_keeps_defaults():
    cache = mq.Cache(8, 128, 4)
    before = [mq.mq_get_decode_config(cache.handle, k) for k in range(3)]
    r = mq.mq_tune(cache.handle, 0.0, 32)
    assert r["status"] == mq.MQ_TUNE_BUDGET_EXHAUSTED
    assert [mq.mq_get_decode_config(cache.handle, k) for k in range(3)] == before


def test_tune_within_budget_and_output_unchanged(tmp_path):
    w = wl.reduced("verify")
    case = GpuCase(w)
    ref = [t.clone() for t in case.decode()]
    log = str(tmp_path / "tune.json")
    budget = 40.0
    r = mq.mq_tune(case.cache.handle, budget, w.n_q_heads, log)
    assert r["status"] in (mq.MQ_OK, mq.MQ_TUNE_BUDGET_EXHAUSTED)
    assert r["elapsed_s"] <= budget + 1.0
    assert r["n_tried"] > 0
    assert r["cost"] <= 1.0 + 1e-9
    d = json.load(open(log))
    assert d["candidates"] and any(c["measured"] and c["bit_identical"] for c in d["candidates"])
    # ring depth never changes the bytes, so those candidates are all admitted
    assert all(c["bit_identical"] for c in d["candidates"] if c["measured"] and c["splits_per_sm"] == 1)
    # the tuned configuration gives the same bytes as the defaults
    out, lse = case.decode()
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1])
    assert case.status() == mq.MQ_OK
