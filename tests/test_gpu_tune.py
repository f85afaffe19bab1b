"""mq_tune on the device: budget handling, bit-identical admission, evidence log."""
import json
import os

import pytest
import torch

import quantized_kv_decode_quantize_b200 as mq
import workloads as wl
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
    # the service cost's terms, the drafter launch among them, and the probe weights
    # weight(p) = sum_t launches(t, p) / time_at_defaults(t)
    terms = {t["name"]: t["default_us"] for t in d["terms"]}
    assert set(terms) == {"decode_4k", "decode_64k", "draft_64k", "verify8_64k", "prefill_4k", "prefill_64k"}
    assert all(v > 0 for v in terms.values())
    probes = {p["name"]: p for p in d["probes"]}
    spec = probes["draft_verify8_64k"]
    assert spec["launches"] == "draft_64k + verify8_64k"
    assert abs(spec["weight_per_s"] - 1e6 * (1 / terms["draft_64k"] + 1 / terms["verify8_64k"])) \
        <= 1e-3 * spec["weight_per_s"]
    assert abs(probes["decode_64k"]["weight_per_s"] - 1e6 / terms["decode_64k"]) <= 1e-3 * 1e6 / terms["decode_64k"]
    # ring depth never changes the bytes, and for the decode class (one query token at
    # GQA <= 8) neither does the split count: those candidates are all admitted
    assert all(c["bit_identical"] for c in d["candidates"] if c["measured"] and c["splits_per_sm"] == 1)
    decode_class = [c for c in d["candidates"] if c["measured"] and c["rows_class"] == 0]
    assert any(c["splits_per_sm"] != 1 for c in decode_class)
    assert all(c["bit_identical"] and c["admitted"] for c in decode_class)
    # the tuned configuration gives the same bytes as the defaults
    out, lse = case.decode()
    assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1])
    assert case.status() == mq.MQ_OK


def _fresh_cache(w):
    return mq.Cache(w.n_kv_heads, w.head_dim, 16)


def test_tune_identity_names_device_driver_toolchain_and_build():
    from quantized_kv_decode_quantize_b200 import build as mqbuild
    w = wl.reduced("verify")
    cache = _fresh_cache(w)
    ident = mq.mq_tune_identity(cache.handle, w.n_q_heads)
    fields = dict(f.split("=", 1) for f in ident.split(";"))
    props = torch.cuda.get_device_properties(0)
    assert fields["sm"] == str(props.multi_processor_count)
    assert fields["cc"] == f"{props.major}.{props.minor}"
    assert int(fields["driver"]) > 0 and int(fields["runtime"]) > 0
    assert fields["lib"] == f"{mq.mq_version()}+{mqbuild.build_id()}"
    assert (fields["D"], fields["Hkv"], fields["Hq"]) == (str(w.head_dim), str(w.n_kv_heads), str(w.n_q_heads))
    assert fields["admit"] == "bit"
    assert mq.mq_tune_identity(cache.handle, w.n_q_heads, mq.MQ_ADMIT_ALPHA).endswith(fields["base"])
    assert "admit=alpha8;" in mq.mq_tune_identity(cache.handle, w.n_q_heads, mq.MQ_ADMIT_ALPHA)
    # the defaults the candidates are compared with are part of the identity
    mq.mq_set_decode_config(cache.handle, 0, 4, 1)
    assert mq.mq_tune_identity(cache.handle, w.n_q_heads) != ident


def test_tune_store_reused_by_the_next_load_and_searched_again_on_a_new_identity(tmp_path):
    w = wl.reduced("verify")
    store = str(tmp_path / "tune_store.tsv")
    first = _fresh_cache(w)
    ident = mq.mq_tune_identity(first.handle, w.n_q_heads)
    r1 = mq.mq_tune(first.handle, 40.0, w.n_q_heads, store_path=store)
    assert r1["status"] == mq.MQ_OK and not r1["from_store"] and r1["n_tried"] > 0
    assert mq.mq_tune_store_get(store, ident) == r1["chosen"]

    # the next load: same identity, the stored choice applied without measuring
    second = _fresh_cache(w)
    log = str(tmp_path / "tune2.json")
    r2 = mq.mq_tune(second.handle, 40.0, w.n_q_heads, log_path=log, store_path=store)
    assert r2["status"] == mq.MQ_OK and r2["from_store"]
    assert r2["n_tried"] == 0 and r2["n_rejected"] == 0 and r2["elapsed_s"] < 1.0
    assert r2["chosen"] == r1["chosen"]
    assert [mq.mq_get_decode_config(second.handle, k) for k in range(3)] == r1["chosen"]
    assert json.load(open(log))["from_store"] is True

    # a different driver on record: the identity no longer matches, so the tuner searches
    text = open(store).read()
    drv = [f for f in ident.split(";") if f.startswith("driver=")][0]
    open(store, "w").write(text.replace(drv, "driver=1"))
    third = _fresh_cache(w)
    r3 = mq.mq_tune(third.handle, 40.0, w.n_q_heads, store_path=store)
    assert r3["status"] == mq.MQ_OK and not r3["from_store"] and r3["n_tried"] > 0
    assert mq.mq_tune_store_get(store, ident) == r3["chosen"]
    assert mq.mq_tune_store_get(store, ident.replace(drv, "driver=1")) == r1["chosen"]


def test_tune_incomplete_search_is_not_stored(tmp_path):
    w = wl.reduced("verify")
    store = str(tmp_path / "tune_store.tsv")
    cache = _fresh_cache(w)
    r = mq.mq_tune(cache.handle, 0.0, w.n_q_heads, store_path=store)
    assert r["status"] == mq.MQ_TUNE_BUDGET_EXHAUSTED and not r["from_store"]
    assert not os.path.exists(store)


def test_tune_alpha_admission(tmp_path):
    """The alpha rule: a candidate is kept when at every point it moves the default
    output by at most 8 x the movement one format step of the stored cache causes."""
    w = wl.reduced("verify")
    case = GpuCase(w)
    ref_out, ref_lse = [t.clone() for t in case.decode()]
    log = str(tmp_path / "tune_alpha.json")
    r = mq.mq_tune(case.cache.handle, 40.0, w.n_q_heads, log_path=log, admission=mq.MQ_ADMIT_ALPHA)
    assert r["status"] == mq.MQ_OK
    d = json.load(open(log))
    assert d["admission"] == "alpha" and d["alpha"] == 8
    assert d["noise"] and all(n["out_median"] > 0 and n["out_zero_points"] == 0 for n in d["noise"])
    measured = [c for c in d["candidates"] if c["measured"]]
    assert measured
    for c in measured:
        assert c["admitted"] == (c["max_ratio"] <= 8.0), c
        if c["bit_identical"]:
            assert c["admitted"] and c["max_ratio"] == 0.0
    # the kept set contains the bit-identical one; the other candidates differ from the
    # default only by fp32 rounding order (another split count), which moves the output
    # by well under one storage step (measured: at most ~0.12 of the noise)
    assert sum(c["admitted"] for c in measured) >= sum(c["bit_identical"] for c in measured)
    assert max(c["max_ratio"] for c in measured if c["admitted"]) < 1.0
    out, lse = case.decode()
    assert (out - ref_out).abs().max().item() <= 1e-3 and (lse - ref_lse).abs().max().item() <= 1e-3
    assert case.status() == mq.MQ_OK


def test_tune_rejects_unknown_admission():
    w = wl.reduced("verify")
    cache = _fresh_cache(w)
    with pytest.raises(mq.MQError) as e:
        mq.mq_tune(cache.handle, 1.0, w.n_q_heads, admission=7)
    assert e.value.status == mq.MQ_ERR_INVALID_ARG
