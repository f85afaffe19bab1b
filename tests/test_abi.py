"""The C-ABI library without a GPU: it loads, exports every entry point include/mq.h
declares, and its host-side validation answers before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

import quantized_kv_decode_quantize_b200 as mq
from quantized_kv_decode_quantize_b200 import build as mqbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mq.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("mq_cache_create", "mq_cache_destroy", "mq_kv_append", "mq_decode_attn", "mq_tune",
              "mq_decode_workspace_bytes", "mq_status_string", "mq_device_status", "mq_decode_attn_static",
              "mq_decode_attn_cascade", "mq_decode_cascade_workspace_bytes", "mq_draft_ngram", "mq_tune_identity",
              "mq_tune_store_get", "mq_tune_store_put", "mq_decode_kernel_count", "mq_kv_export", "mq_prefill_attn"):
        assert n in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", mqbuild.LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(mq_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(mq.lib, n)


def test_header_compiles_as_c():
    """The header is plain C (no CUDA or C++ types in the signatures)."""
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-x", "c", "-"],
                       input='#include "mq.h"\nint main(void){return 0;}\n', text=True, capture_output=True,
                       cwd=os.path.join(ROOT, "include"))
    assert r.returncode == 0, r.stderr


def test_sizes():
    assert mq.mq_page_bytes(128) == 3232 and mq.mq_page_bytes(256) == 6432
    assert mq.mq_page_bytes(64) == 0 and mq.mq_page_bytes(512) == 0
    assert mq.mq_cache_pool_bytes(8, 128, 4096) == 4096 * 8 * 3232
    assert mq.mq_cache_pool_bytes(0, 128, 10) == 0 and mq.mq_cache_pool_bytes(8, 128, 0) == 0
    # less than half of fp16 K+V per (token, kv-head)
    assert 3232 / 16 < 0.5 * 4 * 128 and 6432 / 16 < 0.5 * 4 * 256


def test_status_strings():
    for s in range(9):
        assert mq.mq_status_string(s) and mq.mq_status_string(s) != "unknown status"
    assert mq.mq_status_string(99) == "unknown status"
    assert mq.mq_version() >= 10000


def _create(**kw):
    d = dict(n_kv_heads=8, head_dim=128, n_blocks=16, pool=256 * 1024, pool_bytes=16 * 8 * 3232, page_tokens=16)
    d.update(kw)
    desc = mq.mq_cache_desc(d["n_kv_heads"], d["head_dim"], d["page_tokens"], d["n_blocks"], d["pool"],
                            d["pool_bytes"])
    h = ctypes.c_void_p()
    return mq.lib.mq_cache_create(ctypes.byref(desc), ctypes.byref(h)), h.value


@pytest.mark.parametrize("kw,status", [
    (dict(pool=0), mq.MQ_ERR_INVALID_ARG),
    (dict(pool=256 * 1024 + 16), mq.MQ_ERR_INVALID_ARG),
    (dict(n_kv_heads=0), mq.MQ_ERR_INVALID_ARG),
    (dict(n_blocks=0), mq.MQ_ERR_INVALID_ARG),
    (dict(head_dim=64), mq.MQ_ERR_UNSUPPORTED),
    (dict(page_tokens=32), mq.MQ_ERR_UNSUPPORTED),
    (dict(pool_bytes=100), mq.MQ_ERR_CAPACITY),
])
def test_cache_create_validation(kw, status):
    st, h = _create(**kw)
    assert st == status and h is None


def test_null_arguments_rejected_before_cuda():
    assert mq.lib.mq_cache_create(None, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.lib.mq_cache_destroy(None) == mq.MQ_OK
    assert mq.lib.mq_kv_append(None, 1, 1, 1, 1, 1, 1, 1, 1, 1, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.lib.mq_kv_export(None, 1, 1, 1, 1, 1, 1, 1, 1, 1, 1, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.lib.mq_decode_attn(None, 1, 1, 1, 8, 1, 1, 16, 1, 1, 1, 1, 0.1, 16, None, 256, 1 << 20, None) \
        == mq.MQ_ERR_INVALID_ARG
    assert mq.lib.mq_decode_workspace_bytes(None, 1, 8, 1, 16) == 0
    assert mq.lib.mq_decode_cascade_workspace_bytes(None, 1, 8, 1, 1, 64, 16) == 0
    for bad in ((None, 8, 1, 1, 2, 1, 1), (1, 0, 1, 1, 2, 1, 1), (1, 8, 1, 0, 2, 1, 1), (1, 8, 1, 1, 0, 1, 1),
                (1, 8, 1, 1, 65, 1, 1), (1, 8, 1, 1, 2, 0, 1)):
        t, ml, sl, ns, n, k, d = bad
        assert mq.lib.mq_draft_ngram(t, ml, sl, ns, n, k, d, 1, None) == mq.MQ_ERR_INVALID_ARG
    assert mq.lib.mq_decode_attn_cascade(None, 1, 1, 1, 8, 1, 1, 64, 1, 4, 1, 1, 16, 0.1, 16, None, 256, 1 << 20,
                                         None) == mq.MQ_ERR_INVALID_ARG
    assert mq.lib.mq_device_status(None, None) == mq.MQ_ERR_INVALID_ARG
    cfg = mq.mq_decode_config()
    assert mq.lib.mq_get_decode_config(None, 0, ctypes.byref(cfg)) == mq.MQ_ERR_INVALID_ARG
    p, r = mq.mq_tune_params(1.0, 8, None), mq.mq_tune_result()
    assert mq.lib.mq_tune(None, ctypes.byref(p), ctypes.byref(r)) == mq.MQ_ERR_INVALID_ARG
