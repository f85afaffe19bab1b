"""The tuner's persistent store without a GPU: the file round trip, replacement of an
identity's line, identity changes, malformed lines, the atomic rewrite, and the
layout of the tuner's structs in the binding against the C header.

The deep dive's section 3 ("core mechanism 1: the 60 s first-load tuner") has the
next load reuse the stored choice without measuring and search again when the
driver or toolchain identity changes; these tests pin the host half of that (the
device half, the identity query and a stored choice applied by mq_tune, runs in
tests/test_gpu_tune.py)."""
import ctypes
import os
import subprocess

import pytest

import quantized_kv_decode_quantize_b200 as mq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

ID_A = ("dev=NVIDIA_B200;sm=148;cc=10.0;driver=12090;runtime=12090;lib=10000+0123456789abcdef;"
        "D=128;Hkv=8;Hq=32;admit=bit;base=8:1:4,8:1:4,8:1:8")


def _lines(path):
    return [l for l in open(path).read().splitlines() if l and not l.startswith("#")]


def test_missing_store_is_empty(tmp_path):
    assert mq.mq_tune_store_get(str(tmp_path / "none.tsv"), ID_A) is None


def test_round_trip(tmp_path):
    p = str(tmp_path / "store.tsv")
    mq.mq_tune_store_put(p, ID_A, [(6, 2, 4), (8, 1, 8), (4, 4, 8)], 0.93)
    assert mq.mq_tune_store_get(p, ID_A) == [(6, 2, 4), (8, 1, 8), (4, 4, 8)]
    text = open(p).read()
    assert text.startswith("# mq tuning store v2")
    assert _lines(p) == [ID_A + "\t6:2:4 8:1:8 4:4:8\t0.930000"]


def test_put_replaces_the_identity_and_keeps_the_rest(tmp_path):
    p = str(tmp_path / "store.tsv")
    other = ID_A.replace("Hq=32", "Hq=64")
    mq.mq_tune_store_put(p, ID_A, [(8, 1, 4)] * 3, 1.0)
    mq.mq_tune_store_put(p, other, [(2, 4, 8)] * 3, 0.5)
    mq.mq_tune_store_put(p, ID_A, [(3, 2, 4)] * 3, 0.8)
    lines = _lines(p)
    assert len(lines) == 2
    assert mq.mq_tune_store_get(p, ID_A) == [(3, 2, 4)] * 3
    assert mq.mq_tune_store_get(p, other) == [(2, 4, 8)] * 3
    # one header line, however many rewrites
    assert sum(l.startswith("# mq tuning store v2") for l in open(p).read().splitlines()) == 1


@pytest.mark.parametrize("field,new", [
    ("driver=12090", "driver=12080"),          # a new driver
    ("runtime=12090", "runtime=12080"),        # another CUDA toolchain
    ("lib=10000+0123456789abcdef", "lib=10000+fedcba9876543210"),   # a rebuilt library
    ("dev=NVIDIA_B200", "dev=NVIDIA_H100"),
    ("admit=bit", "admit=alpha8"),
    ("base=8:1:4,8:1:4,8:1:8", "base=4:1:4,8:1:4,8:1:8"),
    ("base=8:1:4,8:1:4,8:1:8", "base=8:1:8,8:1:4,8:1:8"),
])
def test_changed_identity_finds_nothing(tmp_path, field, new):
    p = str(tmp_path / "store.tsv")
    mq.mq_tune_store_put(p, ID_A, [(6, 2, 4)] * 3, 0.9)
    assert field in ID_A
    assert mq.mq_tune_store_get(p, ID_A.replace(field, new)) is None
    # a prefix of a stored identity is a different identity
    assert mq.mq_tune_store_get(p, ID_A[:-1]) is None


def test_malformed_or_out_of_range_lines_are_absent(tmp_path):
    p = str(tmp_path / "store.tsv")
    with open(p, "w") as f:
        f.write("# some header\n")
        f.write(ID_A + "\t9:1:4 8:1:4 8:1:8\t1.0\n")        # ring_stages 9 is out of range
        f.write(ID_A.replace("Hq=32", "Hq=8") + "\t8:3:4 8:1:4 8:1:8\t1.0\n")   # splits 3 not allowed
        f.write(ID_A.replace("Hq=32", "Hq=16") + "\t8:1:4 8:1:4\t1.0\n")        # two configs only
        f.write(ID_A.replace("Hq=32", "Hq=24") + "\t8:1:4 8:1:4 8:1:8 8:1:4\t1.0\n")
        f.write(ID_A.replace("Hq=32", "Hq=40") + "\t8:1:6 8:1:4 8:1:8\t1.0\n")  # 6 softmax warps
        f.write(ID_A.replace("Hq=32", "Hq=48") + "\t8:1 8:1 8:1\t1.0\n")        # the two-field format
        f.write("garbage line without tabs\n")
    for hq in ("Hq=32", "Hq=8", "Hq=16", "Hq=24", "Hq=40", "Hq=48"):
        assert mq.mq_tune_store_get(p, ID_A.replace("Hq=32", hq)) is None
    # put keeps foreign lines and replaces only its own identity
    mq.mq_tune_store_put(p, ID_A, [(2, 1, 4), (2, 2, 8), (2, 4, 8)], 0.7)
    assert mq.mq_tune_store_get(p, ID_A) == [(2, 1, 4), (2, 2, 8), (2, 4, 8)]
    text = open(p).read()
    assert "garbage line without tabs" in text and "# some header" in text
    assert "9:1:4 8:1:4 8:1:8" not in text


def test_invalid_arguments(tmp_path):
    p = str(tmp_path / "store.tsv")
    for bad in ("a\tb", "a\nb", ""):
        with pytest.raises(mq.MQError) as e:
            mq.mq_tune_store_put(p, bad, [(8, 1, 4)] * 3, 1.0)
        assert e.value.status == mq.MQ_ERR_INVALID_ARG
        with pytest.raises(mq.MQError):
            mq.mq_tune_store_get(p, bad)
    with pytest.raises(mq.MQError) as e:
        mq.mq_tune_store_put(p, ID_A, [(8, 1, 4), (8, 1, 4), (1, 1, 8)], 1.0)   # 1 stage is below the range
    assert e.value.status == mq.MQ_ERR_INVALID_ARG
    assert not os.path.exists(p)


def test_unwritable_store_is_an_io_error(tmp_path):
    p = str(tmp_path / "no_such_dir" / "store.tsv")
    with pytest.raises(mq.MQError) as e:
        mq.mq_tune_store_put(p, ID_A, [(8, 1, 4)] * 3, 1.0)
    assert e.value.status == mq.MQ_ERR_IO


def test_rewrite_leaves_no_temporary_files(tmp_path):
    p = str(tmp_path / "store.tsv")
    for i in range(5):
        mq.mq_tune_store_put(p, ID_A.replace("Hq=32", f"Hq={8 * (i + 1)}"), [(8, 1, 4)] * 3, 1.0)
    assert sorted(os.listdir(tmp_path)) == ["store.tsv"]
    assert len(_lines(p)) == 5


def test_null_cache_identity_is_invalid():
    p = mq._tune_params(0.0, 8)
    buf = ctypes.create_string_buffer(512)
    assert mq.lib.mq_tune_identity(None, ctypes.byref(p), buf, 512) == mq.MQ_ERR_INVALID_ARG


def test_struct_layout_matches_the_header(tmp_path):
    """sizeof / offsetof of the tuner structs as a C compiler sees include/mq.h equal
    the binding's ctypes layout."""
    src = r'''
#include <stdio.h>
#include <stddef.h>
#include "mq.h"
#define F(T, m) printf(#T "." #m " %zu\n", offsetof(T, m));
int main(void) {
    printf("mq_tune_params %zu\n", sizeof(mq_tune_params));
    printf("mq_tune_result %zu\n", sizeof(mq_tune_result));
    printf("mq_decode_config %zu\n", sizeof(mq_decode_config));
    F(mq_tune_params, budget_s) F(mq_tune_params, n_q_heads) F(mq_tune_params, log_path)
    F(mq_tune_params, store_path) F(mq_tune_params, admission) F(mq_tune_params, alpha)
    F(mq_tune_result, chosen) F(mq_tune_result, cost) F(mq_tune_result, n_tried) F(mq_tune_result, n_rejected)
    F(mq_tune_result, n_skipped) F(mq_tune_result, elapsed_s) F(mq_tune_result, from_store)
    return 0;
}
'''
    c = tmp_path / "layout.c"
    c.write_text(src)
    exe = str(tmp_path / "layout")
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(c), "-o", exe], check=True)
    got = dict(l.rsplit(" ", 1) for l in subprocess.run([exe], capture_output=True, text=True,
                                                         check=True).stdout.splitlines())
    assert int(got["mq_tune_params"]) == ctypes.sizeof(mq.mq_tune_params)
    assert int(got["mq_tune_result"]) == ctypes.sizeof(mq.mq_tune_result)
    assert int(got["mq_decode_config"]) == ctypes.sizeof(mq.mq_decode_config)
    for struct in (mq.mq_tune_params, mq.mq_tune_result):
        for name, _ in struct._fields_:
            assert int(got[f"{struct.__name__}.{name}"]) == getattr(struct, name).offset, name
