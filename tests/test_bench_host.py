"""bench.py's host logic without a GPU: the validity hash of the committed DRAM
counters (comments and blank space do not count, code does) and the lookup that
turns a stale or missing record into null."""
import json
import os
import shutil

import bench

FILES = ("mq_decode_small.cu", "mq_decode_common.cuh", "mq_decode.cu", "mq_device.cuh", "mq_tc.cuh", "mq_kernels.h")


def _tree(tmp_path):
    root = tmp_path / "repo"
    d = root / "quantized_kv_decode_quantize_b200" / "csrc"
    d.mkdir(parents=True)
    for n in FILES:
        shutil.copy(os.path.join(bench.ROOT, "quantized_kv_decode_quantize_b200", "csrc", n), d / n)
    (root / "profiles").mkdir()
    return root, d


def test_hash_ignores_comments_and_blank_space(tmp_path, monkeypatch):
    root, d = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    h0 = bench.kernel_source_hash()
    p = d / "mq_decode_small.cu"
    src = p.read_text()
    p.write_text("// a new comment line\n/* and a block\n comment */\n" + src.replace("\n", "\n\n", 5))
    assert bench.kernel_source_hash() == h0
    assert "static constexpr int NWB = 2;" in src
    p.write_text(src.replace("static constexpr int NWB = 2;", "static constexpr int NWB = 3;"))
    assert bench.kernel_source_hash() != h0


def test_traffic_record_is_null_when_stale_or_missing(tmp_path, monkeypatch):
    root, d = _tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.ncu_traffic("long_decode_64k") is None                  # no record file
    rec = {"long_decode_64k": {"dram_bytes_per_launch": 123, "kernel_source_hash": bench.kernel_source_hash()}}
    (root / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    assert bench.ncu_traffic("long_decode_64k") == 123
    assert bench.ncu_traffic("tiny_decode_4k") is None                   # another workload
    p = d / "mq_tc.cuh"
    p.write_text(p.read_text() + "\nnamespace mq { constexpr int kChanged = 1; }\n")
    assert bench.ncu_traffic("long_decode_64k") is None                  # the kernel changed


def test_committed_record_names_the_bench_workload():
    with open(os.path.join(bench.ROOT, "profiles", "ncu_traffic.json")) as f:
        rec = json.load(f)
    e = rec["long_decode_64k"]
    assert e["dram_bytes_per_launch"] == e["dram_bytes_read"] + e["dram_bytes_write"]
    assert "--clock-control none" in e["command"]


def test_graph_never_longer_than_the_timed_steps():
    """The kernel events live inside graph replays: at any --steps the timed region
    must hold at least one whole replay (the driver times 20 steps against a default
    graph of 24)."""
    for copies in (2, 3, 6, 8):
        for steps in (1, 3, 5, 20, 23, 24, 25, 200, 20000):
            S = bench.graph_steps(copies, steps)
            assert 1 <= S <= steps
            assert divmod(steps, S)[0] >= 1
    assert bench.graph_steps(6, 20000) == 24
    assert bench.graph_steps(6, 20) == 20
    assert bench.graph_steps(6, 20000, override=12) == 12


def test_packed_buffer_views_are_aligned_and_disjoint():
    """The e2e step's inputs and results each live in one buffer (one copy each way): every
    view starts on a 256-byte boundary, views do not overlap, and writes land in place."""
    import torch
    import bench
    specs = [((3, 32, 128), torch.bfloat16), ((5, 8, 128), torch.float32), ((7,), torch.float16)]
    buf, views = bench.packed_buffer(specs, "cpu", pin=False)
    spans = []
    for (shape, dt), v in zip(specs, views):
        off = v.data_ptr() - buf.data_ptr()
        assert off % 256 == 0 and tuple(v.shape) == shape and v.dtype == dt and v.is_contiguous()
        spans.append((off, off + v.numel() * v.element_size()))
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:])) and spans[-1][1] <= buf.numel()
    for i, v in enumerate(views):
        v.fill_(i + 1)
    for i, v in enumerate(views):
        assert bool((v == i + 1).all())
