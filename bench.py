"""Benchmark of the quantized-KV decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {mq,reference}] [--workload long]

A step is one pass of the whole hot path over the workload: quantize-on-append of
the step's new K/V token(s) into the paged cache (mq_kv_append), then split-K decode
attention of the step's query token(s) against the whole cache (mq_decode_attn).
The default workload is the 64K-context single-stream decode (batch 1, 32 q / 8 kv
heads, head_dim 128, 65536 cached tokens including the step's own, shuffled
16-token blocks, bf16 inputs).  Inputs are seeded synthetic tensors.

Timing: W untimed warm-up steps, then exactly K steps between a barrier +
torch.cuda.synchronize() on both sides, replayed from a CUDA graph of steps; the
caches read by successive steps rotate over copies that together exceed 4x the L2
size, so no step finds its KV in L2.  The timed graph holds the steps as a user runs
them: no event sits between the kernels, whose launches overlap (each kernel lets the
next one start its set-up).  The decode kernel's own duration (the roofline figure)
comes from CUDA events around each decode call in a second graph of the same steps,
replayed right after the timed region.  Multi-GPU (torchrun): every rank runs its own
replica (the work shards over independent sessions; no collective on the data path),
the time is the max over ranks, and the value is the whole job's bytes / that time.

`e2e` times the same step through the C ABI from pinned HOST buffers: per step one
H2D copy of the step's inputs (q and the new K/V, packed in one buffer), the two
calls, one D2H copy of the results (out and lse, packed), and a stream synchronize.  `--impl reference` runs the CPU oracle (the reference arm) on
a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized-KV decode attention: KV GB/s (% of HBM peak) and µs/step at 64K ctx"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=500)
    ap.add_argument("--impl", default="mq", choices=["mq", "reference"])
    ap.add_argument("--workload", default="long",
                    choices=["tiny", "long", "prefix", "verify", "mixed", "prefill_4k", "prefill_64k"])
    ap.add_argument("--graph-steps", type=int, default=0, help="steps per captured graph (0: one rotation)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--tune", type=float, default=0.0, help="run mq_tune with this budget (s) first")
    ap.add_argument("--decode-config", default="",
                    help="ring_stages,splits_per_sm,softmax_warps for every row class (before --tune)")
    ap.add_argument("--cascade", action="store_true",
                    help="decode with mq_decode_attn_cascade over the workload's shared prefix")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0=None, t1=None):
        rows = [r for t, r in self.rows if (t0 is None or t >= t0) and (t1 is None or t <= t1)]
        if not rows:
            rows = [r for _, r in self.rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 5 + i and r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def load_tensor_peak():
    """Dense bf16 (= fp16) tensor TFLOP/s: the measured burst figure, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def prefill_flops(seq_lens, n_q, n_q_heads, head_dim):
    """Algorithmic FLOPs of causal prefill attention: query j of n sees L - n + j + 1
    keys; 2 * D flops for its score and 2 * D for its share of the output per key."""
    vis = sum(n * (L - n) + n * (n + 1) // 2 for L, n in zip(seq_lens, n_q))
    return 4 * head_dim * n_q_heads * vis


def run_prefill(args, rank, world, local):
    """Prompt prefill over the quantized cache (mq_prefill_attn): a whole 4K- or
    64K-token prompt per rank, timed like the decode step (CUDA graph of launches,
    events around the timed region); algorithmic TFLOP/s against the tensor peak."""
    import numpy as np
    import torch
    import torch.distributed as dist

    import quantized_kv_decode_quantize_b200 as mq
    import workloads as wl

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    L = 4096 if args.workload == "prefill_4k" else 65536
    w = wl.Workload(args.workload, 32, 8, 128, [L], [L], [L],
                    note=f"one {L}-token prompt, 32 q / 8 kv heads (GQA 4), D 128, bf16, shuffled 16-token blocks")
    inp = wl.make_inputs(w)
    tabs_np, n_blocks = wl.block_tables(w)
    cache = mq.Cache(w.n_kv_heads, w.head_dim, n_blocks)
    tab = torch.from_numpy(tabs_np[0]).to(dev)
    i32 = dict(dtype=torch.int32, device=dev)
    mq.mq_kv_append(cache.handle, inp.own_k[0].to(dev), inp.own_v[0].to(dev), mq.MQ_BF16, 1, L,
                    torch.tensor([0, L], **i32), torch.tensor([0], **i32), tab, w.max_blocks())
    q = inp.q.to(dev).contiguous()
    lens = torch.tensor([L], **i32)
    out = torch.empty((L, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)
    lse = torch.empty((L, w.n_q_heads), dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(w.head_dim)

    def call(stream):
        mq.mq_prefill_attn(cache.handle, q, mq.MQ_BF16, 1, w.n_q_heads, L, L, L, tab, w.max_blocks(), lens, lens,
                           scale, out, lse, stream)

    stream = torch.cuda.Stream(dev)
    S = max(1, min(args.steps, 4))
    with torch.cuda.stream(stream):
        for _ in range(2):
            call(stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(S):
            call(stream)
    sampler = ClockSampler(local)
    sampler.start()
    with torch.cuda.stream(stream):
        for _ in range(max(1, math.ceil(args.warmup / S))):
            g.replay()
    torch.cuda.synchronize(dev)
    reps, rem = divmod(args.steps, S)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for _ in range(reps):
            g.replay()
        for _ in range(rem):
            call(stream)
        t1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.stop()
    ms = max_over_ranks(t0.elapsed_time(t1), dev)
    assert mq.mq_device_status(cache.handle) == mq.MQ_OK
    flops = prefill_flops(w.seq_lens, w.n_q, w.n_q_heads, w.head_dim)
    tflops = world * flops * args.steps / (ms * 1e-3) / 1e12
    peak, kind = load_tensor_peak()
    if rank == 0:
        clocks = sampler.summary()
        print(json.dumps({
            "metric": "prefill attention over the K8/V4 cache: algorithmic TFLOP/s", "value": tflops,
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp16 tensor-core operands (exact bf16 q, exact key codes, values hi + lo), fp32 accumulate",
            "data": "synthetic",
            "config": {"workload": w.name, "note": w.note, "prompt_tokens": L, "flops_per_step": flops,
                       "parallelism": f"replica x{world}"},
            "roofline": {"bound": "tensor", "achieved": tflops / world, "peak": peak, "unit": "TFLOP/s",
                         "frac": tflops / world / peak, "peak_kind": peak_kind_note(kind),
                         "traffic": None, "kernel": "mq::prefill_kernel"},
            "gpu_launches": args.steps,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"],
                       "samples": clocks["samples"]},
        }), flush=True)
    del g
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def peak_kind_note(kind):
    return (f"{kind} dense bf16 (fp16 runs at the same rate); the kernel issues 1.5x the algorithmic "
            f"MMA work (values as hi + lo)")


def packed_buffer(specs, device, pin=None):
    """One byte buffer holding tensors of the given (shape, dtype), each at a 256-byte
    aligned offset (pinned when on the host, unless pin is False); returns the buffer and
    the views."""
    import torch
    offs, off = [], 0
    for shape, dt in specs:
        offs.append(off)
        n = math.prod(shape) * torch.empty((), dtype=dt).element_size()
        off = (off + n + 255) // 256 * 256
    buf = torch.zeros(off, dtype=torch.uint8, device=device)
    if (device == "cpu") if pin is None else pin:
        buf = buf.pin_memory()
    views = []
    for (shape, dt), o in zip(specs, offs):
        n = math.prod(shape) * torch.empty((), dtype=dt).element_size()
        views.append(buf[o: o + n].view(dt).view(shape))
    return buf, views


def kernel_source_hash():
    """Hash of the decode kernel's own sources (the kernel, its device helpers and its
    parameter block) without comments and blank space: DRAM counters taken on another
    version of the code are stale, an edited comment does not change the kernel."""
    import hashlib
    import re
    h = hashlib.sha256()
    d = os.path.join(ROOT, "quantized_kv_decode_quantize_b200", "csrc")
    for n in ("mq_decode_small.cu", "mq_decode_common.cuh", "mq_decode.cu", "mq_device.cuh", "mq_tc.cuh",
              "mq_kernels.h"):
        with open(os.path.join(d, n)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)   # block comments
        src = re.sub(r"//[^\n]*", " ", src)                 # line comments
        h.update(n.encode() + " ".join(src.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload_name: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload_name)
    if not e or e.get("kernel_source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------------
def graph_steps(copies: int, steps: int, override: int = 0) -> int:
    """Steps captured in one CUDA graph: a whole number of rotations over the cache
    copies (about 24 steps), but never more than the timed steps, so that the timed
    region holds at least one replay and the events recorded around each decode call
    inside it give the kernel duration at any --steps."""
    S = override or copies * max(1, math.ceil(24 / copies))
    return max(1, min(S, steps))


def max_over_ranks(x: float, device) -> float:
    """The max of x over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return x
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def algorithmic_bytes_unique(w, bytes_per_token_head: int):
    """Decode bytes with a shared prefix counted once (the HBM floor of the shared-prefix
    workload); equal to the logical figure without a shared prefix."""
    dec, _ = algorithmic_bytes(w, bytes_per_token_head)
    return dec - (w.n_seqs - 1) * w.shared_prefix * w.n_kv_heads * bytes_per_token_head if w.shared_prefix else dec


def algorithmic_bytes(w, bytes_per_token_head: int):
    """Bytes a decode launch must move: every (token, kv-head) of every sequence once
    (a shared prefix counted once per sequence: the logical figure), q, out, lse and
    the block-table entries read; plus the append of the step's tokens (bf16 K/V
    read, quantized form written)."""
    esz = 4 if w.dtype == "f32" else 2
    kv = sum(w.seq_lens) * w.n_kv_heads * bytes_per_token_head
    q = w.total_q * w.n_q_heads * w.head_dim * esz
    out = w.total_q * w.n_q_heads * (w.head_dim + 1) * 4
    bt = sum((L + 15) // 16 for L in w.seq_lens) * 4 + 8 * w.n_seqs
    decode = kv + q + out + bt
    n_app = sum(w.n_append)
    append = n_app * w.n_kv_heads * (2 * w.head_dim * esz + bytes_per_token_head)
    return decode, append


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle on the host cores, on a bounded sample of
    the workload per step."""
    import numpy as np
    import torch

    import oracle
    import workloads as wl

    if rank != 0:
        return
    if args.workload.startswith("prefill"):
        run_reference_prefill(args, world)
        return
    w = wl.FULL[args.workload]()
    inp = wl.make_inputs(w)
    cores = oracle.max_threads()
    bpt = oracle.kv_bytes_per_token_head(w.head_dim)
    # sample: query heads of kv-head 0 of sequence 0 over a token slice sized so that the
    # whole run stays within a few minutes
    L = w.seq_lens[0]
    G = w.n_q_heads // w.n_kv_heads
    kf = inp.seq_k(0)[:, :1].float().numpy()
    vf = inp.seq_v(0)[:, :1].float().numpy()
    kc, ks = oracle.quantize_k(kf)
    vp, vs = oracle.quantize_v(vf)
    q = inp.q[: w.n_q[0], :G].float().numpy().astype(np.float64)
    scale = 1.0 / math.sqrt(w.head_dim)

    def step(n_tok):
        # quantize the step's token (the append) and attend over the first n_tok tokens
        oracle.quantize_k(kf[L - 1: L])
        oracle.quantize_v(vf[L - 1: L])
        oracle.attention_quant(q, kc[:n_tok], ks[:n_tok], vp[:n_tok], vs[:n_tok], scale, cores)

    t = time.perf_counter()
    step(min(L, 8192))
    per_tok = (time.perf_counter() - t) / min(L, 8192)
    budget = 150.0
    n_tok = int(max(w.n_q[0] + 16, min(L, budget / max(1, args.steps + args.warmup) / max(per_tok, 1e-9))))
    for _ in range(args.warmup):
        step(n_tok)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step(n_tok)
    dt = time.perf_counter() - t0
    bytes_step = n_tok * bpt
    val = bytes_step * args.steps / dt / 1e9
    line = {
        "metric": METRIC, "value": val, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "note": w.note},
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: quantize of the step's K/V token, then fp64 attention of the "
                                   f"{G} q-heads of kv-head 0 over the first {n_tok} of {L} tokens"},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_reference_prefill(args, world):
    """The reference arm of the prefill workloads: the oracle's fp64 attention over the
    quantized cache for a bounded sample of the prompt's query rows (the last query
    tokens, which see the whole prompt) on the host cores; algorithmic TFLOP/s."""
    import numpy as np

    import oracle
    import workloads as wl

    L = 4096 if args.workload == "prefill_4k" else 65536
    w = wl.Workload(args.workload, 32, 8, 128, [L], [L], [L])
    inp = wl.make_inputs(w)
    cores = oracle.max_threads()
    kc, ks = oracle.quantize_k(inp.own_k[0].float().numpy())
    vp, vs = oracle.quantize_v(inp.own_v[0].float().numpy())
    scale = 1.0 / math.sqrt(w.head_dim)
    n_s = 4 if L > 8192 else 32          # sampled query tokens per step (all 32 heads each)
    q = inp.q[L - n_s:].float().numpy().astype(np.float64)

    def step():
        oracle.attention_quant(q, kc, ks, vp, vs, scale, cores)

    for _ in range(min(args.warmup, 1)):
        step()
    steps = max(1, min(args.steps, 5))
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    dt = time.perf_counter() - t0
    flops = prefill_flops([L], [n_s], w.n_q_heads, w.head_dim)
    val = flops * steps / dt / 1e12
    sample = (f"per step: fp64 attention of the last {n_s} query tokens (32 q-heads each) of the {L}-token "
              f"prompt over the quantized cache, {steps} step(s)")
    print(json.dumps({
        "metric": "prefill attention over the K8/V4 cache: algorithmic TFLOP/s", "value": val, "unit": "TFLOP/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": dt / steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference", "config": {"workload": w.name, "prompt_tokens": L},
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def cpu_baseline(w, inp, gpu_out=None, gpu_lse=None, steps_budget_s=20.0):
    """The oracle as it stands, on all host cores: full decode steps of the workload
    (every sequence, every head) until ~steps_budget_s of work; GB/s of KV read.

    The first step's oracle outputs also give the accuracy figures of the GPU result
    (`gpu_out`, `gpu_lse`: numpy copies of the bench's last decode): max-abs error
    against the oracle's fp64 attention over the same quantized cache (the parity
    bar, 1e-3), and max-abs / relative-L2 error against fp64 attention over the
    original, unquantized K/V (reported, not gated).  Returns (baseline, accuracy)."""
    import numpy as np

    import oracle

    cores = oracle.max_threads()
    bpt = oracle.kv_bytes_per_token_head(w.head_dim)
    codes = []
    for b in range(w.n_seqs):
        kc, ks = oracle.quantize_k(inp.seq_k(b).float().numpy())
        vp, vs = oracle.quantize_v(inp.seq_v(b).float().numpy())
        codes.append((kc, ks, vp, vs))
    q = inp.q.float().numpy().astype(np.float64)
    qoff = np.concatenate([[0], np.cumsum(w.n_q)]).astype(int)
    scale = 1.0 / math.sqrt(w.head_dim)
    ref_out = np.empty((w.total_q, w.n_q_heads, w.head_dim))
    ref_lse = np.empty((w.total_q, w.n_q_heads))
    n = 0
    t0 = time.perf_counter()
    while True:
        for b in range(w.n_seqs):
            o, l = oracle.attention_quant(q[qoff[b]: qoff[b + 1]], *codes[b], scale, cores)
            if n == 0:
                ref_out[qoff[b]: qoff[b + 1]], ref_lse[qoff[b]: qoff[b + 1]] = o, l
        n += 1
        if time.perf_counter() - t0 > steps_budget_s or n >= 50:
            break
    dt = time.perf_counter() - t0
    base = {"value": sum(w.seq_lens) * w.n_kv_heads * bpt * n / dt / 1e9, "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": f"{n} full decode step(s) of {w.name} (all sequences and heads, fp64 attention over the "
                      f"quantized cache), {dt:.1f} s"}
    acc = None
    if gpu_out is not None:
        unq = np.empty_like(ref_out)
        for b in range(w.n_seqs):
            o, _ = oracle.attention(q[qoff[b]: qoff[b + 1]], inp.seq_k(b).float().numpy(),
                                    inp.seq_v(b).float().numpy(), scale, cores)
            unq[qoff[b]: qoff[b + 1]] = o
        d_q = np.abs(gpu_out - ref_out)
        d_u = gpu_out - unq
        acc = {"vs_oracle_quantized": {"max_abs_out": float(d_q.max()),
                                       "max_abs_lse": float(np.abs(gpu_lse - ref_lse).max()),
                                       "tolerance": 1e-3},
               "vs_unquantized_fp64": {"max_abs_out": float(np.abs(d_u).max()),
                                       "rel_l2_out": float(np.linalg.norm(d_u) / np.linalg.norm(unq)),
                                       "note": "reported, not gated: K int8 / V int4 quantization error"},
               "sample": f"every output of the bench's last decode step ({w.total_q} query token(s) x "
                         f"{w.n_q_heads} q-heads x {w.head_dim})"}
    return base, acc


def run_mq(args, rank, world, local):
    import numpy as np
    import torch
    import torch.distributed as dist

    import quantized_kv_decode_quantize_b200 as mq
    import workloads as wl

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    w = wl.FULL[args.workload]()
    inp = wl.make_inputs(w)
    props = torch.cuda.get_device_properties(dev)
    l2 = props.L2_cache_size
    bpt = mq.mq_page_bytes(w.head_dim) // 16
    copy_bytes = w.kv_bytes_unique(bpt)
    copies = max(2, math.ceil(4 * l2 / copy_bytes))
    tabs_np, n_blocks = wl.block_tables(w, copies=copies)
    cache = mq.Cache(w.n_kv_heads, w.head_dim, n_blocks)
    tabs = torch.from_numpy(tabs_np).to(dev)
    dt_code = mq.MQ_F32 if w.dtype == "f32" else mq.MQ_BF16
    i32 = dict(dtype=torch.int32, device=dev)

    # history: everything but the step's own appended tokens, in every copy
    hist_k, hist_v, step_k, step_v = [], [], [], []
    for b in range(w.n_seqs):
        n_app = w.n_append[b]
        kb, vb = inp.own_k[b], inp.own_v[b]
        hist_k.append(kb[: kb.shape[0] - n_app])
        hist_v.append(vb[: vb.shape[0] - n_app])
        step_k.append(kb[kb.shape[0] - n_app:])
        step_v.append(vb[vb.shape[0] - n_app:])
    for c in range(copies):
        if w.shared_prefix:
            mq.mq_kv_append(cache.handle, inp.prefix_k.to(dev), inp.prefix_v.to(dev), dt_code, 1, w.shared_prefix,
                            torch.tensor([0, w.shared_prefix], **i32), torch.tensor([0], **i32), tabs[c][:1].contiguous(),
                            w.max_blocks())
        n_h = [int(x.shape[0]) for x in hist_k]
        if sum(n_h):
            mq.mq_kv_append(cache.handle, torch.cat(hist_k).to(dev), torch.cat(hist_v).to(dev), dt_code, w.n_seqs,
                            sum(n_h), torch.tensor(np.concatenate([[0], np.cumsum(n_h)]).astype(np.int32), device=dev),
                            torch.tensor([w.shared_prefix] * w.n_seqs, **i32), tabs[c], w.max_blocks())
    torch.cuda.synchronize(dev)
    assert mq.mq_device_status(cache.handle) == mq.MQ_OK

    if args.decode_config:
        r_, s_, w_ = (int(x) for x in args.decode_config.split(","))
        for k in range(3):
            mq.mq_set_decode_config(cache.handle, k, r_, s_, max(w_, 8) if k == 2 else min(w_, 8))
    if args.tune > 0:
        mq.mq_tune(cache.handle, args.tune, w.n_q_heads)

    n_new = [int(x.shape[0]) for x in step_k]
    # the step's inputs (q, new K, new V) share one device buffer and its results (out,
    # lse) another, so that a step from host memory is one copy each way
    h_k_src, h_v_src = torch.cat(step_k).contiguous(), torch.cat(step_v).contiguous()
    in_specs = [(tuple(inp.q.shape), inp.q.dtype), (tuple(h_k_src.shape), h_k_src.dtype),
                (tuple(h_v_src.shape), h_v_src.dtype)]
    res_specs = [((w.total_q, w.n_q_heads, w.head_dim), torch.float32), ((w.total_q, w.n_q_heads), torch.float32)]
    d_in, (q, new_k, new_v) = packed_buffer(in_specs, dev)
    d_res, (out, lse) = packed_buffer(res_specs, dev)
    q.copy_(inp.q.to(dev))
    new_k.copy_(h_k_src.to(dev))
    new_v.copy_(h_v_src.to(dev))
    cu_new = torch.tensor(np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32), device=dev)
    start = torch.tensor([L - a for L, a in zip(w.seq_lens, w.n_append)], **i32)
    seq_lens = torch.tensor(w.seq_lens, **i32)
    n_q = torch.tensor(w.n_q, **i32)
    cascade = bool(args.cascade and w.shared_prefix)
    if cascade:
        ws_bytes = mq.mq_decode_cascade_workspace_bytes(cache.handle, w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                                                        w.max_seq_len, w.shared_prefix)
    else:
        ws_bytes = mq.mq_decode_workspace_bytes(cache.handle, w.n_seqs, w.n_q_heads, w.max_q, w.max_seq_len)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    scale = 1.0 / math.sqrt(w.head_dim)
    tab_c = [tabs[c] for c in range(copies)]

    def step(c, stream, ev=None, append_only=False):
        mq.mq_kv_append(cache.handle, new_k, new_v, dt_code, w.n_seqs, sum(n_new), cu_new, start, tab_c[c],
                        w.max_blocks(), stream)
        if append_only:
            return
        if ev is not None:
            ev[0].record(stream)
        if cascade:
            mq.mq_decode_attn_cascade(cache.handle, q, dt_code, w.n_seqs, w.n_q_heads, w.total_q, w.max_q,
                                      w.max_seq_len, tab_c[c], w.max_blocks(), seq_lens, n_q, w.shared_prefix, scale,
                                      out, lse, ws, ws_bytes, stream)
        else:
            mq.mq_decode_attn(cache.handle, q, dt_code, w.n_seqs, w.n_q_heads, w.total_q, w.max_q, w.max_seq_len,
                              tab_c[c], w.max_blocks(), seq_lens, n_q, scale, out, lse, ws, ws_bytes, stream)
        if ev is not None:
            ev[1].record(stream)

    # ---- capture S steps (one rotation over the copies, or more) in a graph ----
    # Two graphs of the same steps: `g` as a user runs them (the timed region), and
    # `g_ev` with an event pair around every decode call (the kernel durations).  Events
    # stay out of the timed steps: an event node between two kernels ends the
    # programmatic overlap of the append and the decode kernels.
    S = graph_steps(copies, args.steps, args.graph_steps)
    stream = torch.cuda.Stream(dev)
    evs = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
           for _ in range(S)]
    with torch.cuda.stream(stream):
        for i in range(3):                        # eager warm-up before capture
            step(i % copies, stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(S):
            step(i % copies, stream)
    g_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ev, stream=stream):
        for i in range(S):
            step(i % copies, stream, evs[i])
    torch.cuda.synchronize(dev)

    # warm-up: W steps (whole graphs, rounded up), then ~1 s of untimed soak for clocks
    sampler = ClockSampler(local)
    sampler.start()
    for _ in range(max(1, math.ceil(args.warmup / S))):
        g.replay()
    torch.cuda.synchronize(dev)
    t_soak = time.time()
    while time.time() - t_soak < 1.0:
        g.replay()
        torch.cuda.synchronize(dev)
    reps, rem = divmod(args.steps, S)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for _ in range(reps):
            g.replay()
        for i in range(rem):                      # the remainder eagerly: exactly K steps
            step(i % copies, stream)
        t_end.record(stream)
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    sampler.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    # decode-kernel durations: the same steps replayed right after the timed region, with
    # events around each decode call on the launching stream (first replay warms up)
    kern_ms = []
    with torch.cuda.stream(stream):
        for rep in range(3):
            g_ev.replay()
            stream.synchronize()
            if rep > 0:
                kern_ms += [a.elapsed_time(b) for a, b in evs]
    elapsed_ms = max_over_ranks(elapsed_ms, dev)
    assert mq.mq_device_status(cache.handle, stream) == mq.MQ_OK

    dec_bytes, app_bytes = algorithmic_bytes(w, bpt)
    step_bytes = dec_bytes + app_bytes
    value = world * step_bytes * args.steps / (elapsed_ms * 1e-3) / 1e9
    peak, peak_kind = load_peaks()
    kern_avg = statistics.mean(kern_ms) if kern_ms else None
    # the roofline counts each byte that must come from HBM once (a shared prefix once)
    dec_unique = algorithmic_bytes_unique(w, bpt)
    achieved = dec_unique / (kern_avg * 1e-3) / 1e9 if kern_avg else None

    # ---- the append alone, outside the timed region (events around each launch) ----
    app_ms = []
    with torch.cuda.stream(stream):
        for i in range(20):
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            step(i % copies, stream, append_only=True)
            a1.record(stream)
            a1.synchronize()
            if i >= 4:
                app_ms.append(a0.elapsed_time(a1))
    app_avg = statistics.median(app_ms) if app_ms else None

    # ---- verification against one decode step of the same sequences (several query
    # tokens per sequence): each sequence's last query token alone, on the same caches;
    # decode + merge by CUDA events, each call on a copy no recent call has read ----
    verify_vs_decode = None
    if w.max_q > 1 and not cascade:
        last = torch.as_tensor(np.cumsum(w.n_q) - 1, dtype=torch.long, device=dev)
        q1 = q[last].contiguous()
        nq1 = torch.ones(w.n_seqs, **i32)
        out1 = torch.empty((w.n_seqs, w.n_q_heads, w.head_dim), dtype=torch.float32, device=dev)
        lse1 = torch.empty((w.n_seqs, w.n_q_heads), dtype=torch.float32, device=dev)
        ws1_bytes = mq.mq_decode_workspace_bytes(cache.handle, w.n_seqs, w.n_q_heads, 1, w.max_seq_len)
        ws1 = torch.zeros(max(ws1_bytes, 256), dtype=torch.uint8, device=dev)
        v_ms, d_ms = [], []
        with torch.cuda.stream(stream):
            for i in range(24):
                e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                e[0].record(stream)
                mq.mq_decode_attn(cache.handle, q, dt_code, w.n_seqs, w.n_q_heads, w.total_q, w.max_q, w.max_seq_len,
                                  tab_c[(2 * i) % copies], w.max_blocks(), seq_lens, n_q, scale, out, lse, ws,
                                  ws_bytes, stream)
                e[1].record(stream)
                mq.mq_decode_attn(cache.handle, q1, dt_code, w.n_seqs, w.n_q_heads, w.n_seqs, 1, w.max_seq_len,
                                  tab_c[(2 * i + 1) % copies], w.max_blocks(), seq_lens, nq1, scale, out1, lse1, ws1,
                                  ws1_bytes, stream)
                e[2].record(stream)
                e[2].synchronize()
                if i >= 4:
                    v_ms.append(e[0].elapsed_time(e[1]))
                    d_ms.append(e[1].elapsed_time(e[2]))
        assert mq.mq_device_status(cache.handle, stream) == mq.MQ_OK
        v_med, d_med = statistics.median(v_ms), statistics.median(d_ms)
        verify_vs_decode = {"verify_us": v_med * 1e3, "decode_us": d_med * 1e3, "ratio": v_med / d_med,
                            "decode": "the same sequences and caches, each sequence's last query token alone "
                                      "(one decode step); decode + merge kernels by CUDA events, 20 calls each"}

    def pct(xs, q):
        xs = sorted(xs)
        return xs[min(len(xs) - 1, int(round(q * (len(xs) - 1))))] if xs else None

    if cascade:   # prefix pass + suffix pass + the two-way merge
        n_decode_kernels = (mq.mq_decode_kernel_count(cache.handle, 1, w.n_q_heads, w.total_q, w.shared_prefix)
                            + mq.mq_decode_kernel_count(cache.handle, w.n_seqs, w.n_q_heads, w.max_q,
                                                        w.max_seq_len - w.shared_prefix) + 1)
    else:
        n_decode_kernels = mq.mq_decode_kernel_count(cache.handle, w.n_seqs, w.n_q_heads, w.max_q, w.max_seq_len)

    # ---- e2e through the C ABI from pinned host buffers ----
    e2e = None
    if not args.no_e2e:
        h_in, (hq_, hk_, hv_) = packed_buffer(in_specs, "cpu")
        hq_.copy_(inp.q)
        hk_.copy_(h_k_src)
        hv_.copy_(h_v_src)
        h_res, _ = packed_buffer(res_specs, "cpu")
        K2 = min(args.steps, 2000)
        with torch.cuda.stream(stream):
            for i in range(min(args.warmup, 50)):
                d_in.copy_(h_in, non_blocking=True)
                step(i % copies, stream)
                h_res.copy_(d_res, non_blocking=True)
                stream.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(dev)
            e0 = time.perf_counter()
            for i in range(K2):
                d_in.copy_(h_in, non_blocking=True)
                step(i % copies, stream)
                h_res.copy_(d_res, non_blocking=True)
                stream.synchronize()
            e_dt = time.perf_counter() - e0
        e_dt = max_over_ranks(e_dt, dev)
        h2d = h_in.numel()
        d2h = h_res.numel()
        e2e = {"value": world * step_bytes * K2 / e_dt / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": K2, "ms_per_step": e_dt / K2 * 1e3}

    if rank == 0:
        rows_total = w.n_q_heads // w.n_kv_heads * w.max_q
        cls = 0 if rows_total <= 8 else (1 if rows_total <= 16 or w.head_dim == 256 else 2)
        cfg = mq.mq_get_decode_config(cache.handle, cls)
        clocks = sampler.summary()
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8/int4 KV, fp32 accumulate",
            "data": "synthetic",
            "config": {"workload": w.name, "note": w.note, "n_seqs": w.n_seqs, "seq_lens_sum": int(sum(w.seq_lens)),
                       "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
                       "l2_policy": f"inputs larger than L2: {copies} rotating cache copies "
                                    f"({copies * copy_bytes / 1e6:.0f} MB, L2 {l2 / 1e6:.0f} MB)",
                       "parallelism": f"replica x{world}",
                       "step": "mq_kv_append + " + ("mq_decode_attn_cascade" if cascade else "mq_decode_attn"),
                       "decode_config": cfg, "us_per_step": elapsed_ms / args.steps * 1e3,
                       "pct_of_8TBps": 100 * value / world / 8000.0,
                       "decode_bytes_logical": dec_bytes,
                       "decode_bytes_unique": dec_unique,
                       "append_bytes": app_bytes,
                       "append_us_median": app_avg * 1e3 if app_avg else None,
                       "append_GBps": app_bytes / (app_avg * 1e-3) / 1e9 if app_avg else None,
                       **({"verify_vs_decode": verify_vs_decode} if verify_vs_decode else {})},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": (achieved / peak) if achieved else None, "peak_kind": peak_kind,
                         "traffic": ncu_traffic(w.name), "kernel": "mq::decode_small_kernel",
                         "bytes_per_launch": dec_unique, "kernel_us_mean": kern_avg * 1e3 if kern_avg else None,
                         "kernel_us_median": statistics.median(kern_ms) * 1e3 if kern_ms else None,
                         "kernel_us_p10": pct(kern_ms, 0.1) * 1e3 if kern_ms else None,
                         "kernel_us_p90": pct(kern_ms, 0.9) * 1e3 if kern_ms else None,
                         "kernels_timed": ("cascade: two decode passes + merge_two_kernel" if cascade else
                                           "decode kernel + merge_kernel" if n_decode_kernels == 2 else
                                           "decode kernel"),
                         "kernel_timing": f"CUDA events around each decode call on its stream, {len(kern_ms)} calls "
                                          f"in two replays of the timed step graph right after the timed region "
                                          f"(events there end the append/decode launch overlap, so the decode "
                                          f"runs alone); step-level rate "
                                          f"{dec_unique / (elapsed_ms / args.steps * 1e-3) / 1e9:.0f} GB/s"},
            "e2e": e2e,
            "gpu_launches": (1 + n_decode_kernels) * args.steps,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"], "reasons": clocks["reasons"],
                       "samples": clocks["samples"]},
            "wall_s": wall1 - wall0,
        }
        if not args.no_cpu_baseline and world == 1:
            torch.cuda.synchronize(dev)
            line["cpu_baseline"], line["accuracy"] = cpu_baseline(w, inp, out.cpu().numpy().astype(np.float64),
                                                                  lse.cpu().numpy().astype(np.float64))
        print(json.dumps(line), flush=True)
    del g, g_ev
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.workload.startswith("prefill"):
        run_prefill(args, rank, world, local)
        return
    run_mq(args, rank, world, local)


if __name__ == "__main__":
    main()
