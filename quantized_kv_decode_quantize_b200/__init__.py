"""Python binding of the mq C ABI (``include/mq.h``): argument marshalling only.

Every function here has the name of the C entry point it calls and passes plain
integers (device pointers, sizes) and the current CUDA stream through ctypes.
Torch tensors are accepted wherever the C function takes a device pointer; only
their ``data_ptr()`` is used.  All computation happens in ``libmq.so``'s CUDA
kernels; there is no fallback path: if the library is missing this module raises
ImportError (build it with ``python quantized_kv_decode_quantize_b200/build.py``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmq.so")

MQ_OK, MQ_ERR_INVALID_ARG, MQ_ERR_UNSUPPORTED, MQ_ERR_CAPACITY = 0, 1, 2, 3
MQ_ERR_WORKSPACE, MQ_ERR_CUDA, MQ_ERR_DEVICE, MQ_TUNE_BUDGET_EXHAUSTED = 4, 5, 6, 7
MQ_ERR_IO = 8
MQ_ADMIT_BIT_IDENTICAL, MQ_ADMIT_ALPHA = 0, 1
MQ_F32, MQ_BF16, MQ_F16 = 0, 1, 2
MQ_PAGE_TOKENS = 16


class mq_cache_desc(ctypes.Structure):
    _fields_ = [("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("page_tokens", ctypes.c_int32),
                ("n_blocks", ctypes.c_int64), ("pool", ctypes.c_void_p), ("pool_bytes", ctypes.c_size_t)]


class mq_decode_config(ctypes.Structure):
    _fields_ = [("ring_stages", ctypes.c_int32), ("splits_per_sm", ctypes.c_int32), ("softmax_warps", ctypes.c_int32)]

    def as_tuple(self):
        return (self.ring_stages, self.splits_per_sm, self.softmax_warps)


class mq_tune_params(ctypes.Structure):
    _fields_ = [("budget_s", ctypes.c_double), ("n_q_heads", ctypes.c_int32), ("log_path", ctypes.c_char_p),
                ("store_path", ctypes.c_char_p), ("admission", ctypes.c_int32), ("alpha", ctypes.c_double)]


class mq_tune_result(ctypes.Structure):
    _fields_ = [("chosen", mq_decode_config * 3), ("cost", ctypes.c_double), ("n_tried", ctypes.c_int32),
                ("n_rejected", ctypes.c_int32), ("n_skipped", ctypes.c_int32), ("elapsed_s", ctypes.c_double),
                ("from_store", ctypes.c_int32)]


class MQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {mq_status_string(status)} (status {status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python quantized_kv_decode_quantize_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "mq_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "mq_version": ([], i32),
        "mq_page_bytes": ([i32], sz),
        "mq_cache_pool_bytes": ([i32, i32, i64], sz),
        "mq_cache_create": ([ctypes.POINTER(mq_cache_desc), ctypes.POINTER(P)], ctypes.c_int),
        "mq_cache_destroy": ([P], ctypes.c_int),
        "mq_kv_append": ([P, P, P, ctypes.c_int, i32, i32, P, P, P, i32, P], ctypes.c_int),
        "mq_kv_export": ([P, i32, i32, P, P, P, i32, P, P, P, P, P], ctypes.c_int),
        "mq_decode_workspace_bytes": ([P, i32, i32, i32, i32], sz),
        "mq_decode_kernel_count": ([P, i32, i32, i32, i32], i32),
        "mq_decode_attn": ([P, P, ctypes.c_int, i32, i32, i32, i32, i32, P, i32, P, P, ctypes.c_float, P, P, P, sz, P],
                           ctypes.c_int),
        "mq_prefill_attn": ([P, P, ctypes.c_int, i32, i32, i32, i32, i32, P, i32, P, P, ctypes.c_float, P, P, P],
                            ctypes.c_int),
        "mq_decode_attn_static": ([P, P, ctypes.c_int, i32, i32, i32, i32, i32, P, i32, P, P, ctypes.c_float, P, P,
                                   P], ctypes.c_int),
        "mq_decode_cascade_workspace_bytes": ([P, i32, i32, i32, i32, i32, i32], sz),
        "mq_decode_attn_cascade": ([P, P, ctypes.c_int, i32, i32, i32, i32, i32, P, i32, P, P, i32, ctypes.c_float,
                                    P, P, P, sz, P], ctypes.c_int),
        "mq_draft_ngram": ([P, i32, P, i32, i32, i32, P, P, P], ctypes.c_int),
        "mq_get_decode_config": ([P, i32, ctypes.POINTER(mq_decode_config)], ctypes.c_int),
        "mq_set_decode_config": ([P, i32, ctypes.POINTER(mq_decode_config)], ctypes.c_int),
        "mq_tune": ([P, ctypes.POINTER(mq_tune_params), ctypes.POINTER(mq_tune_result)], ctypes.c_int),
        "mq_tune_identity": ([P, ctypes.POINTER(mq_tune_params), ctypes.c_char_p, sz], ctypes.c_int),
        "mq_tune_store_get": ([ctypes.c_char_p, ctypes.c_char_p, ctypes.POINTER(mq_decode_config),
                               ctypes.POINTER(i32)], ctypes.c_int),
        "mq_tune_store_put": ([ctypes.c_char_p, ctypes.c_char_p, ctypes.POINTER(mq_decode_config), ctypes.c_double],
                              ctypes.c_int),
        "mq_device_status": ([P, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


lib = _load()


def _ptr(x):
    """Device pointer of a tensor / int / None as a ctypes value."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str, ok=(MQ_OK,)):
    if status not in ok:
        raise MQError(status, where)
    return status


# ---- the C entry points -------------------------------------------------------
def mq_status_string(status: int) -> str:
    return lib.mq_status_string(status).decode()


def mq_version() -> int:
    return lib.mq_version()


def mq_page_bytes(head_dim: int) -> int:
    return lib.mq_page_bytes(head_dim)


def mq_cache_pool_bytes(n_kv_heads: int, head_dim: int, n_blocks: int) -> int:
    return lib.mq_cache_pool_bytes(n_kv_heads, head_dim, n_blocks)


def mq_cache_create(n_kv_heads: int, head_dim: int, n_blocks: int, pool, pool_bytes: int,
                    page_tokens: int = MQ_PAGE_TOKENS) -> int:
    d = mq_cache_desc(n_kv_heads, head_dim, page_tokens, n_blocks, _ptr(pool), pool_bytes)
    h = ctypes.c_void_p()
    _check(lib.mq_cache_create(ctypes.byref(d), ctypes.byref(h)), "mq_cache_create")
    return h.value


def mq_cache_destroy(cache: int) -> None:
    _check(lib.mq_cache_destroy(cache), "mq_cache_destroy")


def mq_kv_append(cache: int, k, v, dtype: int, n_seqs: int, n_tokens: int, cu_new, start_pos, block_table,
                 max_blocks_per_seq: int, stream=None) -> None:
    _check(lib.mq_kv_append(cache, _ptr(k), _ptr(v), dtype, n_seqs, n_tokens, _ptr(cu_new), _ptr(start_pos),
                            _ptr(block_table), max_blocks_per_seq, _stream(stream)), "mq_kv_append")


def mq_kv_export(cache: int, n_seqs: int, n_tokens: int, cu_tok, start_pos, block_table, max_blocks_per_seq: int,
                 k_codes, k_scales, v_packed, v_scales, stream=None) -> None:
    _check(lib.mq_kv_export(cache, n_seqs, n_tokens, _ptr(cu_tok), _ptr(start_pos), _ptr(block_table),
                            max_blocks_per_seq, _ptr(k_codes), _ptr(k_scales), _ptr(v_packed), _ptr(v_scales),
                            _stream(stream)), "mq_kv_export")


def mq_decode_workspace_bytes(cache: int, n_seqs: int, n_q_heads: int, max_q_per_seq: int, max_seq_len: int) -> int:
    return lib.mq_decode_workspace_bytes(cache, n_seqs, n_q_heads, max_q_per_seq, max_seq_len)


def mq_decode_kernel_count(cache: int, n_seqs: int, n_q_heads: int, max_q_per_seq: int, max_seq_len: int) -> int:
    return lib.mq_decode_kernel_count(cache, n_seqs, n_q_heads, max_q_per_seq, max_seq_len)


def mq_decode_attn(cache: int, q, q_dtype: int, n_seqs: int, n_q_heads: int, total_q: int, max_q_per_seq: int,
                   max_seq_len: int, block_table, max_blocks_per_seq: int, seq_lens, n_q_per_seq,
                   softmax_scale: float, out, lse, workspace, workspace_bytes: int, stream=None) -> None:
    _check(lib.mq_decode_attn(cache, _ptr(q), q_dtype, n_seqs, n_q_heads, total_q, max_q_per_seq, max_seq_len,
                              _ptr(block_table), max_blocks_per_seq, _ptr(seq_lens), _ptr(n_q_per_seq),
                              float(softmax_scale), _ptr(out), _ptr(lse), _ptr(workspace), workspace_bytes,
                              _stream(stream)), "mq_decode_attn")


def mq_prefill_attn(cache: int, q, q_dtype: int, n_seqs: int, n_q_heads: int, total_q: int, max_q_per_seq: int,
                    max_seq_len: int, block_table, max_blocks_per_seq: int, seq_lens, n_q_per_seq, softmax_scale: float,
                    out, lse, stream=None) -> None:
    _check(lib.mq_prefill_attn(cache, _ptr(q), q_dtype, n_seqs, n_q_heads, total_q, max_q_per_seq, max_seq_len,
                               _ptr(block_table), max_blocks_per_seq, _ptr(seq_lens), _ptr(n_q_per_seq),
                               float(softmax_scale), _ptr(out), _ptr(lse), _stream(stream)), "mq_prefill_attn")


def mq_decode_attn_static(cache: int, q, q_dtype: int, n_seqs: int, n_q_heads: int, total_q: int,
                          max_q_per_seq: int, max_seq_len: int, block_table, max_blocks_per_seq: int, seq_lens,
                          n_q_per_seq, softmax_scale: float, out, lse, stream=None) -> None:
    _check(lib.mq_decode_attn_static(cache, _ptr(q), q_dtype, n_seqs, n_q_heads, total_q, max_q_per_seq, max_seq_len,
                                     _ptr(block_table), max_blocks_per_seq, _ptr(seq_lens), _ptr(n_q_per_seq),
                                     float(softmax_scale), _ptr(out), _ptr(lse), _stream(stream)),
           "mq_decode_attn_static")


def mq_decode_cascade_workspace_bytes(cache: int, n_seqs: int, n_q_heads: int, total_q: int, max_q_per_seq: int,
                                      max_seq_len: int, prefix_len: int) -> int:
    return lib.mq_decode_cascade_workspace_bytes(cache, n_seqs, n_q_heads, total_q, max_q_per_seq, max_seq_len,
                                                 prefix_len)


def mq_decode_attn_cascade(cache: int, q, q_dtype: int, n_seqs: int, n_q_heads: int, total_q: int,
                           max_q_per_seq: int, max_seq_len: int, block_table, max_blocks_per_seq: int, seq_lens,
                           n_q_per_seq, prefix_len: int, softmax_scale: float, out, lse, workspace,
                           workspace_bytes: int, stream=None) -> None:
    _check(lib.mq_decode_attn_cascade(cache, _ptr(q), q_dtype, n_seqs, n_q_heads, total_q, max_q_per_seq,
                                      max_seq_len, _ptr(block_table), max_blocks_per_seq, _ptr(seq_lens),
                                      _ptr(n_q_per_seq), prefix_len, float(softmax_scale), _ptr(out), _ptr(lse),
                                      _ptr(workspace), workspace_bytes, _stream(stream)), "mq_decode_attn_cascade")


def mq_draft_ngram(tokens, max_len: int, seq_lens, n_seqs: int, ngram: int, max_draft: int, drafts, n_drafts,
                   stream=None) -> None:
    _check(lib.mq_draft_ngram(_ptr(tokens), max_len, _ptr(seq_lens), n_seqs, ngram, max_draft, _ptr(drafts),
                              _ptr(n_drafts), _stream(stream)), "mq_draft_ngram")


def mq_get_decode_config(cache: int, rows_class: int) -> tuple:
    c = mq_decode_config()
    _check(lib.mq_get_decode_config(cache, rows_class, ctypes.byref(c)), "mq_get_decode_config")
    return c.as_tuple()


def mq_set_decode_config(cache: int, rows_class: int, ring_stages: int, splits_per_sm: int,
                         softmax_warps: int | None = None) -> None:
    """softmax_warps None keeps the class's current value."""
    if softmax_warps is None:
        softmax_warps = mq_get_decode_config(cache, rows_class)[2]
    c = mq_decode_config(ring_stages, splits_per_sm, softmax_warps)
    _check(lib.mq_set_decode_config(cache, rows_class, ctypes.byref(c)), "mq_set_decode_config")


def _tune_params(budget_s, n_q_heads, log_path=None, store_path=None, admission=MQ_ADMIT_BIT_IDENTICAL, alpha=0.0):
    return mq_tune_params(float(budget_s), n_q_heads, log_path.encode() if log_path else None,
                          store_path.encode() if store_path else None, admission, float(alpha))


def mq_tune(cache: int, budget_s: float, n_q_heads: int, log_path: str | None = None, store_path: str | None = None,
            admission: int = MQ_ADMIT_BIT_IDENTICAL, alpha: float = 0.0) -> dict:
    p = _tune_params(budget_s, n_q_heads, log_path, store_path, admission, alpha)
    r = mq_tune_result()
    st = _check(lib.mq_tune(cache, ctypes.byref(p), ctypes.byref(r)), "mq_tune",
                ok=(MQ_OK, MQ_TUNE_BUDGET_EXHAUSTED))
    return {"status": st, "chosen": [r.chosen[i].as_tuple() for i in range(3)], "cost": r.cost,
            "n_tried": r.n_tried, "n_rejected": r.n_rejected, "n_skipped": r.n_skipped, "elapsed_s": r.elapsed_s,
            "from_store": bool(r.from_store)}


def mq_tune_identity(cache: int, n_q_heads: int, admission: int = MQ_ADMIT_BIT_IDENTICAL, alpha: float = 0.0) -> str:
    p = _tune_params(0.0, n_q_heads, admission=admission, alpha=alpha)
    buf = ctypes.create_string_buffer(512)
    _check(lib.mq_tune_identity(cache, ctypes.byref(p), buf, len(buf)), "mq_tune_identity")
    return buf.value.decode()


def mq_tune_store_get(path: str, identity: str):
    """The stored [(ring_stages, splits_per_sm)] * 3 for `identity`, or None."""
    cfg = (mq_decode_config * 3)()
    found = ctypes.c_int32(0)
    _check(lib.mq_tune_store_get(path.encode(), identity.encode(), cfg, ctypes.byref(found)), "mq_tune_store_get")
    return [cfg[i].as_tuple() for i in range(3)] if found.value else None


def mq_tune_store_put(path: str, identity: str, chosen, cost: float) -> None:
    cfg = (mq_decode_config * 3)(*[mq_decode_config(*c) for c in chosen])
    _check(lib.mq_tune_store_put(path.encode(), identity.encode(), cfg, float(cost)), "mq_tune_store_put")


def mq_device_status(cache: int, stream=None) -> int:
    return lib.mq_device_status(cache, _stream(stream))


# ---- a convenience owner of a pool + handle (torch supplies the memory) --------
class Cache:
    """Owns a device pool (a torch uint8 tensor) and the mq_cache handle over it."""

    def __init__(self, n_kv_heads: int, head_dim: int, n_blocks: int, device="cuda"):
        import torch
        self.n_kv_heads, self.head_dim, self.n_blocks = n_kv_heads, head_dim, n_blocks
        self.pool_bytes = mq_cache_pool_bytes(n_kv_heads, head_dim, n_blocks)
        if self.pool_bytes == 0:
            raise MQError(MQ_ERR_INVALID_ARG, "mq_cache_pool_bytes")
        self.pool = torch.empty(self.pool_bytes, dtype=torch.uint8, device=device)
        self.handle = mq_cache_create(n_kv_heads, head_dim, n_blocks, self.pool, self.pool_bytes)

    def close(self):
        if self.handle:
            mq_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def page_bytes(self) -> int:
        return mq_page_bytes(self.head_dim)
