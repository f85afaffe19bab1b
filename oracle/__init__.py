"""CPU oracle for the K8/V4 quantized-KV decode step — TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
(and its ``--impl reference`` arm) may import this package.  The product path —
the CUDA library under ``quantized_kv_decode_quantize_b200/`` — never imports it,
and the two share no code.

The arithmetic lives in ``mq_oracle.c`` (plain scalar C, fp32 IEEE quantization,
fp64 attention); this module only marshals numpy arrays through ctypes.  What each
function computes, and which page passage it follows, is stated in the C file's
header: the blog.123qwe.co.kr deep dive on magnitudedev/magnitude, section 5
(core mechanism 3: speculative decoding, quantized KV, prefix sharing) names the
``attention_decode_k8v4`` unit and its codec (K 8 bit, V 4 bit, group 32, f16
scale); the pages give no formula, so the exact arithmetic is a fixed reading
of them, stated in the C file's header.

``draft_ngram`` (history-based drafting, the deep dive's section 5 drafting
guarantees) is pinned by hand-worked cases and a cross-check against Python's
``bytes.rfind``.

Parity status: quantization and dequantized attention are pinned by
``tests/test_oracle_*.py`` (hand-worked cases, brute force, closed forms,
invariants, a library cross-check).  The error against unquantized attention is
reported, not gated: parity unpinned for that figure (the pages give no number).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mq_oracle.c")
_LIB = os.path.join(_HERE, "libmq_oracle.so")

CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False, src: str = _SRC, out: str = _LIB, extra_flags=()) -> str:
    """Compile the oracle C source into a shared library (gcc, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, *extra_flags, "-o", tmp, src, "-lm"], check=True)
        os.replace(tmp, out)
    return out


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class OracleLib:
    """ctypes view of one build of the oracle library (the default build, or a
    test's deliberately mutated copy)."""

    def __init__(self, path: str):
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.mqo_f32_to_f16_bits.argtypes = [ctypes.c_float]
        L.mqo_f32_to_f16_bits.restype = ctypes.c_uint16
        L.mqo_f16_bits_to_f64.argtypes = [ctypes.c_uint16]
        L.mqo_f16_bits_to_f64.restype = dbl
        L.mqo_bf16_bits_to_f32.argtypes = [ctypes.c_uint16]
        L.mqo_bf16_bits_to_f32.restype = ctypes.c_float
        L.mqo_quantize_k.argtypes = [P, i64, i32, P, P]
        L.mqo_quantize_v.argtypes = [P, i64, i32, P, P]
        L.mqo_dequantize_k.argtypes = [P, P, i64, i32, P]
        L.mqo_dequantize_v.argtypes = [P, P, i64, i32, P]
        L.mqo_attention_f64.argtypes = [P, P, P, i32, i32, i32, i32, i64, dbl, P, P, P, i32]
        L.mqo_attention_quant_f64.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i64, dbl, P, P, i32]
        L.mqo_draft_ngram.argtypes = [P, i32, i32, i32, P]
        L.mqo_draft_ngram.restype = i32
        L.mqo_max_threads.restype = i32
        for f in ("mqo_quantize_k", "mqo_quantize_v", "mqo_dequantize_k", "mqo_dequantize_v",
                  "mqo_attention_f64", "mqo_attention_quant_f64"):
            getattr(L, f).restype = None
        self.L = L

    # ---- scalar conversions --------------------------------------------------
    def f32_to_f16_bits(self, x) -> np.ndarray:
        """IEEE binary16 round-to-nearest-even of each fp32 value, as uint16 bits."""
        x = np.asarray(x, dtype=np.float32)
        f = self.L.mqo_f32_to_f16_bits
        return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint16).reshape(x.shape)

    def f16_bits_to_f64(self, b) -> np.ndarray:
        b = np.asarray(b, dtype=np.uint16)
        f = self.L.mqo_f16_bits_to_f64
        return np.array([f(int(v)) for v in b.ravel()], dtype=np.float64).reshape(b.shape)

    def bf16_bits_to_f32(self, b) -> np.ndarray:
        b = np.asarray(b, dtype=np.uint16)
        f = self.L.mqo_bf16_bits_to_f32
        return np.array([f(int(v)) for v in b.ravel()], dtype=np.float32).reshape(b.shape)

    # ---- quantization --------------------------------------------------------
    def quantize_k(self, x: np.ndarray):
        """x [..., D] fp32 -> (codes int8 [..., D], scale bits uint16 [...])."""
        x = _c(x, np.float32)
        D = x.shape[-1]
        codes = np.empty(x.shape, np.int8)
        scales = np.empty(x.shape[:-1], np.uint16)
        self.L.mqo_quantize_k(_p(x), x.size // D, D, _p(codes), _p(scales))
        return codes, scales

    def quantize_v(self, x: np.ndarray):
        """x [..., D] fp32 -> (packed uint8 [..., D/2], scale bits uint16 [..., D/32])."""
        x = _c(x, np.float32)
        D = x.shape[-1]
        assert D % 32 == 0
        packed = np.empty(x.shape[:-1] + (D // 2,), np.uint8)
        scales = np.empty(x.shape[:-1] + (D // 32,), np.uint16)
        self.L.mqo_quantize_v(_p(x), x.size // D, D, _p(packed), _p(scales))
        return packed, scales

    def dequantize_k(self, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
        codes = _c(codes, np.int8)
        scales = _c(scales, np.uint16)
        D = codes.shape[-1]
        out = np.empty(codes.shape, np.float64)
        self.L.mqo_dequantize_k(_p(codes), _p(scales), codes.size // D, D, _p(out))
        return out

    def dequantize_v(self, packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
        packed = _c(packed, np.uint8)
        scales = _c(scales, np.uint16)
        D = packed.shape[-1] * 2
        out = np.empty(packed.shape[:-1] + (D,), np.float64)
        self.L.mqo_dequantize_v(_p(packed), _p(scales), packed.size // (D // 2), D, _p(out))
        return out

    # ---- attention -----------------------------------------------------------
    def attention(self, q, k, v, scale: float, n_threads: int = 1, return_weights: bool = False):
        """One sequence, fp64.  q [n_q, Hq, D]; k, v [L, Hkv, D] in logical order.

        Query j sees tokens 0 .. L - n_q + j.  Returns out [n_q, Hq, D], lse
        [n_q, Hq] (and weights [n_q, Hq, L] when asked)."""
        q, k, v = _c(q, np.float64), _c(k, np.float64), _c(v, np.float64)
        n_q, Hq, D = q.shape
        L, Hkv, D2 = k.shape
        assert D2 == D and v.shape == k.shape and Hq % Hkv == 0 and 1 <= n_q <= L
        out = np.empty((n_q, Hq, D), np.float64)
        lse = np.empty((n_q, Hq), np.float64)
        w = np.empty((n_q, Hq, L), np.float64) if return_weights else None
        self.L.mqo_attention_f64(_p(q), _p(k), _p(v), n_q, Hq, Hkv, D, L, float(scale), _p(out), _p(lse), _p(w),
                                 int(n_threads))
        return (out, lse, w) if return_weights else (out, lse)

    def attention_quant(self, q, kc, ks, vp, vs, scale: float, n_threads: int = 1):
        """Same as ``attention`` over the quantized cache (codes + fp16 scale bits,
        logical order): kc [L, Hkv, D] int8, ks [L, Hkv] u16, vp [L, Hkv, D/2] u8,
        vs [L, Hkv, D/32] u16."""
        q = _c(q, np.float64)
        kc, ks, vp, vs = _c(kc, np.int8), _c(ks, np.uint16), _c(vp, np.uint8), _c(vs, np.uint16)
        n_q, Hq, D = q.shape
        L, Hkv, D2 = kc.shape
        assert D2 == D and ks.shape == (L, Hkv) and vp.shape == (L, Hkv, D // 2) and vs.shape == (L, Hkv, D // 32)
        assert Hq % Hkv == 0 and 1 <= n_q <= L
        out = np.empty((n_q, Hq, D), np.float64)
        lse = np.empty((n_q, Hq), np.float64)
        self.L.mqo_attention_quant_f64(_p(q), _p(kc), _p(ks), _p(vp), _p(vs), n_q, Hq, Hkv, D, L, float(scale),
                                       _p(out), _p(lse), int(n_threads))
        return out, lse

    def draft_ngram(self, tokens, n: int, k: int) -> np.ndarray:
        """History-based drafts: the up to k tokens that followed the most recent
        earlier occurrence of the last n tokens of `tokens` (int32 [L])."""
        t = _c(np.asarray(tokens), np.int32)
        out = np.zeros(max(int(k), 1), np.int32)
        cnt = self.L.mqo_draft_ngram(_p(t), int(t.shape[0]), int(n), int(k), _p(out))
        return out[:cnt].copy()

    def max_threads(self) -> int:
        return int(self.L.mqo_max_threads())

    def kv_bytes_per_token_head(self, D: int) -> int:
        """Bytes the quantized form of one (token, kv-head) occupies, measured from
        the oracle's own outputs (codes + K scale + packed V + V scales)."""
        x = np.zeros((1, D), np.float32)
        kc, ks = self.quantize_k(x)
        vp, vs = self.quantize_v(x)
        return kc.nbytes + ks.nbytes + vp.nbytes + vs.nbytes


_default = None


def lib() -> OracleLib:
    global _default
    if _default is None:
        _default = OracleLib(build())
    return _default


def f32_to_f16_bits(x):
    return lib().f32_to_f16_bits(x)


def f16_bits_to_f64(b):
    return lib().f16_bits_to_f64(b)


def bf16_bits_to_f32(b):
    return lib().bf16_bits_to_f32(b)


def quantize_k(x):
    return lib().quantize_k(x)


def quantize_v(x):
    return lib().quantize_v(x)


def dequantize_k(codes, scales):
    return lib().dequantize_k(codes, scales)


def dequantize_v(packed, scales):
    return lib().dequantize_v(packed, scales)


def attention(q, k, v, scale, n_threads=1, return_weights=False):
    return lib().attention(q, k, v, scale, n_threads, return_weights)


def attention_quant(q, kc, ks, vp, vs, scale, n_threads=1):
    return lib().attention_quant(q, kc, ks, vp, vs, scale, n_threads)


def draft_ngram(tokens, n, k):
    return lib().draft_ngram(tokens, n, k)


def max_threads() -> int:
    return lib().max_threads()


def kv_bytes_per_token_head(D: int) -> int:
    return lib().kv_bytes_per_token_head(D)
