"""Reads the library's page format back into logical (token, channel) order.

An independent restatement, in numpy, of the byte permutation documented in
include/mq.h ("Cache layout"); the tests use it to compare the codes and scales the
CUDA append kernel wrote with the CPU oracle's.  Lane L = 4g + t (g = 0..7, t = 0..3).
"""
from __future__ import annotations

import numpy as np


def page_bytes(D: int) -> int:
    return 25 * D + 32


def _k_index(D):
    idx = np.zeros((16, D), np.int64)
    for tau in range(16):
        for c in range(D):
            t, o = c // (D // 4), c % (D // 4)
            chunk = (tau // 8) * (D // 64) + o // 16
            lane = 4 * (tau % 8) + t
            idx[tau, c] = (chunk * 32 + lane) * 16 + o % 16
    return idx


def _v_index(D):
    """byte holding channels (2j, 2j+1) of token tau, for j = 0 .. D/2 - 1"""
    idx = np.zeros((16, D // 2), np.int64)
    base = 16 * D + 32
    for tau in range(16):
        t, par, tp = (tau % 8) // 2, tau % 2, tau // 8
        for j in range(D // 2):
            c = 2 * j
            q, cg = c // 32, c % 32
            gp, h = cg // 4, (cg % 4) // 2
            lane = 4 * gp + t
            w = 2 * q + tp
            idx[tau, j] = base + ((w // 4) * 32 + lane) * 16 + (w % 4) * 4 + par * 2 + h
    return idx


def _vs_index(D):
    NG = D // 32
    idx = np.zeros((16, NG), np.int64)
    for tau in range(16):
        t, hi, par = (tau % 8) // 2, tau // 8, tau % 2
        for q in range(NG):
            idx[tau, q] = ((t * NG + q) * 2 + hi) * 2 + par
    return idx


_CACHE = {}


def _maps(D):
    if D not in _CACHE:
        _CACHE[D] = (_k_index(D), _v_index(D), _vs_index(D))
    return _CACHE[D]


def check_maps_are_permutations(D):
    k, v, vs = _maps(D)
    assert sorted(k.ravel().tolist()) == list(range(16 * D))
    assert sorted(v.ravel().tolist()) == list(range(16 * D + 32, 24 * D + 32))
    assert sorted(vs.ravel().tolist()) == list(range(16 * D // 32))


def decode_pages(pages: np.ndarray, D: int):
    """pages uint8 [n, page_bytes(D)] -> kc int8 [n,16,D], ks u16 [n,16],
    vp u8 [n,16,D/2] (natural packing), vs u16 [n,16,D/32]."""
    pages = np.ascontiguousarray(pages)
    k, v, vs = _maps(D)
    kc = pages[:, k].view(np.int8)
    ks = np.ascontiguousarray(pages[:, 16 * D: 16 * D + 32]).view(np.uint16)
    vp = pages[:, v]
    vsr = np.ascontiguousarray(pages[:, 24 * D + 32: 25 * D + 32]).view(np.uint16)
    return kc, ks, vp, vsr[:, vs]


def gather_sequence(pool: np.ndarray, n_kv_heads: int, D: int, table: np.ndarray, L: int):
    """Logical cache of one sequence: kc [L,Hkv,D], ks [L,Hkv], vp [L,Hkv,D/2], vs [L,Hkv,D/32]."""
    pb = page_bytes(D)
    n_pg = (L + 15) // 16
    blocks = table[:n_pg].astype(np.int64)
    idx = (blocks[:, None] * n_kv_heads + np.arange(n_kv_heads)[None, :]).ravel()  # [n_pg*Hkv]
    pages = pool.reshape(-1, pb)[idx]
    kc, ks, vp, vs = decode_pages(pages, D)

    def arrange(a):
        a = a.reshape((n_pg, n_kv_heads, 16) + a.shape[2:])
        a = np.moveaxis(a, 2, 1).reshape((n_pg * 16, n_kv_heads) + a.shape[3:])
        return a[:L]

    return arrange(kc), arrange(ks), arrange(vp), arrange(vs)
