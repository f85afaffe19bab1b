"""Reads the library's page format back into logical (token, channel) order.

An independent restatement, in numpy, of the page layout documented in include/mq.h
("Cache layout"); the tests use it to compare the codes and scales the CUDA append
kernel wrote with the CPU oracle's.  A page holds two records of 8 tokens each
(tokens 0-7, then 8-15), each record rec_bytes(D) = 12.5 D + 16 bytes:
K codes as 8 x 16-byte blocks, then one 32-bit V word per channel with the 8 tokens'
nibbles, then the 8 K scales, then the 8 x D/32 V scales.
"""
from __future__ import annotations

import numpy as np


def page_bytes(D: int) -> int:
    return 25 * D + 32


def rec_bytes(D: int) -> int:
    return 25 * D // 2 + 16


def _k_index(D):
    R = rec_bytes(D)
    idx = np.zeros((16, D), np.int64)
    for tau in range(16):
        for c in range(D):
            idx[tau, c] = (tau // 8) * R + (c // 16) * 128 + (tau % 8) * 16 + c % 16
    return idx


def _v_index(D):
    """(byte offset of the 32-bit word, bit position of the nibble) of V code (tau, c)"""
    R = rec_bytes(D)
    word = np.zeros((16, D), np.int64)
    bit = np.zeros((16, D), np.int64)
    for tau in range(16):
        for c in range(D):
            word[tau, c] = (tau // 8) * R + 8 * D + 4 * c
            bit[tau, c] = 4 * ((tau % 8) // 2) + 16 * (tau % 2)
    return word, bit


def _ks_index(D):
    R = rec_bytes(D)
    return np.array([(tau // 8) * R + 12 * D + 2 * (tau % 8) for tau in range(16)], np.int64)


def _vs_index(D):
    R, G = rec_bytes(D), D // 32
    idx = np.zeros((16, G), np.int64)
    for tau in range(16):
        for g in range(G):
            idx[tau, g] = (tau // 8) * R + 12 * D + 16 + 2 * ((tau % 8) * G + g)
    return idx


_CACHE = {}


def _maps(D):
    if D not in _CACHE:
        _CACHE[D] = (_k_index(D), _v_index(D), _ks_index(D), _vs_index(D))
    return _CACHE[D]


def check_maps_are_permutations(D):
    """Every byte of a page belongs to exactly one field, every V bit to one code."""
    k, (vw, vb), ks, vs = _maps(D)
    owner = np.zeros(page_bytes(D), np.int64)
    np.add.at(owner, k.ravel(), 1)
    for off in (0, 1):
        np.add.at(owner, ks + off, 1)
        np.add.at(owner, vs.ravel() + off, 1)
    words = np.unique(vw)
    for off in range(4):
        np.add.at(owner, words + off, 1)
    assert np.all(owner == 1)
    # each V word holds 8 distinct nibbles
    bits = {}
    for w, b in zip(vw.ravel().tolist(), vb.ravel().tolist()):
        bits.setdefault(w, set()).add(b)
    assert all(sorted(s) == list(range(0, 32, 4)) for s in bits.values())


def decode_pages(pages: np.ndarray, D: int):
    """pages uint8 [n, page_bytes(D)] -> kc int8 [n,16,D], ks u16 [n,16],
    vp u8 [n,16,D/2] (natural packing: even channel in the low nibble), vs u16 [n,16,D/32]."""
    pages = np.ascontiguousarray(pages)
    k, (vw, vb), ks, vs = _maps(D)
    kc = pages[:, k].view(np.int8)
    word = (pages[:, vw].astype(np.uint32) | (pages[:, vw + 1].astype(np.uint32) << 8)
            | (pages[:, vw + 2].astype(np.uint32) << 16) | (pages[:, vw + 3].astype(np.uint32) << 24))
    nib = ((word >> vb.astype(np.uint32)) & 0xF).astype(np.uint8)            # [n, 16, D]
    vp = (nib[:, :, 0::2] | (nib[:, :, 1::2] << 4)).astype(np.uint8)
    ksv = (pages[:, ks].astype(np.uint16) | (pages[:, ks + 1].astype(np.uint16) << 8))
    vsv = (pages[:, vs].astype(np.uint16) | (pages[:, vs + 1].astype(np.uint16) << 8))
    return kc, ksv, vp, vsv


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
