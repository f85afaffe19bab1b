"""Checks that pin the CPU oracle to facts other than itself.

Each ``check_*`` takes an ``oracle.OracleLib`` and raises AssertionError when the
oracle disagrees with: a hand-worked case (tests/golden/quant_hand_cases.json), an
exact brute-force search, a closed form, an invariant, or a library routine
(numpy's float16 cast, torch's fp64 softmax).  None of them retypes the oracle's
own formula.  ``tests/test_oracle_mutants.py`` runs the same checks against
deliberately broken copies of the oracle to show that each plausible mistake is
caught by at least one of them.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "quant_hand_cases.json")


def golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _pad(x, D):
    v = np.zeros(D, np.float32)
    v[: len(x)] = np.asarray(x, np.float32)
    return v


def _nib(b, j):
    return ((b >> (4 * j)) & 0xF) - 16 * (((b >> (4 * j)) & 0xF) >= 8)


def _unpack(packed):
    packed = np.asarray(packed, np.uint8).astype(np.int32)
    lo = np.where(packed & 0xF >= 8, (packed & 0xF) - 16, packed & 0xF)
    hi = np.where(packed >> 4 >= 8, (packed >> 4) - 16, packed >> 4)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.int32)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


# ---------------------------------------------------------------------------
# conversions
# ---------------------------------------------------------------------------
def check_f16_hand(O):
    for c in golden()["f16"]:
        got = int(O.f32_to_f16_bits(np.float32(c["x"])))
        assert got == int(c["bits"], 16), (c, hex(got))


def check_f16_vs_numpy(O, n=20000, seed=3):
    rng = np.random.default_rng(seed)
    mant = rng.random(n) + 1.0
    expo = rng.integers(-30, 18, n)
    sign = rng.choice([-1.0, 1.0], n)
    x = (sign * mant * np.exp2(expo)).astype(np.float32)
    got = O.f32_to_f16_bits(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)


def check_bf16_hand(O):
    for c in golden()["bf16"]:
        assert float(O.bf16_bits_to_f32(np.uint16(int(c["bits"], 16)))) == c["x"]


# ---------------------------------------------------------------------------
# quantization: hand-worked cases
# ---------------------------------------------------------------------------
def check_k_hand(O):
    for c in golden()["k"]:
        D = c["head_dim"]
        codes, sb = O.quantize_k(_pad(c["x"], D)[None])
        assert int(sb[0]) == int(c["scale_bits"], 16), (c["why"], hex(int(sb[0])))
        exp = np.zeros(D, np.int32)
        exp[: len(c["codes"])] = c["codes"]
        assert np.array_equal(codes[0].astype(np.int32), exp), (c["why"], codes[0][:12])


def check_v_hand(O):
    for c in golden()["v"]:
        D = c["head_dim"]
        if "x_by_group" in c:
            x = np.zeros(D, np.float32)
            for g, vals in enumerate(c["x_by_group"]):
                x[32 * g: 32 * g + len(vals)] = vals
            packed, sb = O.quantize_v(x[None])
            assert [int(s) for s in sb[0]] == [int(s, 16) for s in c["scale_bits"]], c["why"]
            firsts = [int(packed[0, 16 * g]) for g in range(len(c["x_by_group"]))]
            assert firsts == [int(b, 16) for b in c["first_bytes_by_group"]], (c["why"], [hex(b) for b in firsts])
        else:
            packed, sb = O.quantize_v(_pad(c["x"], D)[None])
            assert [int(s) for s in sb[0]] == [int(s, 16) for s in c["scale_bits"]], c["why"]
            exp = np.zeros(D // 2, np.uint8)
            exp[: len(c["bytes"])] = [int(b, 16) for b in c["bytes"]]
            assert np.array_equal(packed[0], exp), (c["why"], [hex(b) for b in packed[0][:8]])


def check_dequant_hand(O):
    # code 3 with scale 1.0 (0x3c00) is 3.0; code -127 with scale 129/16384 (0x2008)
    codes = np.zeros((2, 128), np.int8)
    codes[0, 0] = 3
    codes[1, 5] = -127
    out = O.dequantize_k(codes, np.array([0x3C00, 0x2008], np.uint16))
    assert out[0, 0] == 3.0 and out[1, 5] == -127 * 129 / 16384 and out[1, 0] == 0.0
    # byte 0x87 holds codes (7, -8); group scale 2^-4 (0x2c00) -> 0.4375, -0.5
    packed = np.zeros((1, 64), np.uint8)
    packed[0, 0] = 0x87
    vs = np.array([[0x2C00, 0, 0, 0]], np.uint16)
    v = O.dequantize_v(packed, vs)
    assert v[0, 0] == 0.4375 and v[0, 1] == -0.5 and np.all(v[0, 2:] == 0)


# ---------------------------------------------------------------------------
# quantization: exact search and properties
# ---------------------------------------------------------------------------
def _f16_values():
    return np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)


_F16 = None


def _nearest_f16_set(v: float):
    """All finite non-negative fp16 values at minimal distance from v (exact)."""
    global _F16
    if _F16 is None:
        _F16 = _f16_values()
    i = int(np.searchsorted(_F16, v))
    cand = [_F16[j] for j in (i - 1, i, i + 1) if 0 <= j < len(_F16)]
    fv = Fraction(v)
    d = [abs(Fraction(c) - fv) for c in cand]
    m = min(d)
    return [cand[j] for j in range(len(cand)) if d[j] == m]


def _x_data(seed, n, D):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, D)).astype(np.float32)
    x[:, :4] *= 10.0                      # outlier channels, as in the workloads
    x[n // 2:] *= np.exp2(rng.integers(-12, 6, (n - n // 2, 1))).astype(np.float32)
    return x


def _scale_ok(absmax: float, qmax: int, s: float):
    """s must be an fp16 value nearest to absmax/qmax (fp32 quotient, exact search)."""
    quo = float(np.float32(absmax) / np.float32(qmax))
    near = _nearest_f16_set(quo)
    return s in near


def _nearest_codes(x, s, lo, hi):
    """Exact nearest multiple of s in [lo, hi], ties to the even multiple.

    This equals the round-half-even of the fp32 quotient x / s for fp32 x and an
    fp16 scale s: a half-integer below 128 has at most 8 significant bits, so the
    fp32 quotient can land on one only when the exact quotient is that
    half-integer, and it can never round across one.  The search therefore
    checks the reading 'rne(x / s) in fp32' without retyping it."""
    fx, fs = Fraction(float(x)), Fraction(float(s))
    base = math.floor(fx / fs)
    best = None
    for k in (base - 1, base, base + 1, base + 2):
        kk = min(max(k, lo), hi)
        d = abs(fx - kk * fs)
        if best is None or d < best[0] or (d == best[0] and kk % 2 == 0):
            best = (d, kk)
    return best[1]


def check_k_bruteforce(O, n=96, D=128, seed=5):
    x = _x_data(seed, n, D)
    codes, sb = O.quantize_k(x)
    svals = O.f16_bits_to_f64(sb)
    for i in range(n):
        a = float(np.max(np.abs(x[i])))
        assert _scale_ok(a, 127, svals[i]), (i, a, svals[i])
        for c in range(D):
            k = _nearest_codes(x[i, c], svals[i], -127, 127)
            assert codes[i, c] == k, (i, c, x[i, c], svals[i], codes[i, c], k)


def check_v_bruteforce(O, n=96, D=128, seed=6):
    x = _x_data(seed, n, D)
    packed, sb = O.quantize_v(x)
    codes = _unpack(packed)
    svals = O.f16_bits_to_f64(sb)
    for i in range(n):
        for g in range(D // 32):
            a = float(np.max(np.abs(x[i, 32 * g: 32 * g + 32])))
            assert _scale_ok(a, 7, svals[i, g]), (i, g, a, svals[i, g])
            for c in range(32 * g, 32 * g + 32):
                k = _nearest_codes(x[i, c], svals[i, g], -8, 7)
                assert codes[i, c] == k, (i, c, x[i, c], svals[i, g], codes[i, c], k)


def check_tiny_scales(O, seed=8):
    """Vectors whose scale is an fp16 subnormal or underflows: brute force still
    holds (codes clamp at -127/127 and -8/7), and an underflowed scale gives 0."""
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((64, 128)) * np.exp2(rng.integers(-34, -18, (64, 1)))).astype(np.float32)
    codes, sb = O.quantize_k(x)
    s = O.f16_bits_to_f64(sb)
    packed, vsb = O.quantize_v(x)
    vcodes = _unpack(packed)
    vs = O.f16_bits_to_f64(vsb)
    for i in range(64):
        assert _scale_ok(float(np.max(np.abs(x[i]))), 127, s[i])
        for c in range(0, 128, 7):
            if s[i] == 0:
                assert codes[i, c] == 0
            else:
                assert codes[i, c] == _nearest_codes(x[i, c], s[i], -127, 127)
            g = c // 32
            if vs[i, g] == 0:
                assert vcodes[i, c] == 0
            else:
                assert vcodes[i, c] == _nearest_codes(x[i, c], vs[i, g], -8, 7)
    assert np.any(s == 0) and np.any((s > 0) & (s < 2 ** -14))


def check_near_ties(O):
    """Inputs at, and 1-2 ulps either side of, every half-integer multiple of a
    set of fp16 scales: the codes must equal the exact nearest multiple (ties to
    even).  This is where a reciprocal-multiply or a mis-rounded division shows."""
    scales = [129.0 / 16384.0, 2047.0 / 1024.0 * 2 ** -9, 1.0 / 3.0, 0.1, 1531.0 / 1024.0 * 2 ** -5]
    for s16 in scales:
        s = float(np.float16(s16))
        xs = []
        for k in range(-126, 126):
            t = np.float32((k + 0.5) * s)
            xs.append(t)
            for step in (1, 2):
                up, dn = t, t
                for _ in range(step):
                    up = np.nextafter(up, np.float32(np.inf), dtype=np.float32)
                    dn = np.nextafter(dn, np.float32(-np.inf), dtype=np.float32)
                xs += [up, dn]
        xs = np.array(xs, np.float32)
        D = 128
        n = (len(xs) + D - 2) // (D - 1)
        vec = np.zeros((n, D), np.float32)
        vec[:, 0] = np.float32(127.0 * s)                 # absmax/127 == s exactly
        flat = np.zeros(n * (D - 1), np.float32)
        flat[: len(xs)] = xs
        vec[:, 1:] = flat.reshape(n, D - 1)
        codes, sb = O.quantize_k(vec)
        assert np.all(O.f16_bits_to_f64(sb) == s)
        for i in range(n):
            for c in range(1, D):
                assert codes[i, c] == _nearest_codes(vec[i, c], s, -127, 127), (s, float(vec[i, c]), codes[i, c])


def check_roundtrip(O, n=256, seed=7):
    x = _x_data(seed, n, 128)
    codes, sb = O.quantize_k(x)
    s = O.f16_bits_to_f64(sb)[:, None]
    err = np.abs(O.dequantize_k(codes, sb) - x.astype(np.float64))
    assert np.all(err <= s / 2 * (1 + 2 ** -20) + 1e-30)
    packed, vsb = O.quantize_v(x)
    vs = np.repeat(O.f16_bits_to_f64(vsb), 32, axis=1)
    err = np.abs(O.dequantize_v(packed, vsb) - x.astype(np.float64))
    assert np.all(err <= vs / 2 * (1 + 2 ** -20) + 1e-30)


def check_memory_claim(O):
    """K+V+scale bytes per (token, kv-head) are less than half of fp16 K+V
    (the launch page's 'more than half' KV-memory cut)."""
    for D, expect in ((128, 202), (256, 402)):
        b = O.kv_bytes_per_token_head(D)
        assert b == expect and b < 0.5 * (2 * 2 * D), (D, b)


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------
def _rand_kv(rng, L, Hkv, D):
    k = rng.standard_normal((L, Hkv, D))
    v = rng.standard_normal((L, Hkv, D))
    return k, v


def check_attn_single_token(O):
    rng = np.random.default_rng(11)
    q = rng.standard_normal((1, 4, 128))
    k, v = _rand_kv(rng, 1, 2, 128)
    out, lse = O.attention(q, k, v, 1 / math.sqrt(128))
    for h in range(4):
        assert np.array_equal(out[0, h], v[0, h // 2])
        assert abs(lse[0, h] - q[0, h] @ k[0, h // 2] / math.sqrt(128)) < 1e-12


def check_attn_two_token_closed_form(O):
    rng = np.random.default_rng(12)
    D = 128
    q = rng.standard_normal((1, 1, D))
    k, v = _rand_kv(rng, 2, 1, D)
    sc = 0.3
    z0, z1 = sc * float(q[0, 0] @ k[0, 0]), sc * float(q[0, 0] @ k[1, 0])
    w0 = 1.0 / (1.0 + math.exp(z1 - z0))
    w1 = 1.0 / (1.0 + math.exp(z0 - z1))
    exp = w0 * v[0, 0] + w1 * v[1, 0]
    out, lse = O.attention(q, k, v, sc)
    assert np.max(np.abs(out[0, 0] - exp)) < 1e-12
    assert abs(lse[0, 0] - (max(z0, z1) + math.log1p(math.exp(-abs(z0 - z1))))) < 1e-12


def check_attn_constant_v(O):
    rng = np.random.default_rng(13)
    L, Hkv, D = 300, 2, 128
    q = rng.standard_normal((2, 8, D))
    k = rng.standard_normal((L, Hkv, D)) * 3
    v = np.broadcast_to(rng.standard_normal((1, Hkv, D)), (L, Hkv, D)).copy()
    out, _ = O.attention(q, k, v, 1 / math.sqrt(D))
    for h in range(8):
        assert np.max(np.abs(out[:, h] - v[0, h // 4])) < 1e-12


def check_attn_weights(O):
    rng = np.random.default_rng(14)
    L, Hkv, D, n = 64, 2, 128, 3
    q = rng.standard_normal((n, 4, D))
    k, v = _rand_kv(rng, L, Hkv, D)
    sc = 1 / math.sqrt(D)
    out, lse, w = O.attention(q, k, v, sc, return_weights=True)
    for j in range(n):
        vis = L - n + j + 1
        for h in range(4):
            ww = w[j, h]
            assert abs(ww.sum() - 1.0) < 1e-12 and np.all(ww >= 0) and np.all(ww[vis:] == 0)
            z = sc * (k[:vis, h // 2] @ q[j, h])
            # ratios follow exp(z_a - z_b), and lse = log sum exp z
            assert np.max(np.abs(np.log(ww[:vis]) - (z - lse[j, h]))) < 1e-10
            assert np.max(np.abs(out[j, h] - ww[:vis] @ v[:vis, h // 2])) < 1e-12


def check_attn_dominant_key(O):
    rng = np.random.default_rng(15)
    L, D = 200, 128
    k, v = _rand_kv(rng, L, 1, D)
    j = 77
    k[j, 0] *= 3.0                      # |k_j| exceeds every other key's norm
    errs = []
    for c in (0.002, 0.02, 1.0):
        q = (c * k[j, 0])[None, None, :]
        out, _ = O.attention(q, k, v, 1 / math.sqrt(D))
        errs.append(float(np.max(np.abs(out[0, 0] - v[j, 0]))))
    assert errs[0] > 1e-2 and errs[0] > errs[1] > errs[2] and errs[2] < 1e-9, errs


def check_attn_torch(O):
    import torch
    rng = np.random.default_rng(16)
    L, Hkv, Hq, D, n = 50, 2, 8, 128, 3
    q = rng.standard_normal((n, Hq, D))
    k, v = _rand_kv(rng, L, Hkv, D)
    sc = 1 / math.sqrt(D)
    out, lse = O.attention(q, k, v, sc)
    tq = torch.from_numpy(q).permute(1, 0, 2)                       # [Hq, n, D]
    tk = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    tv = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    z = sc * tq @ tk.transpose(1, 2)                                  # [Hq, n, L]
    mask = torch.arange(L)[None, :] > (L - n + torch.arange(n))[:, None]
    z = z.masked_fill(mask[None], float("-inf"))
    ref = torch.softmax(z, -1) @ tv
    ref_lse = torch.logsumexp(z, -1)
    assert np.max(np.abs(out - ref.permute(1, 0, 2).numpy())) < 1e-12
    assert np.max(np.abs(lse - ref_lse.permute(1, 0).numpy())) < 1e-12


def check_attn_causal(O):
    rng = np.random.default_rng(17)
    L, Hkv, D, n = 90, 2, 128, 8
    q = rng.standard_normal((n, 8, D))
    k, v = _rand_kv(rng, L, Hkv, D)
    sc = 1 / math.sqrt(D)
    out, lse = O.attention(q, k, v, sc)
    for j in range(n):
        vis = L - n + j + 1
        o1, l1 = O.attention(q[j: j + 1], k[:vis], v[:vis], sc)
        assert np.array_equal(out[j], o1[0]) and np.array_equal(lse[j], l1[0])


def check_attn_gqa(O):
    rng = np.random.default_rng(18)
    L, Hkv, D, G = 40, 4, 128, 3
    q = rng.standard_normal((1, Hkv * G, D))
    k, v = _rand_kv(rng, L, Hkv, D)
    out, _ = O.attention(q, k, v, 0.1)
    for h in range(Hkv * G):
        o1, _ = O.attention(q[:, h: h + 1], k[:, h // G: h // G + 1], v[:, h // G: h // G + 1], 0.1)
        assert np.array_equal(out[0, h], o1[0, 0])


def check_attn_permutation(O):
    rng = np.random.default_rng(19)
    L, D = 128, 128
    q = rng.standard_normal((1, 2, D))
    k, v = _rand_kv(rng, L, 1, D)
    out, lse = O.attention(q, k, v, 0.2)
    p = rng.permutation(L)
    out2, lse2 = O.attention(q, k[p], v[p], 0.2)
    assert np.max(np.abs(out - out2)) < 1e-13 and np.max(np.abs(lse - lse2)) < 1e-12


def check_attn_quant_form(O):
    rng = np.random.default_rng(20)
    L, Hkv, D, n = 70, 2, 256, 2
    x = _x_data(21, L * Hkv, D).reshape(L, Hkv, D)
    y = _x_data(22, L * Hkv, D).reshape(L, Hkv, D)
    kc, ks = O.quantize_k(x)
    vp, vs = O.quantize_v(y)
    q = rng.standard_normal((n, 4, D))
    o1, l1 = O.attention(q, O.dequantize_k(kc, ks), O.dequantize_v(vp, vs), 1 / 16)
    o2, l2 = O.attention_quant(q, kc, ks, vp, vs, 1 / 16)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def check_attn_prefix_split(O):
    """Attention over a whole cache equals the log-sum-exp merge of attention over a
    prefix (every query sees all of it) and over the rest (causal among the drafts):
    the identity the shared-prefix cascade rests on, and a pin on lse, which carries
    the merge weights."""
    rng = np.random.default_rng(23)
    L, P, Hkv, D, n = 90, 48, 2, 128, 3
    x = _x_data(24, L * Hkv, D).reshape(L, Hkv, D)
    y = _x_data(25, L * Hkv, D).reshape(L, Hkv, D)
    kc, ks = O.quantize_k(x)
    vp, vs = O.quantize_v(y)
    q = rng.standard_normal((n, 4, D))
    o, l = O.attention_quant(q, kc, ks, vp, vs, 1 / math.sqrt(D))
    o2, l2 = O.attention_quant(q, kc[P:], ks[P:], vp[P:], vs[P:], 1 / math.sqrt(D))
    for j in range(n):
        o1, l1 = O.attention_quant(q[j:j + 1], kc[:P], ks[:P], vp[:P], vs[:P], 1 / math.sqrt(D))
        m = np.maximum(l1[0], l2[j])
        w1, w2 = np.exp(l1[0] - m), np.exp(l2[j] - m)
        om = (o1[0] * w1[:, None] + o2[j] * w2[:, None]) / (w1 + w2)[:, None]
        lm = m + np.log(w1 + w2)
        assert np.max(np.abs(om - o[j])) < 1e-12 and np.max(np.abs(lm - l[j])) < 1e-12


QUANT_CHECKS = [check_f16_hand, check_f16_vs_numpy, check_bf16_hand, check_k_hand, check_v_hand,
                check_dequant_hand, check_k_bruteforce, check_v_bruteforce, check_tiny_scales,
                check_near_ties, check_roundtrip, check_memory_claim]
ATTN_CHECKS = [check_attn_single_token, check_attn_two_token_closed_form, check_attn_constant_v,
               check_attn_weights, check_attn_dominant_key, check_attn_torch, check_attn_causal,
               check_attn_gqa, check_attn_permutation, check_attn_quant_form, check_attn_prefix_split]


# ---- history-based drafting ------------------------------------------------------
DRAFT_GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "draft_ngram_cases.json")


def check_draft_hand(O):
    """The hand-worked cases of tests/golden/draft_ngram_cases.json."""
    with open(DRAFT_GOLDEN) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        got = O.draft_ngram(np.array(c["tokens"], np.int32), c["n"], c["k"]).tolist()
        assert got == c["drafts"], (c, got)


def _rfind_drafts(tokens, n, k):
    """The same drafts found with bytes.rfind: each token (0 <= t < 250) is the 4-byte
    word 0xFF t 0xFE 0xFD, so a byte match can only start on a token boundary; the
    window must end before the last token, i.e. inside bytes [0, 4 (L - 1))."""
    L = len(tokens)
    if L <= n:
        return []
    enc = b"".join(bytes([0xFF, int(t), 0xFE, 0xFD]) for t in tokens)
    at = enc.rfind(enc[4 * (L - n):], 0, 4 * (L - 1))
    if at < 0:
        return []
    assert at % 4 == 0
    i = at // 4
    return [int(t) for t in tokens[i + n: min(i + n + k, L)]]


def check_draft_rfind(O, trials=300, seed=11):
    """Random short-alphabet histories (many repeats) against the bytes.rfind search."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        L = int(rng.integers(1, 200))
        alpha = int(rng.integers(2, 6))
        t = rng.integers(0, alpha, L).astype(np.int32)
        n = int(rng.integers(1, 6))
        k = int(rng.integers(1, 9))
        assert O.draft_ngram(t, n, k).tolist() == _rfind_drafts(t, n, k), (t.tolist(), n, k)


DRAFT_CHECKS = [check_draft_hand, check_draft_rfind]
