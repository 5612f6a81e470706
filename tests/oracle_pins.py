"""Pins for the CPU oracle: each check compares it with something other than
itself -- 50-digit decimal brute force, hand-derived closed forms, a library
routine (torch's scaled_dot_product_attention and logsumexp in float64),
mathematical invariants, and the split identity that the Flash-Decoding page
relies on ("the attention/softmax can be calculated iteratively", section
"A faster attention for decoding: Flash-Decoding").

Every pin is a plain function of an ``oracle.Oracle`` that raises
AssertionError on a mismatch, so the same list runs against the real oracle
(tests/test_oracle_pins.py) and against builds with a planted mistake
(tests/test_oracle_mutants.py), where at least one pin must fail.
"""
import itertools
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "worked_examples.json")


# ---------------------------------------------------------------- helpers --

def to_bits(x) -> np.ndarray:
    """float array -> bf16 bit patterns (round to nearest even)."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_f64(b) -> np.ndarray:
    u = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def rand_case(rng, B, Hq, Hkv, D, Lmax, seqlens=None, sigma=(1.0, 1.0, 1.0), integer_v=False):
    q = to_bits(rng.standard_normal((B, Hq, D)) * sigma[0])
    k = to_bits(rng.standard_normal((B, Hkv, Lmax, D)) * sigma[1])
    if integer_v:
        v = to_bits(rng.integers(-8, 9, (B, Hkv, Lmax, D)).astype(np.float32))
    else:
        v = to_bits(rng.standard_normal((B, Hkv, Lmax, D)) * sigma[2])
    if seqlens is None:
        seqlens = np.full((B,), Lmax, np.int32)
    return q, k, v, np.asarray(seqlens, np.int32)


def close(a, b, tol, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        err = np.where(both_inf, 0.0, np.abs(a - b))
    if not np.all(err <= tol):
        raise AssertionError(f"{what}: max error {np.nanmax(err):.3e} > {tol:.1e}")


def decimal_row(qf, kf, vf, L, scale):
    """One row of attention in 50-digit decimal arithmetic, straight from the
    definition: logits, their log-sum-exp, softmax-weighted values."""
    getcontext().prec = 50
    s = Decimal(scale)
    z = [s * sum(Decimal(float(qf[d])) * Decimal(float(kf[t, d])) for d in range(len(qf))) for t in range(L)]
    total = sum(zt.exp() for zt in z)
    lse = total.ln()
    out = [sum((z[t] - lse).exp() * Decimal(float(vf[t, d])) for t in range(L)) for d in range(vf.shape[1])]
    return [float(o) for o in out], float(lse)


# ------------------------------------------------------------------- pins --

def pin_brute_force_decimal(orc):
    """Tiny random cases against 50-digit decimal evaluation of the definition."""
    rng = np.random.default_rng(1234)
    for trial in range(12):
        Hkv = [1, 2][trial % 2]
        g = [1, 2, 3][trial % 3]
        Hq = Hkv * g
        D = 1 + trial % 4
        Lmax = 8
        seqlens = rng.integers(1, Lmax + 1, (2,)).astype(np.int32)
        scale = float(rng.uniform(0.2, 1.5))
        q, k, v, seqlens = rand_case(rng, 2, Hq, Hkv, D, Lmax, seqlens, sigma=(1.0, 2.0, 1.0))
        out, lse = orc.attention(q, k, v, seqlens, scale)
        qf, kf, vf = bits_to_f64(q), bits_to_f64(k), bits_to_f64(v)
        for b in range(2):
            for i in range(Hq):
                j = i // g
                eo, el = decimal_row(qf[b, i], kf[b, j], vf[b, j], int(seqlens[b]), scale)
                close(out[b, i], eo, 1e-12, f"brute force out b={b} i={i}")
                close(lse[b, i], el, 1e-12, f"brute force lse b={b} i={i}")


def pin_worked_examples(orc):
    """Hand-derived examples stored under tests/golden (closed forms below)."""
    with open(GOLDEN) as f:
        cases = {c["name"]: c for c in json.load(f)["cases"]}
    E = math.e
    expected = {
        "three_integer_logits": ([[(1 + 2 * E * E) / (1 + E + E * E), (E + 2 * E * E) / (1 + E + E * E)]],
                                 [math.log(1 + E + E * E)]),
        "one_key": ([[3.0, -1.0]], [0.25]),
        "two_equal_logits": ([[0.5, 1.5]], [1.0 + math.log(2.0)]),
        "gqa_pair": ([[E / (1 + E), 1 / (1 + E)], [1 / (1 + E), E / (1 + E)]],
                     [math.log(1 + E), math.log(1 + E)]),
    }
    for name, (eo, el) in expected.items():
        c = cases[name]
        q = to_bits(np.array(c["q"])[None])
        k = to_bits(np.array(c["k"])[None])
        v = to_bits(np.array(c["v"])[None])
        L = k.shape[2]
        out, lse = orc.attention(q, k, v, np.array([L], np.int32), c["scale"])
        close(out[0], eo, 1e-14, f"worked example {name} out")
        close(lse[0], el, 1e-14, f"worked example {name} lse")


def pin_closed_forms(orc):
    """One key gives out = v; identical keys give out = mean(V) and
    lse = z + log L; scale 0 gives out = mean(V) and lse = log L."""
    rng = np.random.default_rng(7)
    D, Lmax = 8, 24
    # one key
    q, k, v, _ = rand_case(rng, 3, 4, 2, D, Lmax)
    out, lse = orc.attention(q, k, v, np.array([1, 1, 1], np.int32), 0.3)
    qf, kf, vf = bits_to_f64(q), bits_to_f64(k), bits_to_f64(v)
    for b in range(3):
        for i in range(4):
            j = i // 2
            if not np.array_equal(out[b, i], vf[b, j, 0]):
                raise AssertionError("one key: out != v")
            z = 0.3 * math.fsum(qf[b, i] * kf[b, j, 0])
            close(lse[b, i], z, 1e-14 * max(1.0, abs(z)), "one key: lse != scale*q.k")
    # identical keys
    L = 17
    k_same = np.repeat(k[:, :, :1, :], Lmax, axis=2)
    out, lse = orc.attention(q, k_same, v, np.array([L, L, L], np.int32), 0.3)
    for b in range(3):
        for i in range(4):
            j = i // 2
            mean = np.array([math.fsum(vf[b, j, :L, d]) / L for d in range(D)])
            close(out[b, i], mean, 1e-13, "identical keys: out != mean(V)")
            z = 0.3 * math.fsum(qf[b, i] * kf[b, j, 0])
            close(lse[b, i], z + math.log(L), 1e-13, "identical keys: lse != z + log L")
    # scale 0
    seq = np.array([5, 24, 11], np.int32)
    out, lse = orc.attention(q, k, v, seq, 0.0)
    for b in range(3):
        Lb = int(seq[b])
        for i in range(4):
            j = i // 2
            mean = np.array([math.fsum(vf[b, j, :Lb, d]) / Lb for d in range(D)])
            close(out[b, i], mean, 1e-13, "scale 0: out != mean(V)")
            close(lse[b, i], math.log(Lb), 1e-14, "scale 0: lse != log L")


def pin_library_sdpa(orc):
    """Grouped-query case against torch.nn.functional.scaled_dot_product_attention
    (float64, enable_gqa) and torch.logsumexp."""
    rng = np.random.default_rng(99)
    B, Hq, Hkv, D, Lmax = 2, 8, 2, 16, 40
    seq = np.array([37, 21], np.int32)
    scale = 0.21
    q, k, v, seq = rand_case(rng, B, Hq, Hkv, D, Lmax, seq, sigma=(1.0, 2.0, 1.0))
    out, lse = orc.attention(q, k, v, seq, scale)
    qf, kf, vf = (torch.from_numpy(bits_to_f64(a)) for a in (q, k, v))
    for b in range(B):
        L = int(seq[b])
        qb = qf[b][None, :, None, :]                    # [1, Hq, 1, D]
        kb = kf[b, :, :L][None]                          # [1, Hkv, L, D]
        vb = vf[b, :, :L][None]
        ref = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, scale=scale, enable_gqa=True)
        close(out[b], ref[0, :, 0].numpy(), 1e-12, "sdpa out")
        kexp = kb[0].repeat_interleave(Hq // Hkv, dim=0)  # [Hq, L, D]
        logits = scale * torch.matmul(kexp, qf[b][:, :, None])[..., 0]
        close(lse[b], torch.logsumexp(logits, dim=-1).numpy(), 1e-12, "logsumexp lse")


def pin_split_identity(orc):
    """Every set of contiguous split points, reduced through the per-split
    log-sum-exp, gives the unsplit result (brute-force enumeration)."""
    rng = np.random.default_rng(5)
    for L in range(1, 11):
        q, k, v, seq = rand_case(rng, 1, 2, 1, 3, L, sigma=(1.0, 3.0, 1.0))
        ref_out, ref_lse = orc.attention(q, k, v, seq, 0.7)
        for r in range(0, L):
            for cuts in itertools.combinations(range(1, L), r):
                bounds = [0, *cuts, L]
                out, lse = orc.split_attention(q, k, v, seq, 0.7, bounds)
                close(out, ref_out, 1e-12, f"split {bounds} out")
                close(lse, ref_lse, 1e-12, f"split {bounds} lse")
        # empty splits at both ends and past the row's end carry no weight
        out, lse = orc.split_attention(q, k, v, seq, 0.7, [0, 0, (L + 1) // 2, L, L + 3, L + 9])
        close(out, ref_out, 1e-12, "split with empty chunks out")
        close(lse, ref_lse, 1e-12, "split with empty chunks lse")


def pin_combine_by_hand(orc):
    """The final reduction on partials whose result is known by hand:
    lse (ln 1, ln 3) weights the outputs 1/4 and 3/4; an empty split is
    ignored; all-empty rows give 0 and -inf."""
    po = np.array([[[1.0, 2.0], [4.0, 0.0], [9.0, 9.0]],
                   [[5.0, 5.0], [6.0, 6.0], [7.0, 7.0]]])
    pl = np.array([[0.0, math.log(3.0), -math.inf],
                   [-math.inf, -math.inf, -math.inf]])
    out, lse = orc.combine(po, pl)
    close(out[0], [0.25 * 1 + 0.75 * 4, 0.25 * 2], 1e-15, "combine out")
    close(lse[0], math.log(4.0), 1e-15, "combine lse")
    close(out[1], [0.0, 0.0], 0.0, "all-empty combine out")
    if not (lse[1] == -math.inf):
        raise AssertionError("all-empty combine lse != -inf")


def pin_invariants(orc):
    """Token permutation, affine maps of V, and a constant shift of every
    logit (through one extra head dimension) act as the math says."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, D, Lmax = 2, 4, 2, 6, 19
    seq = np.array([19, 13], np.int32)
    q, k, v, seq = rand_case(rng, B, Hq, Hkv, D, Lmax, seq, integer_v=True)
    out, lse = orc.attention(q, k, v, seq, 0.125)
    # permutation of (k_t, v_t) pairs inside each row
    kp, vp = k.copy(), v.copy()
    for b in range(B):
        perm = rng.permutation(int(seq[b]))
        kp[b, :, :seq[b]] = k[b][:, perm]
        vp[b, :, :seq[b]] = v[b][:, perm]
    o2, l2 = orc.attention(q, kp, vp, seq, 0.125)
    close(o2, out, 1e-12, "permutation out")
    close(l2, lse, 1e-12, "permutation lse")
    # out(2V + 3) = 2 out(V) + 3  (integer V keeps 2V + 3 exact in bf16)
    v2 = to_bits(2.0 * bits_to_f64(v) + 3.0)
    o3, l3 = orc.attention(q, k, v2, seq, 0.125)
    close(o3, 2.0 * out + 3.0, 1e-12, "affine V out")
    close(l3, lse, 0.0, "affine V lse")
    # extra dimension: q' = [q, 1], k'_t = [k_t, 8]: every logit + 0.125 * 8 = +1
    qa = np.concatenate([q, np.full((B, Hq, 1), to_bits([1.0])[0], np.uint16)], axis=2)
    ka = np.concatenate([k, np.full((B, Hkv, Lmax, 1), to_bits([8.0])[0], np.uint16)], axis=3)
    va = np.concatenate([v, np.zeros((B, Hkv, Lmax, 1), np.uint16)], axis=3)
    o4, l4 = orc.attention(qa, ka, va, seq, 0.125)
    close(o4[..., :D], out, 1e-12, "logit shift out")
    close(l4, lse + 1.0, 1e-12, "logit shift lse")


def pin_padding_and_empty(orc):
    """Positions at or beyond seqlen never matter (NaN there gives the bitwise
    same result as zeros), and an empty row gives out 0, lse -inf."""
    rng = np.random.default_rng(3)
    B, Hq, Hkv, D, Lmax = 3, 2, 2, 5, 16
    seq = np.array([5, 16, 0], np.int32)
    q, k, v, seq = rand_case(rng, B, Hq, Hkv, D, Lmax, seq)
    nan = to_bits([np.nan])[0]
    kz, vz, kn, vn = k.copy(), v.copy(), k.copy(), v.copy()
    for b in range(B):
        kz[b, :, seq[b]:] = 0
        vz[b, :, seq[b]:] = 0
        kn[b, :, seq[b]:] = nan
        vn[b, :, seq[b]:] = nan
    oz, lz = orc.attention(q, kz, vz, seq, 0.4)
    on, ln = orc.attention(q, kn, vn, seq, 0.4)
    if not (np.array_equal(oz, on) and np.array_equal(lz, ln)):
        raise AssertionError("NaN padding changed the result")
    if not (np.all(on[2] == 0.0) and np.all(ln[2] == -math.inf)):
        raise AssertionError("empty row is not (0, -inf)")
    # seqlens above Lmax are clamped to Lmax, negative ones to 0
    o5, l5 = orc.attention(q, k, v, np.array([5, 99, -3], np.int32), 0.4)
    o6, l6 = orc.attention(q, k, v, np.array([5, 16, 0], np.int32), 0.4)
    if not (np.array_equal(o5, o6) and np.array_equal(l5, l6)):
        raise AssertionError("seqlens are not clamped to [0, Lmax]")


def pin_group_mapping(orc):
    """Query head i reads kv head i // g: the grouped problem equals, head by
    head, the problem restricted to one kv head and its g query heads."""
    rng = np.random.default_rng(21)
    B, g, Hkv, D, Lmax = 2, 3, 2, 4, 9
    Hq = g * Hkv
    q, k, v, seq = rand_case(rng, B, Hq, Hkv, D, Lmax, np.array([9, 4], np.int32))
    out, lse = orc.attention(q, k, v, seq, 0.5)
    for j in range(Hkv):
        qs = np.ascontiguousarray(q[:, j * g:(j + 1) * g])
        o, l = orc.attention(qs, np.ascontiguousarray(k[:, j:j + 1]), np.ascontiguousarray(v[:, j:j + 1]), seq, 0.5)
        if not (np.array_equal(o, out[:, j * g:(j + 1) * g]) and np.array_equal(l, lse[:, j * g:(j + 1) * g])):
            raise AssertionError(f"group mapping: kv head {j} differs")


def pin_multi_query_decimal(orc):
    """Several queries per sequence against 50-digit decimal evaluation:
    query j of a sequence with L cached tokens sees its first
    L - (q_len - 1 - j) tokens."""
    rng = np.random.default_rng(77)
    for trial in range(6):
        q_len = 1 + trial % 4
        Hkv, g = [1, 2][trial % 2], [1, 3][trial % 2]
        Hq, D, Lmax = Hkv * g, 1 + trial % 3, 9
        seqlens = np.array([9, q_len + (trial % 3)], np.int32)
        scale = float(rng.uniform(0.3, 1.2))
        q = to_bits(rng.standard_normal((2, q_len, Hq, D)))
        _, k, v, _ = rand_case(rng, 2, Hq, Hkv, D, Lmax, seqlens, sigma=(1.0, 2.0, 1.0))
        out, lse = orc.attention_multi(q, k, v, seqlens, scale)
        qf, kf, vf = bits_to_f64(q), bits_to_f64(k), bits_to_f64(v)
        for b in range(2):
            for j in range(q_len):
                Lq = int(seqlens[b]) - (q_len - 1 - j)
                for i in range(Hq):
                    eo, el = decimal_row(qf[b, j, i], kf[b, i // g], vf[b, i // g], Lq, scale)
                    close(out[b, j, i], eo, 1e-12, f"multi-query out b={b} j={j} i={i}")
                    close(lse[b, j, i], el, 1e-12, f"multi-query lse b={b} j={j} i={i}")


def pin_multi_query_library_mask(orc):
    """Several queries against torch scaled_dot_product_attention (float64)
    with an explicit boolean mask built from the causal-offset rule."""
    rng = np.random.default_rng(78)
    B, q_len, Hq, Hkv, D, Lmax = 2, 4, 6, 2, 8, 30
    seq = np.array([30, 11], np.int32)
    q = to_bits(rng.standard_normal((B, q_len, Hq, D)))
    _, k, v, seq = rand_case(rng, B, Hq, Hkv, D, Lmax, seq)
    out, lse = orc.attention_multi(q, k, v, seq, 0.3)
    qf, kf, vf = (torch.from_numpy(bits_to_f64(a)) for a in (q, k, v))
    for b in range(B):
        L = int(seq[b])
        mask = torch.zeros((q_len, L), dtype=torch.bool)
        for j in range(q_len):
            mask[j, :L - (q_len - 1 - j)] = True
        ref = torch.nn.functional.scaled_dot_product_attention(
            qf[b].permute(1, 0, 2)[None], kf[b, :, :L][None], vf[b, :, :L][None], attn_mask=mask, scale=0.3,
            enable_gqa=True)                                            # [1, Hq, q_len, D]
        close(out[b], ref[0].permute(1, 0, 2).numpy(), 1e-12, "multi-query sdpa out")


# ----------------------------------------------- quantised key/value cache --

def one_key_codes(orc, kv_type, codes, v_scale):
    """A row with one cached token whose value holds `codes`: the softmax
    weight is 1, so out = v_scale * decode(code) for each element."""
    D = len(codes)
    q = to_bits(np.full((1, 1, D), 0.5))
    k8 = np.full((1, 1, 1, D), 0x38 if kv_type == "e4m3" else 1, np.uint8)
    v8 = np.asarray(codes, np.uint8).reshape(1, 1, 1, D)
    out, lse = orc.attention_quant(q, k8, v8, np.array([0.25], np.float32), np.array([v_scale], np.float32),
                                   np.array([1], np.int32), 0.5, kv_type)
    return out[0, 0], lse[0, 0]


def pin_e4m3_codes(orc):
    """Every E4M3 code against torch's float8_e4m3fn conversion (library),
    plus values fixed by the format's definition: 0x38 = 1, 0x7E = 448 (the
    largest), 0x08 = 2^-6 (smallest normal), 0x01 = 2^-9 (smallest
    subnormal), 0x80 = -0, 0x7F = NaN."""
    codes = np.arange(256, dtype=np.uint8)
    out, lse = one_key_codes(orc, "e4m3", codes, 1.0)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    if not np.array_equal(np.isnan(out), np.isnan(ref)):
        raise AssertionError("e4m3: NaN codes differ from torch")
    close(out[~np.isnan(ref)], ref[~np.isnan(ref)], 0.0, "e4m3 code values vs torch")
    for c, val in ((0x38, 1.0), (0x7E, 448.0), (0x08, 2.0 ** -6), (0x01, 2.0 ** -9), (0xB8, -1.0), (0x80, 0.0)):
        close(out[c], val, 0.0, f"e4m3 code {c:#04x}")
    if not (np.isnan(out[0x7F]) and np.isnan(out[0xFF])):
        raise AssertionError("e4m3: 0x7F / 0xFF must be NaN")
    # one key of all-ones codes (k = 0.25 each): lse = 0.5 * 0.25 * 0.5 * D
    close(lse, 0.5 * 0.25 * 0.5 * 256, 1e-12, "e4m3 one-key lse")


def pin_int8_codes(orc):
    """Every int8 code is its two's-complement value times the head's scale."""
    codes = np.arange(256, dtype=np.uint8)
    out, _ = one_key_codes(orc, "int8", codes, 0.5)
    close(out, codes.view(np.int8).astype(np.float64) * 0.5, 0.0, "int8 codes")


def quant_case(rng, kv_type, B, q_len, Hq, Hkv, D, Lmax):
    """Random codes (no NaN codes) and distinct per-head scales."""
    q = to_bits(rng.standard_normal((B, q_len, Hq, D)))
    if kv_type == "e4m3":
        pool = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
        k8, v8 = (rng.choice(pool, (B, Hkv, Lmax, D)) for _ in range(2))
    else:
        k8, v8 = (rng.integers(0, 256, (B, Hkv, Lmax, D)).astype(np.uint8) for _ in range(2))
    ks = (rng.uniform(0.5, 2.0, Hkv) * (0.02 if kv_type == "e4m3" else 0.03)).astype(np.float32)
    vs = (rng.uniform(0.5, 2.0, Hkv) * (0.05 if kv_type == "e4m3" else 0.04)).astype(np.float32)
    return q, k8, v8, ks, vs


def dequant_torch(codes, scales, kv_type):
    t = torch.from_numpy(np.ascontiguousarray(codes))
    vals = t.view(torch.float8_e4m3fn).to(torch.float64) if kv_type == "e4m3" else t.view(torch.int8).to(torch.float64)
    return vals * torch.from_numpy(scales.astype(np.float64))[None, :, None, None]


def pin_quant_library_sdpa(orc):
    """Quantised cache against torch scaled_dot_product_attention (float64)
    over the cache dequantised by torch's own conversions, with grouped heads,
    ragged lengths and several queries (causal-offset mask)."""
    rng = np.random.default_rng(91)
    for kv_type in ("e4m3", "int8"):
        B, q_len, Hq, Hkv, D, Lmax = 3, 2, 6, 2, 16, 40
        q, k8, v8, ks, vs = quant_case(rng, kv_type, B, q_len, Hq, Hkv, D, Lmax)
        seq = np.array([40, 17, 1], np.int32)
        out, lse = orc.attention_quant(q, k8, v8, ks, vs, seq, 0.25, kv_type)
        qf = torch.from_numpy(bits_to_f64(q))
        kf, vf = dequant_torch(k8, ks, kv_type), dequant_torch(v8, vs, kv_type)
        for b in range(B):
            L = int(seq[b])
            mask = torch.zeros((q_len, L), dtype=torch.bool)
            for j in range(q_len):
                mask[j, :max(0, L - (q_len - 1 - j))] = True
            qb = qf[b].permute(1, 0, 2)                                   # [Hq, q_len, D]
            ref = torch.nn.functional.scaled_dot_product_attention(
                qb[None], kf[b, :, :L][None], vf[b, :, :L][None], attn_mask=mask, scale=0.25, enable_gqa=True)
            z = 0.25 * torch.einsum("hqd,htd->hqt", qb, kf[b, :, :L].repeat_interleave(Hq // Hkv, 0))
            ref_lse = torch.logsumexp(z.masked_fill(~mask[None], -math.inf), dim=-1)   # [Hq, q_len]
            for j in range(q_len):
                if mask[j].any():
                    close(out[b, j], ref[0, :, j].numpy(), 1e-12, f"{kv_type} sdpa out b={b} j={j}")
                    close(lse[b, j], ref_lse[:, j].numpy(), 1e-12, f"{kv_type} lse b={b} j={j}")
                else:
                    close(out[b, j], 0.0, 0.0, f"{kv_type} empty query out")
                    if not np.all(np.isneginf(lse[b, j])):
                        raise AssertionError(f"{kv_type}: a query that sees no token must have lse = -inf")


def pin_quant_scales(orc):
    """Scale laws: multiplying every k_scale by c is multiplying the softmax
    scale by c; multiplying v_scale[h] by c multiplies the outputs of that
    head's group by c and leaves every lse and the other heads unchanged."""
    rng = np.random.default_rng(92)
    for kv_type in ("e4m3", "int8"):
        B, Hq, Hkv, D, Lmax = 2, 4, 2, 8, 25
        q, k8, v8, ks, vs = quant_case(rng, kv_type, B, 1, Hq, Hkv, D, Lmax)
        seq = np.array([25, 9], np.int32)
        o1, l1 = orc.attention_quant(q, k8, v8, ks * np.float32(2.0), vs, seq, 0.3, kv_type)
        o2, l2 = orc.attention_quant(q, k8, v8, ks, vs, seq, 0.6, kv_type)
        close(o1, o2, 1e-13, f"{kv_type}: k_scale*2 vs scale*2 out")
        close(l1, l2, 1e-12, f"{kv_type}: k_scale*2 vs scale*2 lse")
        vs2 = vs.copy()
        vs2[1] *= np.float32(4.0)
        o3, l3 = orc.attention_quant(q, k8, v8, ks, vs, seq, 0.3, kv_type)
        o4, l4 = orc.attention_quant(q, k8, v8, ks, vs2, seq, 0.3, kv_type)
        close(l3, l4, 0.0, f"{kv_type}: v_scale must not move lse")
        close(o4[:, :, :2], o3[:, :, :2], 0.0, f"{kv_type}: v_scale of head 1 moved head 0's group")
        close(o4[:, :, 2:], 4.0 * o3[:, :, 2:], 1e-13, f"{kv_type}: v_scale of head 1")


ALL_PINS = [
    pin_brute_force_decimal,
    pin_worked_examples,
    pin_closed_forms,
    pin_library_sdpa,
    pin_split_identity,
    pin_combine_by_hand,
    pin_invariants,
    pin_padding_and_empty,
    pin_group_mapping,
    pin_multi_query_decimal,
    pin_multi_query_library_mask,
    pin_e4m3_codes,
    pin_int8_codes,
    pin_quant_library_sdpa,
    pin_quant_scales,
]
