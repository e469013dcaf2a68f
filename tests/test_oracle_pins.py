"""Pins for the CPU oracle, checked against facts other than the oracle itself.

Every test here runs on the CPU.  Each pin is chosen so that a plausible
mistake in the oracle (a dropped term, a wrong sign or index, a transposed
operand, the wrong rounding) fails at least one of them:

  * the KV-memory closed form reproduces every size the pages print
    [KV Cache 优化全景解析——从基础原理到工程实践, §2.3, §3.3, §11.4];
  * quantisation: the round-trip bound |x - c*s| <= s/2 + 2^-24 |x|, exact
    rational brute force of the IEEE single division and ties-to-even rint,
    and the special vectors (zero, one-hot, constant, ties, sign flip,
    power-of-two scaling) [KV-Cache 全栈优化系统, 主要特性];
  * attention: closed forms (one token, uniform weights, two tokens), a
    cross-check with torch's scaled_dot_product_attention in float64 on the
    dequantised cache, GQA head routing, block-permutation invariance and
    prefix sharing [KV Cache 优化全景解析, §2.1, §3.3, §4.2].
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from workloads import bf16_bits_to_f32, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- memory
def test_kv_memory_printed_values(oracle_mod):
    with open(os.path.join(GOLDEN, "kv_memory_pages.json")) as f:
        g = json.load(f)
    for c in g["cases"]:
        b = oracle_mod.kv_cache_bytes(c["layers"], c["batch"], c["seq_len"],
                                      c["kv_heads"], c["head_dim"],
                                      c["bytes_num"], c["bytes_den"])
        gib = b / 2.0 ** 30
        assert round(gib, 2) == pytest.approx(c["printed_gb"], abs=1e-9), c["cite"]
        # decimal GB (1e9) would not reproduce the table: the unit is GiB
    b = oracle_mod.kv_cache_bytes(80, 1, 1024, 8, 128, 2, 1)
    assert round(b / 1e9, 2) != 0.31


def test_kv_memory_contradiction_documented(oracle_mod):
    with open(os.path.join(GOLDEN, "kv_memory_pages.json")) as f:
        c = json.load(f)["contradiction"]
    full = oracle_mod.kv_cache_bytes(c["layers"], c["batch"], c["seq_len"],
                                     c["kv_heads"], c["head_dim"],
                                     c["bytes_num"], c["bytes_den"])
    assert full == 2.0 ** 30
    no_heads = oracle_mod.kv_cache_bytes(c["layers"], c["batch"], c["seq_len"],
                                         1, c["head_dim"], c["bytes_num"],
                                         c["bytes_den"])
    assert no_heads == c["printed_product_bytes"]


def test_kv_memory_int8_and_int4(oracle_mod):
    # bytes per element: FP16 = 2, INT8 = 1, INT4 = 1/2 [§2.3 symbol table]
    fp16 = oracle_mod.kv_cache_bytes(32, 64, 32768, 8, 128, 2, 1)
    int8 = oracle_mod.kv_cache_bytes(32, 64, 32768, 8, 128, 1, 1)
    int4 = oracle_mod.kv_cache_bytes(32, 64, 32768, 8, 128, 1, 2)
    assert fp16 == 2 * int8 == 4 * int4
    # one layer of the batch-64 x 32K workload: 4 GiB of codes + 128 MiB of scales
    assert oracle_mod.kv_cache_bytes(1, 64, 32768, 8, 128, 1, 1) == 4 * 2 ** 30
    assert oracle_mod.kv8_scale_bytes(1, 64, 32768, 8) == 128 * 2 ** 20


# ---------------------------------------------------------------- quantiser
def _quant(oracle_mod, x_f32, n_kv_heads=1):
    """Quantise rows of x (float32, exactly bf16-representable) via the oracle."""
    x = np.asarray(x_f32, dtype=np.float32).reshape(-1, n_kv_heads, 128)
    bits = f32_to_bf16_bits(x)
    assert np.array_equal(bf16_bits_to_f32(bits), x), "test input must be bf16"
    n = x.shape[0]
    nb = (n + 15) // 16
    cache = np.full((nb, n_kv_heads, 16, 128), 127, dtype=np.int8)
    scales = np.full((nb, n_kv_heads, 16), np.nan, dtype=np.float32)
    oracle_mod.quantize_append(bits, np.arange(n, dtype=np.int64), cache, scales)
    c = np.stack([cache[i // 16, :, i % 16, :] for i in range(n)])
    s = np.stack([scales[i // 16, :, i % 16] for i in range(n)])
    return c, s


def _round_f32(fr: Fraction) -> Fraction:
    """Round a rational to the nearest binary32 value, ties to even (normal range)."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 23)
    q, r = divmod(a, ulp)
    q = int(q)
    if r * 2 > ulp or (r * 2 == ulp and q % 2 == 1):
        q += 1
    return sign * q * ulp


def _round_half_even(fr: Fraction) -> int:
    fl = math.floor(fr)
    r = fr - fl
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and fl % 2 == 1):
        return fl + 1
    return fl


def test_quant_exact_rational_bruteforce(oracle_mod):
    rng = np.random.default_rng(7)
    x = bf16_bits_to_f32(f32_to_bf16_bits(
        rng.standard_normal((6, 128)).astype(np.float32) * np.float32(3.0)))
    c, s = _quant(oracle_mod, x)
    for i in range(x.shape[0]):
        a = max(abs(Fraction(float(v))) for v in x[i])
        s_exp = _round_f32(a / 127)
        assert Fraction(float(s[i, 0])) == s_exp
        for j in range(128):
            y = _round_f32(Fraction(float(x[i, j])) / s_exp)
            code = max(-127, min(127, _round_half_even(y)))
            assert int(c[i, 0, j]) == code, (i, j)


def test_quant_round_trip_bound(oracle_mod):
    rng = np.random.default_rng(11)
    x = bf16_bits_to_f32(f32_to_bf16_bits(
        rng.standard_normal((64, 4, 128)).astype(np.float32)))
    x[:, :, 5] *= np.float32(10.0)  # an outlier channel
    x = bf16_bits_to_f32(f32_to_bf16_bits(x))
    c, s = _quant(oracle_mod, x.reshape(64, 4 * 128), n_kv_heads=4)
    xd = x.astype(np.float64)
    sd = s.astype(np.float64)[:, :, None]
    err = np.abs(xd - c.astype(np.float64) * sd)
    bound = sd / 2 + np.abs(xd) * 2.0 ** -24
    assert np.all(err <= bound)
    # the largest element of each (token, head) maps to +-127
    am = np.argmax(np.abs(x), axis=2)
    top = np.take_along_axis(c, am[:, :, None], axis=2)[:, :, 0]
    assert np.all(np.abs(top) == 127)
    assert np.all(np.abs(c) <= 127)


def test_quant_special_vectors(oracle_mod):
    rows = np.zeros((8, 128), dtype=np.float32)
    rows[1, 17] = -3.5                     # one-hot
    rows[2, :] = 0.75                      # constant
    rows[3, 0] = 127.0                     # scale exactly 1.0 ...
    rows[3, 1:5] = [2.5, 3.5, -2.5, -0.5]  # ... so these are exact ties
    rows[4, :] = np.linspace(-1, 1, 128, dtype=np.float32)
    rows[4] = bf16_bits_to_f32(f32_to_bf16_bits(rows[4]))
    rows[5] = -rows[4]                     # sign flip
    rows[6] = rows[4] * np.float32(8.0)    # power-of-two scaling
    c, s = _quant(oracle_mod, rows)
    c, s = c[:, 0, :], s[:, 0]
    # zero vector: scale 0, codes 0 (no NaN)
    assert s[0] == 0.0 and np.all(c[0] == 0)
    # one-hot: the nonzero maps to -127, the rest to 0
    assert c[1, 17] == -127 and np.count_nonzero(c[1]) == 1
    assert s[1] == np.float32(3.5) / np.float32(127.0)
    # constant: every element is the maximum
    assert np.all(c[2] == 127)
    # ties go to the even neighbour
    assert s[3] == 1.0
    assert list(c[3, :5]) == [127, 2, 4, -2, 0]
    # sign flip negates the codes, keeps the scale
    assert s[5] == s[4] and np.array_equal(c[5], -c[4])
    # power-of-two scaling keeps the codes, scales the scale exactly
    assert s[6] == s[4] * 8 and np.array_equal(c[6], c[4])
    # last row all zero as well
    assert s[7] == 0.0


def test_quant_slot_mapping_and_padding(oracle_mod):
    rng = np.random.default_rng(3)
    x = f32_to_bf16_bits(rng.standard_normal((5, 2, 128)).astype(np.float32))
    cache = np.full((4, 2, 16, 128), 127, dtype=np.int8)
    scales = np.full((4, 2, 16), np.nan, dtype=np.float32)
    slots = np.array([3 * 16 + 5, -1, 0, 2 * 16 + 15, -7], dtype=np.int64)
    oracle_mod.quantize_append(x, slots, cache, scales)
    written = {(3, 5): 0, (0, 0): 2, (2, 15): 3}
    for blk in range(4):
        for off in range(16):
            if (blk, off) in written:
                assert np.all(np.isfinite(scales[blk, :, off]))
                ref_c = np.full((1, 2, 16, 128), 127, dtype=np.int8)
                ref_s = np.zeros((1, 2, 16), dtype=np.float32)
                i = written[(blk, off)]
                oracle_mod.quantize_append(x[i:i + 1], np.array([off]), ref_c, ref_s)
                assert np.array_equal(cache[blk, :, off], ref_c[0, :, off])
                assert np.array_equal(scales[blk, :, off], ref_s[0, :, off])
            else:
                assert np.all(np.isnan(scales[blk, :, off]))
                assert np.all(cache[blk, :, off] == 127)
    with pytest.raises(ValueError):
        oracle_mod.quantize_append(x[:1], np.array([4 * 16]), cache, scales)


# ---------------------------------------------------------------- attention
def _paged(codes_k, codes_v, sk, sv, lens, perm=None, hkv=1):
    """Lay per-sequence token arrays [T, H_kv, 128] into a shuffled paged cache."""
    B = len(lens)
    nblk = [math.ceil(t / 16) for t in lens]
    nb = sum(nblk) + 2
    order = np.arange(nb) if perm is None else np.asarray(perm)
    kc = np.full((nb, hkv, 16, 128), 127, dtype=np.int8)
    vc = np.full_like(kc, 127)
    ks = np.full((nb, hkv, 16), np.nan, dtype=np.float32)
    vs = np.full_like(ks, np.nan)
    mbs = max(nblk + [1])
    bt = np.full((B, mbs), int(order[-1]), dtype=np.int32)
    cur = 0
    for b in range(B):
        for t in range(lens[b]):
            if t % 16 == 0:
                bt[b, t // 16] = order[cur]
                cur += 1
            p, o = bt[b, t // 16], t % 16
            kc[p, :, o] = codes_k[b][t]
            vc[p, :, o] = codes_v[b][t]
            ks[p, :, o] = sk[b][t]
            vs[p, :, o] = sv[b][t]
    return kc, vc, ks, vs, bt


def _rand_seq(rng, lens, hkv):
    ck = [rng.integers(-127, 128, (t, hkv, 128)).astype(np.int8) for t in lens]
    cv = [rng.integers(-127, 128, (t, hkv, 128)).astype(np.int8) for t in lens]
    sk = [(rng.random((t, hkv)) * 0.05 + 1e-3).astype(np.float32) for t in lens]
    sv = [(rng.random((t, hkv)) * 0.05 + 1e-3).astype(np.float32) for t in lens]
    return ck, cv, sk, sv


def _q(rng, B, hq):
    return f32_to_bf16_bits(rng.standard_normal((B, hq, 128)).astype(np.float32))


def test_attention_one_token_is_v_hat(oracle_mod):
    rng = np.random.default_rng(1)
    ck, cv, sk, sv = _rand_seq(rng, [1, 1], 2)
    kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, [1, 1], hkv=2)
    q = _q(rng, 2, 8)
    out = oracle_mod.decode_attention(q, kc, vc, ks, vs, bt, np.array([1, 1]))
    for b in range(2):
        for h in range(8):
            vhat = cv[b][0, h // 4].astype(np.float64) * np.float64(sv[b][0, h // 4])
            assert np.array_equal(out[b, h], vhat)


def test_attention_uniform_weights_and_identical_keys(oracle_mod):
    rng = np.random.default_rng(2)
    lens = [37, 5]
    ck, cv, sk, sv = _rand_seq(rng, lens, 1)
    kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, lens)
    # q = 0: every score is 0, the output is the mean of v_hat
    q0 = np.zeros((2, 2, 128), dtype=np.uint16)
    out = oracle_mod.decode_attention(q0, kc, vc, ks, vs, bt, np.array(lens))
    for b in range(2):
        mean = (cv[b][:, 0].astype(np.float64) * sv[b][:, 0:1].astype(np.float64)).mean(0)
        np.testing.assert_allclose(out[b, 0], mean, rtol=0, atol=1e-13)
    # identical keys: the same code row and scale for every token
    ck2 = [np.repeat(c[:1], c.shape[0], axis=0) for c in ck]
    sk2 = [np.repeat(s[:1], s.shape[0], axis=0) for s in sk]
    kc, vc, ks, vs, bt = _paged(ck2, cv, sk2, sv, lens)
    out = oracle_mod.decode_attention(_q(rng, 2, 2), kc, vc, ks, vs, bt, np.array(lens))
    for b in range(2):
        mean = (cv[b][:, 0].astype(np.float64) * sv[b][:, 0:1].astype(np.float64)).mean(0)
        np.testing.assert_allclose(out[b, 0], mean, rtol=0, atol=1e-13)


def test_attention_two_token_closed_form(oracle_mod):
    # two tokens: out = v1 + sigmoid(s2 - s1) * (v2 - v1), s = q.k_hat / sqrt(128)
    q = np.zeros((1, 1, 128), dtype=np.float32)
    q[0, 0, 0] = 1.0
    q[0, 0, 1] = -2.0
    ck = [np.zeros((2, 1, 128), dtype=np.int8)]
    ck[0][0, 0, 0] = 100
    ck[0][1, 0, 1] = -50
    sk = [np.array([[0.02], [0.03]], dtype=np.float32)]
    cv = [np.zeros((2, 1, 128), dtype=np.int8)]
    cv[0][0, 0, :] = 10
    cv[0][1, 0, :] = -20
    sv = [np.array([[0.5], [0.25]], dtype=np.float32)]
    kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, [2])
    out = oracle_mod.decode_attention(f32_to_bf16_bits(q), kc, vc, ks, vs, bt,
                                      np.array([2]))
    s1 = 1.0 * 100 * float(np.float32(0.02)) / math.sqrt(128)
    s2 = -2.0 * -50 * float(np.float32(0.03)) / math.sqrt(128)
    w2 = 1.0 / (1.0 + math.exp(s1 - s2))
    expect = 10 * 0.5 + w2 * (-20 * 0.25 - 10 * 0.5)
    np.testing.assert_allclose(out[0, 0], expect, rtol=1e-14, atol=0)


def test_attention_matches_torch_sdpa_float64(oracle_mod):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(5)
    for hq, hkv in [(8, 8), (8, 4), (8, 2), (8, 1)]:
        lens = [1, 16, 17, 40]
        ck, cv, sk, sv = _rand_seq(rng, lens, hkv)
        kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, lens, hkv=hkv,
                                    perm=rng.permutation(sum(math.ceil(t / 16) for t in lens) + 2))
        q = _q(rng, len(lens), hq)
        out = oracle_mod.decode_attention(q, kc, vc, ks, vs, bt, np.array(lens))
        g = hq // hkv
        for b, t in enumerate(lens):
            kh = torch.from_numpy(ck[b].astype(np.float64) * sk[b][:, :, None].astype(np.float64))
            vh = torch.from_numpy(cv[b].astype(np.float64) * sv[b][:, :, None].astype(np.float64))
            qq = torch.from_numpy(bf16_bits_to_f32(q[b]).astype(np.float64))  # [hq, D]
            kk = kh.permute(1, 0, 2).repeat_interleave(g, dim=0)  # [hq, t, D]
            vv = vh.permute(1, 0, 2).repeat_interleave(g, dim=0)
            ref = torch.nn.functional.scaled_dot_product_attention(
                qq[:, None, :], kk, vv)[:, 0, :].numpy()
            np.testing.assert_allclose(out[b], ref, rtol=1e-12, atol=1e-13)


def test_attention_gqa_head_routing(oracle_mod):
    rng = np.random.default_rng(9)
    lens = [20]
    ck, cv, sk, sv = _rand_seq(rng, lens, 4)
    kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, lens, hkv=4)
    q = _q(rng, 1, 8)
    base = oracle_mod.decode_attention(q, kc, vc, ks, vs, bt, np.array(lens))
    vc2 = vc.copy()
    vc2[:, 2] = -vc2[:, 2]  # change KV head 2 only
    out = oracle_mod.decode_attention(q, kc, vc2, ks, vs, bt, np.array(lens))
    changed = [h for h in range(8) if not np.array_equal(out[0, h], base[0, h])]
    assert changed == [4, 5]  # query heads 2*2 and 2*2+1 read KV head 2


def test_attention_block_permutation_invariance(oracle_mod):
    rng = np.random.default_rng(10)
    lens = [100, 33, 16]
    ck, cv, sk, sv = _rand_seq(rng, lens, 2)
    q = _q(rng, 3, 4)
    nb = sum(math.ceil(t / 16) for t in lens) + 2
    a = _paged(ck, cv, sk, sv, lens, hkv=2)
    b = _paged(ck, cv, sk, sv, lens, hkv=2, perm=rng.permutation(nb))
    oa = oracle_mod.decode_attention(q, *a, np.array(lens))
    ob = oracle_mod.decode_attention(q, *b, np.array(lens))
    assert np.array_equal(oa, ob)
    assert np.all(np.isfinite(oa))  # poisoned unused blocks never read


def test_attention_prefix_sharing(oracle_mod):
    rng = np.random.default_rng(12)
    hkv = 2
    pre = 48
    ck, cv, sk, sv = _rand_seq(rng, [pre + 10], hkv)
    # sequences 0 and 1 share the prefix blocks and have equal suffixes;
    # sequence 2 holds a private copy of the same tokens
    bt = np.array([[0, 1, 2, 3], [0, 1, 2, 4], [5, 6, 7, 8]], dtype=np.int32)
    kc = np.full((9, hkv, 16, 128), 127, dtype=np.int8)
    vc = np.full_like(kc, 127)
    ks = np.full((9, hkv, 16), np.nan, dtype=np.float32)
    vs = np.full_like(ks, np.nan)
    for b in range(3):
        for t in range(pre + 10):
            p, o = bt[b, t // 16], t % 16
            kc[p, :, o], vc[p, :, o] = ck[0][t], cv[0][t]
            ks[p, :, o], vs[p, :, o] = sk[0][t], sv[0][t]
    q1 = _q(rng, 1, 4)
    q = np.repeat(q1, 3, axis=0)
    out = oracle_mod.decode_attention(q, kc, vc, ks, vs, bt, np.array([pre + 10] * 3))
    assert np.array_equal(out[0], out[1]) and np.array_equal(out[0], out[2])


def test_attention_empty_context_and_scale_default(oracle_mod):
    rng = np.random.default_rng(13)
    lens = [0, 23]
    ck, cv, sk, sv = _rand_seq(rng, lens, 1)
    kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, lens)
    q = _q(rng, 2, 2)
    out = oracle_mod.decode_attention(q, kc, vc, ks, vs, bt, np.array(lens))
    assert np.all(out[0] == 0.0)
    out2 = oracle_mod.decode_attention(q, kc, vc, ks, vs, bt, np.array(lens),
                                       softmax_scale=1.0 / math.sqrt(128))
    assert np.array_equal(out, out2)
    out3 = oracle_mod.decode_attention(q, kc, vc, ks, vs, bt, np.array(lens),
                                       softmax_scale=2.0 / math.sqrt(128))
    assert not np.array_equal(out[1], out3[1])


def test_attention_pairs_subset(oracle_mod):
    rng = np.random.default_rng(14)
    lens = [30, 7, 64]
    ck, cv, sk, sv = _rand_seq(rng, lens, 2)
    kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, lens, hkv=2)
    q = _q(rng, 3, 8)
    full = oracle_mod.decode_attention(q, kc, vc, ks, vs, bt, np.array(lens))
    pairs = [(2, 7), (0, 0), (1, 3)]
    sub = oracle_mod.decode_attention(q, kc, vc, ks, vs, bt, np.array(lens), pairs=pairs)
    for i, (b, h) in enumerate(pairs):
        assert np.array_equal(sub[i], full[b, h])
