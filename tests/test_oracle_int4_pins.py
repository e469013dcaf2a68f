"""Pins of the oracle's INT4 variant (CPU only).

The K/V of historical tokens are quantised to 4 bits [nano-KvLLM, §2.2
量化感知缓存]; INT4 takes half a byte per element [KV Cache 优化全景解析——
从基础原理到工程实践, §2.3].  The oracle's reading: per (token, KV head)
s = fl32(max|x| / 7), c = clamp(rint(fl32(x / s)), -7, 7), stored as the
nibble c + 8, dims 2i / 2i+1 in the low / high nibble of byte i.  Pins:
  * the scale and every code against exact rational arithmetic (IEEE single
    division, ties to even) on random rows;
  * round trip |x - c s| <= s/2 (+ the division's rounding) on every element;
  * special rows: zero, one-hot, constant, exact ties between codes;
  * the nibble layout and slot mapping (padding skipped);
  * attention over the dequantised cache against torch SDPA in float64 for
    g in {1, 2, 4, 8}, a one-token context, and block-permutation invariance.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from tests.test_oracle_pins import _round_f32, _round_half_even
from workloads import bf16_bits_to_f32, f32_to_bf16_bits


def _quant4(oracle_mod, x_f32, n_kv_heads=1):
    x = np.asarray(x_f32, dtype=np.float32).reshape(-1, n_kv_heads, 128)
    bits = f32_to_bf16_bits(x)
    assert np.array_equal(bf16_bits_to_f32(bits), x), "test input must be bf16"
    n = x.shape[0]
    nb = (n + 15) // 16
    cache = np.zeros((nb, n_kv_heads, 16, 64), dtype=np.uint8)
    scales = np.full((nb, n_kv_heads, 16), np.nan, dtype=np.float32)
    oracle_mod.quantize_append_int4(bits, np.arange(n, dtype=np.int64), cache, scales)
    packed = np.stack([cache[i // 16, :, i % 16, :] for i in range(n)])
    s = np.stack([scales[i // 16, :, i % 16] for i in range(n)])
    codes = np.empty(packed.shape[:-1] + (128,), dtype=np.int64)
    codes[..., 0::2] = (packed & 15).astype(np.int64) - 8
    codes[..., 1::2] = (packed >> 4).astype(np.int64) - 8
    return codes, s, packed


def test_int4_exact_rational_bruteforce(oracle_mod):
    rng = np.random.default_rng(41)
    x = bf16_bits_to_f32(f32_to_bf16_bits(
        rng.standard_normal((6, 128)).astype(np.float32) * np.float32(2.5)))
    c, s, _ = _quant4(oracle_mod, x)
    for i in range(x.shape[0]):
        a = max(abs(Fraction(float(v))) for v in x[i])
        s_exp = _round_f32(a / 7)
        assert Fraction(float(s[i, 0])) == s_exp
        for j in range(128):
            y = _round_f32(Fraction(float(x[i, j])) / s_exp)
            assert int(c[i, 0, j]) == max(-7, min(7, _round_half_even(y))), (i, j)


def test_int4_round_trip_bound(oracle_mod):
    rng = np.random.default_rng(42)
    x = bf16_bits_to_f32(f32_to_bf16_bits(
        rng.standard_normal((48, 4, 128)).astype(np.float32)))
    c, s, _ = _quant4(oracle_mod, x.reshape(48, 4 * 128), n_kv_heads=4)
    xd = x.astype(np.float64)
    sd = s.astype(np.float64)[:, :, None]
    err = np.abs(xd - c * sd)
    assert np.all(err <= sd / 2 * (1 + 2.0 ** -22) + 2.0 ** -24 * np.abs(xd))
    assert np.all(np.abs(c) <= 7)
    # the largest element of every row maps to +-7
    amax = np.argmax(np.abs(xd), axis=2)
    for i in range(48):
        for h in range(4):
            assert abs(c[i, h, amax[i, h]]) == 7


def test_int4_special_rows(oracle_mod):
    rows = np.zeros((4, 128), dtype=np.float32)
    rows[1, 17] = -3.0                       # one-hot
    rows[2, :] = 0.75                        # constant
    rows[3, :2] = [7.0, 0.5]                 # s = 1: 0.5 is a tie -> 0 (even)
    rows[3, 2:4] = [1.5, -2.5]               # ties -> 2, -2
    c, s, packed = _quant4(oracle_mod, rows)
    assert s[0, 0] == 0.0 and np.all(c[0] == 0) and np.all(packed[0] == 0x88)
    assert c[1, 0, 17] == -7 and np.count_nonzero(c[1]) == 1
    assert np.all(c[2] == 7)
    assert s[3, 0] == 1.0
    assert list(c[3, 0, :4]) == [7, 0, 2, -2]


def test_int4_layout_and_padding(oracle_mod):
    x = np.zeros((3, 1, 128), dtype=np.float32)
    x[0, 0, 0], x[0, 0, 1] = 7.0, -7.0       # byte 0: low nibble 15, high 1
    x[1, 0, 127] = 1.0
    bits = f32_to_bf16_bits(x)
    cache = np.full((2, 1, 16, 64), 0xAB, dtype=np.uint8)
    scales = np.full((2, 1, 16), np.nan, dtype=np.float32)
    oracle_mod.quantize_append_int4(bits, np.array([19, -1, 3]), cache, scales)
    assert cache[1, 0, 3, 0] == (15 | (1 << 4))           # token 0 at slot 19
    assert np.all(cache[1, 0, 3, 1:] == 0x88)
    assert np.all(cache[0, 0, 3] == 0x88) and scales[0, 0, 3] == 0.0  # token 2
    untouched = np.ones((2, 1, 16), dtype=bool)
    untouched[1, 0, 3] = untouched[0, 0, 3] = False
    assert np.all(cache[untouched] == 0xAB) and np.all(np.isnan(scales[untouched]))


def _paged4(rng, lens, hkv, perm=None):
    nblk = [math.ceil(t / 16) for t in lens]
    nb = sum(nblk) + 2
    order = np.arange(nb) if perm is None else np.asarray(perm)
    kc = rng.integers(1, 16, (nb, hkv, 16, 64)).astype(np.uint8)
    kc |= (rng.integers(1, 16, kc.shape).astype(np.uint8) << 4)
    vc = rng.integers(1, 16, kc.shape).astype(np.uint8)
    vc |= (rng.integers(1, 16, kc.shape).astype(np.uint8) << 4)
    ks = (rng.random((nb, hkv, 16)) * 0.3 + 0.01).astype(np.float32)
    vs = (rng.random((nb, hkv, 16)) * 0.3 + 0.01).astype(np.float32)
    bt = np.zeros((len(lens), max(nblk + [1])), dtype=np.int32)
    cur = 0
    for b, n in enumerate(nblk):
        bt[b, :n] = order[cur:cur + n]
        cur += n
    return kc, vc, ks, vs, bt


def _dequant(packed, scale):
    c = np.empty(packed.shape[:-1] + (128,), dtype=np.float64)
    c[..., 0::2] = (packed & 15).astype(np.float64) - 8
    c[..., 1::2] = (packed >> 4).astype(np.float64) - 8
    return c * scale.astype(np.float64)[..., None]


def test_int4_attention_matches_torch_sdpa_float64(oracle_mod):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(43)
    for hq, hkv in [(8, 8), (8, 4), (8, 2), (8, 1)]:
        lens = [1, 16, 17, 40]
        kc, vc, ks, vs, bt = _paged4(rng, lens, hkv)
        q = f32_to_bf16_bits(rng.standard_normal((4, hq, 128)).astype(np.float32))
        out = oracle_mod.decode_attention_int4(q, kc, vc, ks, vs, bt, np.array(lens))
        g = hq // hkv
        for b, t in enumerate(lens):
            blocks = [bt[b, i // 16] for i in range(t)]
            kh = np.stack([_dequant(kc[blocks[i], :, i % 16], ks[blocks[i], :, i % 16])
                           for i in range(t)])  # [t, hkv, 128]
            vh = np.stack([_dequant(vc[blocks[i], :, i % 16], vs[blocks[i], :, i % 16])
                           for i in range(t)])
            kk = torch.from_numpy(kh).permute(1, 0, 2).repeat_interleave(g, dim=0)
            vv = torch.from_numpy(vh).permute(1, 0, 2).repeat_interleave(g, dim=0)
            qq = torch.from_numpy(bf16_bits_to_f32(q[b]).astype(np.float64))
            ref = torch.nn.functional.scaled_dot_product_attention(
                qq[:, None, :], kk, vv)[:, 0, :].numpy()
            np.testing.assert_allclose(out[b], ref, rtol=1e-12, atol=1e-13)
    # one token: the dequantised V row exactly
    kc, vc, ks, vs, bt = _paged4(rng, [1], 2)
    q = f32_to_bf16_bits(rng.standard_normal((1, 4, 128)).astype(np.float32))
    out = oracle_mod.decode_attention_int4(q, kc, vc, ks, vs, bt, np.array([1]))
    for h in range(4):
        assert np.array_equal(out[0, h], _dequant(vc[bt[0, 0], h // 2, 0], vs[bt[0, 0], h // 2, 0]))


def test_int4_block_permutation_invariance(oracle_mod):
    rng = np.random.default_rng(44)
    lens = [70, 33]
    nb = sum(math.ceil(t / 16) for t in lens) + 2
    kc, vc, ks, vs, bt = _paged4(rng, lens, 2)
    q = f32_to_bf16_bits(rng.standard_normal((2, 8, 128)).astype(np.float32))
    a = oracle_mod.decode_attention_int4(q, kc, vc, ks, vs, bt, np.array(lens))
    perm = rng.permutation(nb)
    kc2, vc2, ks2, vs2 = (np.empty_like(x) for x in (kc, vc, ks, vs))
    for old in range(nb):
        for x, y in ((kc, kc2), (vc, vc2), (ks, ks2), (vs, vs2)):
            y[perm[old]] = x[old]
    b = oracle_mod.decode_attention_int4(q, kc2, vc2, ks2, vs2, perm[bt].astype(np.int32),
                                         np.array(lens))
    assert np.array_equal(a, b)
