"""Pins of the oracle's KIVI variant (CPU only).

Keys are quantised per channel and values per token, to 2-bit asymmetric
codes [KV Cache 优化全景解析——从基础原理到工程实践, §7.1 量化的核心挑战
and §7.2 KIVI：2bit 无损非对称量化].  The oracle's readings: a group is
quantised by its minimum z and s = fl32(fl32(max - z) / 3), codes
c = clamp(rint(fl32(fl32(x - z) / s)), 0, 3), x_hat = c s + z; a key group is
one channel of one 16-token page; a page is quantised when its last token
arrives, and until then its rows stay in bf16 in the sequence's tail, read
exactly by attention [nano-KvLLM, §2.2 量化感知缓存: recent tokens keep their
precision].  Pins:
  * scale, zero and every code against exact rational arithmetic;
  * every code is a nearest level of its group (|x - x_hat| <= s/2, plus the
    rounding of the two single-precision steps);
  * pages whose channels (keys) or tokens (values) sit exactly on four
    evenly spaced levels of their own are reconstructed exactly -- which
    fails if an axis is swapped, since the spacings differ along the other
    axis;
  * constant groups (s = 0); a context whose tokens all carry one key
    gives the plain mean of its values (pages and tail alike);
  * attention over pages built that way, plus bf16 tail rows, equals torch
    SDPA in float64 on the original K/V, for g in {1, 2, 4, 8}, ragged
    contexts and permuted block tables;
  * pages are written only when full, and the tail holds the partial page;
  * the append gives the same cache however the tokens are split into calls.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from tests.test_oracle_pins import _round_f32, _round_half_even
from workloads import bf16_bits_to_f32, f32_to_bf16_bits

D, BS = 128, 16


def _bits(x):
    x = np.asarray(x, dtype=np.float32)
    b = f32_to_bf16_bits(x)
    assert np.array_equal(bf16_bits_to_f32(b), x), "test input must be bf16"
    return b


def _one_page(oracle_mod, k, v):
    """Append 16 tokens ([16, H, D] float32, bf16-exact) of one sequence into
    block 0; returns the oracle cache."""
    h = k.shape[1]
    c = oracle_mod.KiviCache(1, h, 1)
    oracle_mod.kivi_append(c, _bits(k), _bits(v), np.array([0, BS]),
                           np.array([BS]), np.zeros((1, 1), np.int32))
    return c


def _dequant(c):
    kh = (c.k_codes.astype(np.float64) * c.k_scale.astype(np.float64)[:, :, None, :]
          + c.k_zero.astype(np.float64)[:, :, None, :])
    vh = (c.v_codes.astype(np.float64) * c.v_scale.astype(np.float64)[:, :, :, None]
          + c.v_zero.astype(np.float64)[:, :, :, None])
    return kh, vh


def _expected_group(xs):
    """Exact-rational scale, zero and codes of one group (bf16 values)."""
    fr = [Fraction(float(x)) for x in xs]
    lo, hi = min(fr), max(fr)
    s = _round_f32(_round_f32(hi - lo) / 3)
    if s == 0:
        return s, lo, [0] * len(fr)
    codes = [max(0, min(3, _round_half_even(_round_f32(_round_f32(x - lo) / s))))
             for x in fr]
    return s, lo, codes


def test_kivi_exact_rational_bruteforce(oracle_mod):
    rng = np.random.default_rng(71)
    k = bf16_bits_to_f32(_bits(bf16_bits_to_f32(f32_to_bf16_bits(
        (rng.standard_normal((BS, 2, D)) * 2.0).astype(np.float32)))))
    v = bf16_bits_to_f32(f32_to_bf16_bits(
        (rng.standard_normal((BS, 2, D)) * 0.5 + 0.25).astype(np.float32)))
    c = _one_page(oracle_mod, k, v)
    for h in range(2):
        for j in range(0, D, 7):  # keys: channel j over the page's tokens
            s, z, codes = _expected_group(k[:, h, j])
            assert Fraction(float(c.k_scale[0, h, j])) == s
            assert Fraction(float(c.k_zero[0, h, j])) == z
            assert [int(x) for x in c.k_codes[0, h, :, j]] == codes, (h, j)
        for t in range(BS):  # values: token t over the channels
            s, z, codes = _expected_group(v[t, h, :])
            assert Fraction(float(c.v_scale[0, h, t])) == s
            assert Fraction(float(c.v_zero[0, h, t])) == z
            assert [int(x) for x in c.v_codes[0, h, t, :]] == codes, (h, t)


def test_kivi_nearest_level(oracle_mod):
    rng = np.random.default_rng(72)
    k = rng.standard_normal((BS, 4, D)).astype(np.float32)
    k[:, :, 5] *= 40.0  # an outlier channel, as keys have
    v = rng.standard_normal((BS, 4, D)).astype(np.float32)
    k = bf16_bits_to_f32(f32_to_bf16_bits(k))
    v = bf16_bits_to_f32(f32_to_bf16_bits(v))
    c = _one_page(oracle_mod, k, v)
    kh, vh = _dequant(c)
    ks = c.k_scale.astype(np.float64)[0][None, :, :]      # [1, H, D]
    vs = c.v_scale.astype(np.float64)[0].T[:, :, None]    # [BS, H, 1]
    ek = np.abs(kh[0].transpose(1, 0, 2) - k)             # [BS, H, D]
    ev = np.abs(vh[0].transpose(1, 0, 2) - v)
    # nearest level up to the rounding of x - z and of the division
    assert np.all(ek <= ks * (0.5 + 2.0 ** -20))
    assert np.all(ev <= vs * (0.5 + 2.0 ** -20))
    # the minimum is reproduced exactly (code 0) and codes span 0..3
    assert np.array_equal(c.k_zero[0], k.min(axis=0))
    assert np.array_equal(c.v_zero[0].T, v.min(axis=2))
    assert c.k_codes.max() == 3 and c.v_codes.min() == 0


def _levels(rng, shape, spacing_exp, axis):
    """Values (m + c) * 2^e with per-group e (along `axis` of the groups),
    every group holding codes 0 and 3 so that min = m 2^e, max = (m+3) 2^e."""
    codes = rng.integers(0, 4, size=shape)
    idx = [slice(None)] * len(shape)
    idx[axis] = 0
    codes[tuple(idx)] = 0
    idx[axis] = 1
    codes[tuple(idx)] = 3
    m = rng.integers(-60, 60, size=spacing_exp.shape)
    x = (np.expand_dims(m, axis) + codes) * np.exp2(np.expand_dims(spacing_exp, axis))
    return x.astype(np.float32), codes, m


def test_kivi_axes_exact_levels(oracle_mod):
    rng = np.random.default_rng(73)
    H = 2
    # keys: channel j of head h has its own spacing 2^e[h, j]
    ek = rng.integers(-8, 6, size=(H, D)).astype(np.float64)
    kt, kcodes, km = _levels(rng, (BS, H, D), ek, axis=0)
    # values: token t of head h has its own spacing 2^e[t, h]
    ev = rng.integers(-8, 6, size=(BS, H)).astype(np.float64)
    vt, vcodes, vm = _levels(rng, (BS, H, D), ev, axis=2)
    c = _one_page(oracle_mod, kt, vt)
    assert np.array_equal(c.k_codes[0].transpose(1, 0, 2), kcodes)
    assert np.array_equal(c.v_codes[0].transpose(1, 0, 2), vcodes)
    assert np.array_equal(c.k_scale[0], np.exp2(ek).astype(np.float32))
    assert np.array_equal(c.v_scale[0].T, np.exp2(ev).astype(np.float32))
    kh, vh = _dequant(c)
    assert np.array_equal(kh[0].transpose(1, 0, 2), kt.astype(np.float64))
    assert np.array_equal(vh[0].transpose(1, 0, 2), vt.astype(np.float64))


def test_kivi_constant_groups(oracle_mod):
    rng = np.random.default_rng(74)
    k = bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((BS, 1, D)).astype(np.float32)))
    v = bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((BS, 1, D)).astype(np.float32)))
    k[:, 0, 9] = 1.5       # a constant key channel
    k[:, 0, 10] = 0.0
    v[3, 0, :] = -2.25     # a constant value token
    c = _one_page(oracle_mod, k, v)
    for j, val in ((9, 1.5), (10, 0.0)):
        assert c.k_scale[0, 0, j] == 0.0 and c.k_zero[0, 0, j] == val
        assert not c.k_codes[0, 0, :, j].any()
    assert c.v_scale[0, 0, 3] == 0.0 and c.v_zero[0, 0, 3] == -2.25
    assert not c.v_codes[0, 0, 3].any()
    kh, vh = _dequant(c)
    assert np.all(kh[0, 0, :, 9] == 1.5) and np.all(vh[0, 0, 3] == -2.25)


def _exact_batch(rng, lens, hkv, nb_extra=3):
    """A batch whose full pages sit on exact per-channel (K) / per-token (V)
    levels and whose partial pages are arbitrary bf16; block tables are a
    random permutation.  Returns (k, v) per sequence [n, H, D] float32, the
    block table and the number of blocks."""
    mbs = max(1, max((n + BS - 1) // BS for n in lens))
    nb = sum((n + BS - 1) // BS for n in lens) + nb_extra
    perm = rng.permutation(nb)
    bt = np.full((len(lens), mbs), nb - 1, np.int32)
    at = 0
    ks, vs = [], []
    for b, n in enumerate(lens):
        pages = (n + BS - 1) // BS
        bt[b, :pages] = perm[at:at + pages]
        at += pages
        kk = np.empty((n, hkv, D), np.float32)
        vv = np.empty((n, hkv, D), np.float32)
        for p in range(n // BS):
            ek = rng.integers(-10, -3, size=(hkv, D)).astype(np.float64)
            kk[p * BS:(p + 1) * BS] = _levels(rng, (BS, hkv, D), ek, 0)[0]
            ev = rng.integers(-10, -3, size=(BS, hkv)).astype(np.float64)
            vv[p * BS:(p + 1) * BS] = _levels(rng, (BS, hkv, D), ev, 2)[0]
        f = n // BS * BS
        kk[f:] = bf16_bits_to_f32(f32_to_bf16_bits(
            rng.standard_normal((n - f, hkv, D)).astype(np.float32)))
        vv[f:] = bf16_bits_to_f32(f32_to_bf16_bits(
            rng.standard_normal((n - f, hkv, D)).astype(np.float32)))
        ks.append(kk)
        vs.append(vv)
    return ks, vs, bt, nb


def _append_all(oracle_mod, ks, vs, bt, nb, hkv, splits=None):
    """Append every sequence's tokens, in calls that cut each sequence at
    the positions in splits[b] (None: one call)."""
    lens = [k.shape[0] for k in ks]
    c = oracle_mod.KiviCache(nb, hkv, len(lens))
    cuts = [sorted(set([0, n] + list((splits or {}).get(b, [])))) for b, n in enumerate(lens)]
    rounds = max(len(x) - 1 for x in cuts)
    for r in range(rounds):
        cu, kn, vn, cl = [0], [], [], []
        for b in range(len(lens)):
            lo, hi = (cuts[b][r], cuts[b][r + 1]) if r + 1 < len(cuts[b]) else (lens[b], lens[b])
            kn.append(ks[b][lo:hi])
            vn.append(vs[b][lo:hi])
            cu.append(cu[-1] + hi - lo)
            cl.append(hi if r + 1 < len(cuts[b]) else lens[b])
        oracle_mod.kivi_append(c, _bits(np.concatenate(kn)), _bits(np.concatenate(vn)),
                               np.array(cu), np.array(cl), bt)
    return c


def test_kivi_attention_matches_torch_sdpa_float64(oracle_mod):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(75)
    lens = [0, 1, 15, 16, 17, 40, 64]
    for hq, hkv in [(4, 4), (4, 2), (8, 2), (8, 1)]:
        ks, vs, bt, nb = _exact_batch(rng, lens, hkv)
        c = _append_all(oracle_mod, ks, vs, bt, nb, hkv)
        q = f32_to_bf16_bits(rng.standard_normal((len(lens), hq, D)).astype(np.float32))
        out = oracle_mod.kivi_decode_attention(q, c, bt, np.array(lens))
        g = hq // hkv
        for b, n in enumerate(lens):
            if n == 0:
                assert not out[b].any()
                continue
            kk = torch.from_numpy(ks[b].astype(np.float64)).permute(1, 0, 2).repeat_interleave(g, 0)
            vv = torch.from_numpy(vs[b].astype(np.float64)).permute(1, 0, 2).repeat_interleave(g, 0)
            qq = torch.from_numpy(bf16_bits_to_f32(q[b]).astype(np.float64))
            ref = torch.nn.functional.scaled_dot_product_attention(
                qq[:, None, :], kk, vv)[:, 0, :].numpy()
            np.testing.assert_allclose(out[b], ref, rtol=1e-12, atol=1e-12)


def test_kivi_pages_written_only_when_full(oracle_mod):
    rng = np.random.default_rng(76)
    hkv = 2
    k = bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((BS, hkv, D)).astype(np.float32)))
    v = bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((BS, hkv, D)).astype(np.float32)))
    c = oracle_mod.KiviCache(2, hkv, 1)
    bt = np.array([[1]], np.int32)
    oracle_mod.kivi_append(c, _bits(k[:15]), _bits(v[:15]), np.array([0, 15]), np.array([15]), bt)
    assert np.all(c.k_codes == 0xFF) and np.all(np.isnan(c.k_scale))
    assert np.array_equal(c.tail[0, :, 0, :15], f32_to_bf16_bits(k[:15]).transpose(1, 0, 2))
    assert np.array_equal(c.tail[0, :, 1, :15], f32_to_bf16_bits(v[:15]).transpose(1, 0, 2))
    oracle_mod.kivi_append(c, _bits(k[15:]), _bits(v[15:]), np.array([0, 1]), np.array([16]), bt)
    assert np.all(c.k_codes[0] == 0xFF) and c.k_codes[1].max() <= 3
    assert not np.isnan(c.k_scale[1]).any() and not np.isnan(c.v_zero[1]).any()


def test_kivi_append_split_invariance(oracle_mod):
    rng = np.random.default_rng(77)
    lens = [5, 16, 33, 47, 64]
    hkv = 2
    ks, vs, bt, nb = _exact_batch(rng, lens, hkv)
    ref = _append_all(oracle_mod, ks, vs, bt, nb, hkv)
    for splits in ({b: list(range(1, n)) for b, n in enumerate(lens)},
                   {b: sorted(rng.integers(1, max(n, 2), size=3).tolist())
                    for b, n in enumerate(lens)},
                   {2: [16, 32], 3: [15], 4: [17, 18]}):
        c = _append_all(oracle_mod, ks, vs, bt, nb, hkv, splits)
        for a, r in zip(c.fields(), ref.fields()):
            assert np.array_equal(a.view(np.uint8), r.view(np.uint8))
        for b, n in enumerate(lens):
            f = n % BS
            assert np.array_equal(c.tail[b, :, :, :f], ref.tail[b, :, :, :f])
            assert np.array_equal(c.tail[b, :, 0, :f],
                                  f32_to_bf16_bits(ks[b][n - f:]).transpose(1, 0, 2))


def test_kivi_bad_args(oracle_mod):
    c = oracle_mod.KiviCache(2, 1, 1)
    x = np.zeros((3, 1, D), np.uint16)
    bt = np.zeros((1, 2), np.int32)
    with pytest.raises(ValueError):  # more new tokens than the context
        oracle_mod.kivi_append(c, x, x, np.array([0, 3]), np.array([2]), bt)
    with pytest.raises(ValueError):  # context longer than the table
        oracle_mod.kivi_append(c, x, x, np.array([0, 3]), np.array([40]), bt)
    y = np.full((1, 1, D), 0x7F80, np.uint16)  # +inf
    c2 = oracle_mod.KiviCache(2, 1, 1)
    y16 = np.repeat(y, 16, axis=0)
    with pytest.raises(ValueError):
        oracle_mod.kivi_append(c2, y16, y16, np.array([0, 16]), np.array([16]), bt)
    assert math.isnan(float(c2.k_scale[0, 0, 0]))


def test_kivi_uniform_weights_give_the_mean(oracle_mod):
    # every token carries the same key (a constant channel quantises to its
    # zero point exactly, and the tail keeps bf16), so every weight is 1/n
    # and the output is the plain mean of the values, pages and tail alike
    rng = np.random.default_rng(78)
    hkv, hq, n = 2, 4, 40
    key = bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((hkv, D)).astype(np.float32)))
    k = np.broadcast_to(key, (n, hkv, D)).copy()
    v = np.empty((n, hkv, D), np.float32)
    for p in range(n // BS):
        ev = rng.integers(-9, -3, size=(BS, hkv)).astype(np.float64)
        v[p * BS:(p + 1) * BS] = _levels(rng, (BS, hkv, D), ev, 2)[0]
    f = n // BS * BS
    v[f:] = bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((n - f, hkv, D)).astype(np.float32)))
    c = oracle_mod.KiviCache(4, hkv, 1)
    table = np.array([[2, 0, 3]], np.int32)
    oracle_mod.kivi_append(c, _bits(k), _bits(v), np.array([0, n]), np.array([n]), table)
    q = f32_to_bf16_bits(rng.standard_normal((1, hq, D)).astype(np.float32))
    out = oracle_mod.kivi_decode_attention(q, c, table, np.array([n]))
    mean = v.astype(np.float64).mean(axis=0)            # [hkv, D]
    for h in range(hq):
        np.testing.assert_allclose(out[0, h], mean[h // (hq // hkv)], rtol=1e-12, atol=1e-14)
