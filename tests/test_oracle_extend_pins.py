"""Pins of the oracle's extend (prefill) attention, CPU only.

Prefill processes a prompt's tokens together and fills the cache; chunked
prefill feeds a long prompt in pieces, each attending to everything cached
before it [KV Cache 优化全景解析——从基础原理到工程实践, §2.2 Prefill 与 Decode
两阶段, §11.2].  The oracle's extend attention gives each new query row the
causal softmax(q K^T / sqrt(d)) V over the dequantised paged cache
[same page, §2.1].  Each pin below fixes it against something other than
itself:
  * torch's scaled_dot_product_attention in float64 with an explicit causal
    mask over the dequantised cache, for every GQA group size;
  * closed forms: a pure prefill's first row is v_hat of token 0 exactly, its
    second row the two-token sigmoid form;
  * causality: changing K/V of later tokens leaves earlier rows unchanged;
  * one new row per sequence is the decode case: the same numbers as the
    oracle's decode attention, pinned on its own;
  * physical block permutation leaves every row unchanged.
"""
import math

import numpy as np
import pytest

from tests.test_oracle_pins import _paged, _rand_seq
from workloads import bf16_bits_to_f32, f32_to_bf16_bits


def _qrows(rng, n, hq):
    return f32_to_bf16_bits(rng.standard_normal((n, hq, 128)).astype(np.float32))


def test_extend_matches_torch_sdpa_causal_float64(oracle_mod):
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(21)
    for hq, hkv in [(8, 8), (8, 4), (8, 2), (8, 1)]:
        lens = [1, 16, 33, 50]
        new = [1, 5, 33, 17]  # 33 of 33: a whole prompt; others extend a cache
        ck, cv, sk, sv = _rand_seq(rng, lens, hkv)
        nb = sum(math.ceil(t / 16) for t in lens) + 2
        kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, lens, hkv=hkv,
                                    perm=rng.permutation(nb))
        qs = np.concatenate([[0], np.cumsum(new)]).astype(np.int32)
        q = _qrows(rng, int(qs[-1]), hq)
        out = oracle_mod.extend_attention(q, kc, vc, ks, vs, bt, np.array(lens), qs)
        g = hq // hkv
        for b, t in enumerate(lens):
            kh = torch.from_numpy(ck[b].astype(np.float64) * sk[b][:, :, None].astype(np.float64))
            vh = torch.from_numpy(cv[b].astype(np.float64) * sv[b][:, :, None].astype(np.float64))
            kk = kh.permute(1, 0, 2).repeat_interleave(g, dim=0)  # [hq, t, D]
            vv = vh.permute(1, 0, 2).repeat_interleave(g, dim=0)
            rows = bf16_bits_to_f32(q[qs[b]:qs[b + 1]]).astype(np.float64)  # [n, hq, D]
            qq = torch.from_numpy(rows).permute(1, 0, 2)  # [hq, n, D]
            pos = torch.arange(t - new[b], t)[:, None]
            mask = torch.arange(t)[None, :] <= pos  # [n, t] causal
            ref = torch.nn.functional.scaled_dot_product_attention(
                qq, kk, vv, attn_mask=mask).permute(1, 0, 2).numpy()
            np.testing.assert_allclose(out[qs[b]:qs[b + 1]], ref, rtol=1e-12,
                                       atol=1e-13)


def test_extend_prefill_first_rows_closed_form(oracle_mod):
    rng = np.random.default_rng(22)
    ck, cv, sk, sv = _rand_seq(rng, [20], 1)
    kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, [20])
    q = _qrows(rng, 20, 2)
    out = oracle_mod.extend_attention(q, kc, vc, ks, vs, bt, np.array([20]),
                                      np.array([0, 20]))
    v = [cv[0][t, 0].astype(np.float64) * np.float64(sv[0][t, 0]) for t in range(2)]
    for h in range(2):
        # row 0 sees token 0 only
        assert np.array_equal(out[0, h], v[0])
        # row 1: two tokens, out = v0 + sigmoid(s1 - s0) (v1 - v0)
        qf = bf16_bits_to_f32(q[1, h]).astype(np.float64)
        s = [float(qf @ (ck[0][t, 0].astype(np.float64) * np.float64(sk[0][t, 0])))
             / math.sqrt(128) for t in range(2)]
        w1 = 1.0 / (1.0 + math.exp(s[0] - s[1]))
        np.testing.assert_allclose(out[1, h], v[0] + w1 * (v[1] - v[0]),
                                   rtol=1e-12, atol=1e-14)


def test_extend_causality(oracle_mod):
    rng = np.random.default_rng(23)
    lens = [45]
    ck, cv, sk, sv = _rand_seq(rng, lens, 2)
    q = _qrows(rng, 30, 4)
    qs = np.array([0, 30])
    a = oracle_mod.extend_attention(q, *_paged(ck, cv, sk, sv, lens, hkv=2)[:5],
                                    np.array(lens), qs)
    # rewrite tokens 30..44: rows at positions 15..29 (the first 15 rows)
    # never see them
    ck2 = [c.copy() for c in ck]
    cv2 = [c.copy() for c in cv]
    ck2[0][30:] = rng.integers(-127, 128, ck2[0][30:].shape)
    cv2[0][30:] = rng.integers(-127, 128, cv2[0][30:].shape)
    b = oracle_mod.extend_attention(q, *_paged(ck2, cv2, sk, sv, lens, hkv=2)[:5],
                                    np.array(lens), qs)
    assert np.array_equal(a[:15], b[:15])
    assert not np.array_equal(a[15:], b[15:])


def test_extend_one_row_is_decode(oracle_mod):
    rng = np.random.default_rng(24)
    lens = [7, 64, 100]
    ck, cv, sk, sv = _rand_seq(rng, lens, 2)
    kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, lens, hkv=2)
    q = _qrows(rng, 3, 8)
    ext = oracle_mod.extend_attention(q, kc, vc, ks, vs, bt, np.array(lens),
                                      np.array([0, 1, 2, 3]))
    dec = oracle_mod.decode_attention(q, kc, vc, ks, vs, bt, np.array(lens))
    assert np.array_equal(ext, dec)


def test_extend_block_permutation_invariance(oracle_mod):
    rng = np.random.default_rng(25)
    lens = [40, 70]
    ck, cv, sk, sv = _rand_seq(rng, lens, 1)
    nb = sum(math.ceil(t / 16) for t in lens) + 2
    q = _qrows(rng, 50, 2)
    qs = np.array([0, 20, 50])
    a = oracle_mod.extend_attention(q, *_paged(ck, cv, sk, sv, lens)[:5],
                                    np.array(lens), qs)
    b = oracle_mod.extend_attention(
        q, *_paged(ck, cv, sk, sv, lens, perm=rng.permutation(nb))[:5],
        np.array(lens), qs)
    assert np.array_equal(a, b)


def test_extend_rejects_more_rows_than_context(oracle_mod):
    rng = np.random.default_rng(26)
    ck, cv, sk, sv = _rand_seq(rng, [5], 1)
    kc, vc, ks, vs, bt = _paged(ck, cv, sk, sv, [5])
    with pytest.raises(ValueError):
        oracle_mod.extend_attention(_qrows(rng, 6, 1), kc, vc, ks, vs, bt,
                                    np.array([5]), np.array([0, 6]))
