"""Pins for the oracle's indexer, block pooling, top-16 selection and attention.

Each pin rests on something other than the oracle itself: brute force written
independently in Python, numpy/torch library routines (matmul, argsort,
scaled_dot_product_attention), closed forms and invariants stated on the pages
("vLLM Adds Day-0 Support for MiniMax-M3.1-Flash", section "A model built for
efficient inference": 128-token blocks, top 16, recent block kept, <= 2,048 keys).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests._common import golden_dict

BLK = 128


def _rand_cache(rng, B, H, lmax, D, s=None):
    x = rng.standard_normal((B, H, lmax, D)).astype(np.float32)
    st = oracle.tensor_scale(x) if s is None else s
    c = oracle.nvfp4_encode(x, st)
    return c, oracle.nvfp4_decode(c)


def _bf16(rng, shape):
    return torch.tensor(rng.standard_normal(shape), dtype=torch.float32).to(torch.bfloat16).float().numpy()


# ----------------------------------------------------------------------------- indexer


def test_index_brute_force_small():
    rng = np.random.default_rng(10)
    B, Tq, HI, DI, lmax = 2, 3, 2, 16, 300
    lens = [300, 131]
    ik, kd = _rand_cache(rng, B, 1, lmax, DI)
    q = _bf16(rng, (B, Tq, HI, DI))
    w = np.abs(rng.standard_normal((B, Tq, HI))).astype(np.float32)
    bs, ts = oracle.index(q, ik, lens, w, token_scores=True)
    for b in range(B):
        for t in range(Tq):
            pos = lens[b] - Tq + t
            sc = []
            for j in range(pos + 1):
                s = 0.0
                for h in range(HI):
                    d = sum(float(q[b, t, h, i]) * float(kd[b, 0, j, i]) for i in range(DI))
                    s += float(w[b, t, h]) * max(d, 0.0)
                sc.append(s)
                assert math.isclose(ts[b, t, j], s, rel_tol=1e-12, abs_tol=1e-12)
            assert np.isnan(ts[b, t, pos + 1:]).all()  # invisible keys are never scored
            for n in range((lmax + BLK - 1) // BLK):
                blk = sc[n * BLK:(n + 1) * BLK]
                if blk:
                    assert math.isclose(bs[b, t, n], sum(blk) / len(blk), rel_tol=1e-12)
                else:
                    assert bs[b, t, n] == -np.inf


def test_index_single_head_positive_is_matmul():
    """HI = 1, w = 1 and every q.k > 0: token scores are a plain matrix product."""
    rng = np.random.default_rng(11)
    B, DI, lmax = 1, 64, 512
    x = np.abs(rng.standard_normal((B, 1, lmax, DI))).astype(np.float32)
    ik = oracle.nvfp4_encode(x, oracle.tensor_scale(x))
    kd = oracle.nvfp4_decode(ik)
    q = np.abs(_bf16(rng, (B, 1, 1, DI))) + 0.01
    _, ts = oracle.index(q, ik, [lmax], token_scores=True)
    ref = kd[0, 0].astype(np.float64) @ q[0, 0, 0].astype(np.float64)
    np.testing.assert_allclose(ts[0, 0], ref, rtol=1e-12)


def test_index_relu_and_head_weights():
    """s(q) + s(-q) = |q.k| for one head, and s is the w-weighted sum of per-head scores."""
    rng = np.random.default_rng(12)
    B, HI, DI, lmax = 1, 4, 32, 256
    ik, kd = _rand_cache(rng, B, 1, lmax, DI)
    q = _bf16(rng, (B, 1, HI, DI))
    w = np.array([[[0.5, 2.0, 0.0, 1.25]]], dtype=np.float32)
    _, ts = oracle.index(q, ik, [lmax], w, token_scores=True)
    per_head = []
    for h in range(HI):
        _, a = oracle.index(q[:, :, h:h + 1], ik, [lmax], token_scores=True)
        _, m = oracle.index(-q[:, :, h:h + 1], ik, [lmax], token_scores=True)
        dot = kd[0, 0].astype(np.float64) @ q[0, 0, h].astype(np.float64)
        np.testing.assert_allclose(a[0, 0] + m[0, 0], np.abs(dot), rtol=1e-12, atol=1e-12)
        per_head.append(a[0, 0])
    ref = sum(float(w[0, 0, h]) * per_head[h] for h in range(HI))
    np.testing.assert_allclose(ts[0, 0], ref, rtol=1e-12)


def test_index_causal_truncation_invariance():
    """Query t of a Tq-token step scores exactly like a 1-token step at length pos_t + 1."""
    rng = np.random.default_rng(13)
    Tq, HI, DI, lmax = 8, 4, 64, 700
    ik, _ = _rand_cache(rng, 1, 1, lmax, DI)
    q = _bf16(rng, (1, Tq, HI, DI))
    L = 645
    bs, _ = oracle.index(q, ik, [L])
    for t in range(Tq):
        pos = L - Tq + t
        b1, _ = oracle.index(q[:, t:t + 1], ik, [pos + 1])
        np.testing.assert_array_equal(bs[0, t], b1[0, 0])


def test_index_max_pooling():
    rng = np.random.default_rng(14)
    ik, _ = _rand_cache(rng, 1, 1, 400, 16)
    q = _bf16(rng, (1, 1, 2, 16))
    bs, ts = oracle.index(q, ik, [390], pool_mode=1, token_scores=True)
    for n in range(4):
        seg = ts[0, 0, n * BLK:min(390, (n + 1) * BLK)]
        assert bs[0, 0, n] == seg.max()


# ----------------------------------------------------------------------------- selection


def _brute_select(scores, pos):
    r = pos // BLK
    others = sorted((n for n in range(r)), key=lambda n: (-scores[n], n))[:15]
    s = sorted([r] + others)
    return s + [-1] * (16 - len(s))


def test_select_brute_force_sort():
    rng = np.random.default_rng(20)
    B, Tq, nb = 3, 4, 40
    lens = [nb * BLK, 17 * BLK + 5, 7 * BLK]
    bs = rng.standard_normal((B, Tq, nb))
    bs[:, :, ::7] = 0.25  # planted exact ties
    sel = oracle.select(bs, lens)
    for b in range(B):
        for t in range(Tq):
            pos = lens[b] - Tq + t
            assert list(sel[b, t]) == _brute_select(bs[b, t], pos)


def test_select_recent_forced_even_if_worst_and_ties_low_index():
    nb = 64
    bs = np.zeros((1, 1, nb))
    bs[0, 0, nb - 1] = -1e30  # the query's own block has the worst score
    sel = oracle.select(bs, [nb * BLK])
    assert list(sel[0, 0]) == list(range(15)) + [nb - 1]  # all others tie -> lowest indices


def test_select_fewer_blocks_than_k_is_dense_and_keys_bounded():
    g = golden_dict("page_figures.txt")
    k, maxk = int(g["top_blocks"][0]), int(g["max_keys_per_query"][0])
    for L in (1, 100, 128, 129, 1500, 2048, 2049, 50000):
        nb = (L + BLK - 1) // BLK
        bs = np.random.default_rng(L).standard_normal((1, 1, nb))
        sel = oracle.select(bs, [L])[0, 0]
        valid = sel[sel >= 0]
        assert len(valid) == min(k, nb)
        assert (L - 1) // BLK in valid
        assert list(valid) == sorted(valid) and len(set(valid)) == len(valid)
        assert sum(min(BLK, L - n * BLK) for n in valid) <= maxk == k * BLK
        if nb <= k:
            assert list(valid) == list(range(nb))


# ----------------------------------------------------------------------------- attention


def _sdpa_masked(q, kd, vd, mask, scale):
    """torch scaled_dot_product_attention in float64 with an explicit boolean mask."""
    qt = torch.tensor(q, dtype=torch.float64)
    kt = torch.tensor(kd, dtype=torch.float64)
    vt = torch.tensor(vd, dtype=torch.float64)
    m = torch.tensor(mask)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale).numpy()


def test_attend_matches_sdpa_with_selection_mask():
    rng = np.random.default_rng(30)
    B, Tq, Hq, Hkv, D, lmax = 2, 3, 8, 2, 32, 40 * BLK
    lens = [40 * BLK - 3, 23 * BLK + 77]
    k, kd = _rand_cache(rng, B, Hkv, lmax, D)
    v, vd = _rand_cache(rng, B, Hkv, lmax, D)
    q = _bf16(rng, (B, Tq, Hq, D))
    bs = rng.standard_normal((B, Tq, lmax // BLK))
    sel = oracle.select(bs, lens)
    out, lse = oracle.attend(q, k, v, sel, lens)
    scale = 1 / math.sqrt(D)
    g = Hq // Hkv
    for b in range(B):
        for t in range(Tq):
            pos = lens[b] - Tq + t
            mask = np.zeros(lmax, dtype=bool)
            for n in sel[b, t]:
                if n >= 0:
                    mask[n * BLK:(n + 1) * BLK] = True
            mask[pos + 1:] = False
            for h in range(Hq):
                ref = _sdpa_masked(q[b, t, h][None], kd[b, h // g], vd[b, h // g], mask[None], scale)[0]
                np.testing.assert_allclose(out[b, t, h], ref, rtol=1e-10, atol=1e-12)
                s = (kd[b, h // g][mask].astype(np.float64) @ q[b, t, h].astype(np.float64)) * scale
                assert math.isclose(lse[b, t, h], np.logaddexp.reduce(s), rel_tol=1e-12)


def test_decode_short_context_equals_dense_causal():
    """With L <= 2,048 every block is selected: MSA decode == dense causal attention."""
    rng = np.random.default_rng(31)
    B, Tq, Hq, Hkv, D, HI, DI, L = 1, 4, 4, 1, 64, 2, 32, 1900
    k, kd = _rand_cache(rng, B, Hkv, L, D)
    v, vd = _rand_cache(rng, B, Hkv, L, D)
    ik, _ = _rand_cache(rng, B, 1, L, DI)
    q = _bf16(rng, (B, Tq, Hq, D))
    qi = _bf16(rng, (B, Tq, HI, DI))
    res = oracle.decode(q, qi, k, v, ik, [L])
    qt = torch.tensor(q[0], dtype=torch.float64).transpose(0, 1)  # [Hq, Tq, D]
    kt = torch.tensor(kd[0], dtype=torch.float64).expand(Hq, L, D)
    vt = torch.tensor(vd[0], dtype=torch.float64).expand(Hq, L, D)
    causal = torch.ones(Tq, L, dtype=torch.bool).tril(diagonal=L - Tq)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=causal).transpose(0, 1).numpy()
    np.testing.assert_allclose(res["out"][0], ref, rtol=1e-10, atol=1e-12)


def test_attend_zero_query_is_mean_and_single_key_is_value():
    rng = np.random.default_rng(32)
    D, lmax = 64, 5 * BLK
    k, kd = _rand_cache(rng, 1, 1, lmax, D)
    v, vd = _rand_cache(rng, 1, 1, lmax, D)
    q = np.zeros((1, 1, 2, D), dtype=np.float32)
    L = 3 * BLK + 10
    sel = np.array([[[1, 3] + [-1] * 14]], dtype=np.int32)
    out, _ = oracle.attend(q, k, v, sel, [L])
    ref = np.concatenate([vd[0, 0, BLK:2 * BLK], vd[0, 0, 3 * BLK:L]]).astype(np.float64).mean(0)
    np.testing.assert_allclose(out[0, 0, 0], ref, rtol=1e-12, atol=1e-14)
    q1 = _bf16(rng, (1, 1, 2, D))
    out1, _ = oracle.attend(q1, k, v, np.array([[[0] + [-1] * 15]], dtype=np.int32), [1])
    np.testing.assert_array_equal(out1[0, 0, 1], vd[0, 0, 0].astype(np.float64))


def test_attend_order_of_selection_irrelevant():
    rng = np.random.default_rng(33)
    D, lmax = 32, 20 * BLK
    k, _ = _rand_cache(rng, 1, 1, lmax, D)
    v, _ = _rand_cache(rng, 1, 1, lmax, D)
    q = _bf16(rng, (1, 1, 4, D))
    s1 = np.array([[[0, 2, 5, 9, 19] + [-1] * 11]], dtype=np.int32)
    s2 = np.array([[[19, -1, 9, 5, -1, 2, 0] + [-1] * 9]], dtype=np.int32)
    o1, _ = oracle.attend(q, k, v, s1, [lmax])
    o2, _ = oracle.attend(q, k, v, s2, [lmax])
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-15)
