"""msa_select on crafted pooled scores against the oracle, bit-exact: exact ties (at and
away from the cutoff), rows where every score is equal, negative scores, and row lengths
that reach each selection kernel (one warp per row up to 1,024 blocks, a two-level CTA
up to 4,096, the round-based CTA beyond), also with thousands of such rows."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_10_b200 import msa

pytestmark = pytest.mark.gpu


def _select(scores, seq_lens, Tq):
    B, _, nbmax = scores.shape
    lens = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    bs = torch.tensor(scores, dtype=torch.float32, device="cuda")
    sel = torch.full((B, Tq, 16), 12345, dtype=torch.int32, device="cuda")
    fake = msa._Cache(0x1000, 0x2000, 1.0)  # never read by the selection
    prm = msa._Params(B, Tq, 8, 1, 128, 4, 64, nbmax * 128, lens.data_ptr(), fake, fake, fake, 0x3000, 0x4000,
                      None, 0.0, 0, None)
    r = msa.lib().msa_select(ctypes.byref(prm), ctypes.c_void_p(bs.data_ptr()), ctypes.c_void_p(sel.data_ptr()),
                             None)
    assert r == 0
    torch.cuda.synchronize()
    return sel.cpu().numpy()


def _pattern(kind, rng, n):
    if kind == "distinct":
        return rng.standard_normal(n).astype(np.float32)
    if kind == "few_levels":  # many exact ties everywhere, including at the cutoff
        return rng.integers(0, 6, n).astype(np.float32)
    if kind == "all_equal":
        return np.full(n, 0.75, np.float32)
    if kind == "negative":
        return -np.abs(rng.standard_normal(n)).astype(np.float32) - 1.0
    if kind == "tie_at_cutoff":  # up to 10 clear winners, then up to 40 equal runners-up
        x = rng.uniform(0, 1, n).astype(np.float32)
        idx = rng.permutation(n)
        top = idx[:min(10, n)]
        x[top] = 5.0 + np.arange(len(top), dtype=np.float32)
        x[idx[len(top):50]] = 3.0
        return x
    raise ValueError(kind)


@pytest.mark.parametrize("nbmax", [16, 512, 1024, 2048, 4096, 4608])
@pytest.mark.parametrize("kind", ["distinct", "few_levels", "all_equal", "negative", "tie_at_cutoff"])
def test_select_crafted_scores_bit_exact(nbmax, kind):
    rng = np.random.default_rng(nbmax * 7 + len(kind))
    lmax = nbmax * 128
    Tq = 2
    # visible-block counts from 1 up to the whole row; query t of sequence b sits at L - Tq + t
    lens = sorted({2, 129, 130, 16 * 128 + 1, 17 * 128, lmax // 2 + 5, lmax - 1, lmax} & set(range(2, lmax + 1)))
    B = len(lens)
    scores = np.full((B, Tq, nbmax), -np.inf, np.float32)
    for b, L in enumerate(lens):
        for t in range(Tq):
            nvis = (L - Tq + t) // 128 + 1
            scores[b, t, :nvis] = _pattern(kind, rng, nvis)
    got = _select(scores, lens, Tq)
    want = oracle.select(scores.astype(np.float64), lens)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("nbmax", [1056, 2048])
@pytest.mark.parametrize("kind", ["distinct", "few_levels", "tie_at_cutoff"])
def test_select_many_long_rows_bit_exact(nbmax, kind):
    """Thousands of rows of more than 1,024 blocks, as in a chunk of prefill tokens (the
    two-level CTA kernel, one CTA per row)."""
    rng = np.random.default_rng(nbmax + 3 * len(kind))
    lmax = nbmax * 128
    Tq = 1500
    lens = [lmax, lmax - 1, lmax // 2 + 5, Tq + 1000]
    B = len(lens)
    scores = np.full((B, Tq, nbmax), -np.inf, np.float32)
    for b, L in enumerate(lens):
        for t in range(Tq):
            nvis = (L - Tq + t) // 128 + 1
            scores[b, t, :nvis] = _pattern(kind, rng, nvis)
    got = _select(scores, lens, Tq)
    want = oracle.select(scores.astype(np.float64), lens)
    assert np.array_equal(got, want)
