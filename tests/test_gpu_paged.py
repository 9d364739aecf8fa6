"""Paged caches (a block table mapping each 128-token block to a page of a shared pool)
against the same problem with contiguous caches: identical arithmetic, so every output is
bitwise equal — pooled scores, token scores, selection, attention, lse — for decode (warp
and CTA selection, clusters of 4/8/16), multi-token causal rows and chunked prefill (the
tensor-core indexer).  Unused pages hold garbage, so a read of a wrong page would show.
A page id outside the pool sets MSA_STATUS_PAGE and reads page 0 instead (no fault).
The paged path is also checked against the oracle directly (selection, fp32 and bf16
attention output), so a block-table error shared by both layouts would still show."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_10_b200 import msa, synth
from tests._common import bf16_values, check_attention, check_attention_bf16, check_selection, oracle_caches
from tests._gpu import paged_problem, problem_from_inputs, run_decode, run_steps, status_of

pytestmark = pytest.mark.gpu


def _case(B, Tq, Hq, Hkv, HI, DI, lens, lmax, needles=2, seed=11):
    w = synth.Workload("paged", B=B, Tq=Tq, Hq=Hq, Hkv=Hkv, D=128, HI=HI, DI=DI, seq_len=max(lens), lmax=lmax,
                       needles=needles, seed=seed)
    inp = synth.make_inputs(w)
    inp.seq_lens = list(lens)
    for b, L in enumerate(lens):
        inp.k[b, :, L:] = 0
        inp.v[b, :, L:] = 0
        inp.ik[b, :, L:] = 0
    return inp


CASES = {
    "gqa8_di128_clusters4": lambda: _case(40, 1, 32, 4, 8, 128, [3000 + 97 * i for i in range(40)], 7168),
    "di64_tq4_clusters16": lambda: _case(2, 4, 8, 1, 4, 64, [5000, 777], 5120),
    "long_rows_cta_select": lambda: _case(2, 1, 8, 1, 4, 64, [140000, 131200], 140032, needles=3),
    "prefill_tq64_hi8": lambda: _case(2, 64, 16, 2, 8, 128, [2500, 700], 2560, needles=0),
}


@pytest.mark.parametrize("name", list(CASES))
def test_paged_equals_contiguous(name):
    inp = CASES[name]()
    p = problem_from_inputs(inp)
    pp = paged_problem(p, seed=len(name))
    assert pp.nbmax == p.nbmax
    prefill = inp.w.Tq * inp.w.HI > 32
    if not prefill:  # the prefill indexer has no per-token output
        a, b = run_steps(p), run_steps(pp)
        for key in ("block_scores", "token_scores", "sel", "out", "lse"):
            assert np.array_equal(np.nan_to_num(a[key]).view(np.uint32), np.nan_to_num(b[key]).view(np.uint32)), key
    d, e = run_decode(p), run_decode(pp)
    assert status_of(p) == 0 and status_of(pp) == 0
    for key in ("sel", "out", "lse"):
        assert np.array_equal(d[key].view(np.uint32), e[key].view(np.uint32)), key


@pytest.mark.parametrize("name", list(CASES))
def test_paged_matches_oracle(name):
    inp = CASES[name]()
    k, v, ik = oracle_caches(inp)
    pp = paged_problem(problem_from_inputs(inp), seed=len(name) + 3)
    d = run_decode(pp)
    assert status_of(pp) == 0
    Tq = inp.w.Tq
    bs, _ = oracle.index(bf16_values(inp.q_idx), ik, inp.seq_lens)
    check_selection(d["sel"], oracle.select(bs, inp.seq_lens), bs, inp.seq_lens, Tq)
    out, lse = oracle.attend(bf16_values(inp.q), k, v, d["sel"], inp.seq_lens)
    check_attention(d["out"], out)
    np.testing.assert_allclose(d["lse"], lse, rtol=1e-4, atol=1e-4)
    pp.out_bf16 = True
    d16 = run_decode(pp)
    assert status_of(pp) == 0
    assert np.array_equal(d16["sel"], d["sel"])
    check_attention_bf16(d16["out"], out)


def test_page_outside_pool_is_flagged():
    inp = CASES["di64_tq4_clusters16"]()
    pp = paged_problem(problem_from_inputs(inp))
    npages = pp.ik.data.shape[0]
    pp.block_table[0, 3] = npages + 5
    pp.block_table[1, 0] = -2  # changed in place: same address, the cached parameter block stays valid
    d = run_decode(pp)
    assert status_of(pp) & 8  # MSA_STATUS_PAGE
    assert np.isfinite(d["out"]).all()
