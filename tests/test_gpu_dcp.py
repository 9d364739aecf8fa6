"""Indexer decode context parallelism on one GPU: G = 1, 2, 4, 8 ranks simulated in
sequence (every exchange done by stacking, no kernel waits for another), against the
oracle's single-rank decode and against msa_decode.

The merged selection must equal msa_decode's bit for bit (the same per-block scores,
and the best 15 blocks of the context are among the ranks' best 15); the combined
output must match the oracle within the attention tolerance.  One test gives every rank
its own paged problem whose block table names pages only for the rank's range (-1
elsewhere): a read outside the range would set MSA_STATUS_PAGE, so a clean status shows
that each rank reads only the blocks it holds."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_10_b200 import configs, dcp, msa, synth
from tests._common import bf16_values, check_attention, check_attention_bf16, check_selection, oracle_caches
from tests._gpu import paged_problem, problem_from_inputs, run_decode, status_of

pytestmark = pytest.mark.gpu


def _custom(B, Tq, Hq, Hkv, HI, DI, lens, lmax, needles=3, seed=77):
    w = synth.Workload("dcp", B=B, Tq=Tq, Hq=Hq, Hkv=Hkv, D=128, HI=HI, DI=DI, seq_len=max(lens), lmax=lmax,
                       needles=needles, seed=seed)
    inp = synth.make_inputs(w)
    inp.seq_lens = list(lens)
    for b, L in enumerate(lens):
        inp.k[b, :, L:] = 0
        inp.v[b, :, L:] = 0
        inp.ik[b, :, L:] = 0
    return inp


CASES = {
    # ragged: some ranks hold no visible block of the short sequence, some rows < 16 blocks
    "gqa8_di128_ragged": lambda: _custom(3, 1, 32, 4, 8, 128, [9000, 777, 5001], 9088),
    "tq4_di64_causal": lambda: _custom(2, 4, 8, 1, 4, 64, [20000, 3000], 20096, needles=5),
    "tq8_hi4_long": lambda: _custom(2, 8, 8, 1, 4, 64, [140000, 100001], 140032, needles=6),
}


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    inp = CASES[request.param]()
    k, v, ik = oracle_caches(inp)
    ref = oracle.decode(bf16_values(inp.q), bf16_values(inp.q_idx), k, v, ik, inp.seq_lens)
    return request.param, inp, ref


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_simulated_ranks_match_oracle_and_decode(case, G):
    name, inp, ref = case
    p = problem_from_inputs(inp)
    d = run_decode(p)
    out, lse, _ = msa.outputs(p)
    sel = dcp.simulate_ranks(p, G, out, lse)
    torch.cuda.synchronize()
    assert status_of(p) == 0
    sel_h = sel.cpu().numpy()
    assert np.array_equal(sel_h, d["sel"])  # the single-rank selection, bit for bit
    check_selection(sel_h, ref["sel"], ref["block_scores"], inp.seq_lens, inp.w.Tq)
    o, l = oracle.attend(bf16_values(inp.q), *oracle_caches(inp)[:2], sel_h, inp.seq_lens)
    check_attention(out.cpu().numpy(), o)
    np.testing.assert_allclose(lse.cpu().numpy(), l, rtol=1e-4, atol=1e-4)
    check_attention(out.cpu().numpy(), d["out"])


@pytest.mark.parametrize("pool_mode,weights", [(1, False), (0, True), (1, True)])
def test_simulated_ranks_max_pooling_and_head_weights(pool_mode, weights):
    inp = _custom(2, 4, 16, 2, 4, 64, [20000, 3001], 20096, needles=5, seed=91)
    if weights:
        w = synth.Workload("dcpw", B=2, Tq=4, Hq=16, Hkv=2, D=128, HI=4, DI=64, seq_len=20000, lmax=20096,
                           needles=5, seed=91, weights=True)
        inp.w_idx = synth.queries(w, [0, 1])[2]
    k, v, ik = oracle_caches(inp)
    p = problem_from_inputs(inp)
    p.pool_mode = pool_mode
    d = run_decode(p)
    out, lse, _ = msa.outputs(p)
    sel = dcp.simulate_ranks(p, 3, out, lse)
    torch.cuda.synchronize()
    assert status_of(p) == 0
    assert np.array_equal(sel.cpu().numpy(), d["sel"])
    wts = None if inp.w_idx is None else inp.w_idx.numpy()
    bs, _ = oracle.index(bf16_values(inp.q_idx), ik, inp.seq_lens, wts, pool_mode=pool_mode)
    check_selection(sel.cpu().numpy(), oracle.select(bs, inp.seq_lens), bs, inp.seq_lens, inp.w.Tq)
    o, _ = oracle.attend(bf16_values(inp.q), k, v, sel.cpu().numpy(), inp.seq_lens)
    check_attention(out.cpu().numpy(), o)


def test_bf16_combine(case):
    name, inp, ref = case
    p = problem_from_inputs(inp)
    p.out_bf16 = True
    out, lse, _ = msa.outputs(p)
    sel = dcp.simulate_ranks(p, 4, out, lse)
    torch.cuda.synchronize()
    o, _ = oracle.attend(bf16_values(inp.q), *oracle_caches(inp)[:2], sel.cpu().numpy(), inp.seq_lens)
    check_attention_bf16(out.float().cpu().numpy(), o)


def _rank_problem(p, n0, n1, seed):
    """p as rank [n0, n1) would hold it: a paged pool with pages only for its blocks."""
    pp = paged_problem(p, extra_pages=3, seed=seed)
    bt = pp.block_table.clone()
    bt[:, :n0] = -1
    bt[:, n1:] = -1
    pp.block_table = bt
    return pp


@pytest.mark.parametrize("G", [2, 3])
def test_ranks_read_only_their_own_blocks(case, G):
    name, inp, ref = case
    p = problem_from_inputs(inp)
    d = run_decode(p)
    B, Tq, Hq, D = p.q.shape
    ranges = dcp.block_ranges(p.nbmax, G)
    ranks = [_rank_problem(p, n0, n1, seed=g + 1) for g, (n0, n1) in enumerate(ranges)]
    cs = torch.empty(G, B, Tq, 16, dtype=torch.float32, device="cuda")
    ci = torch.empty(G, B, Tq, 16, dtype=torch.int32, device="cuda")
    for g, (n0, n1) in enumerate(ranges):
        msa.msa_dcp_candidates(ranks[g], n0, n1, dcp.CudaOps.workspace(ranks[g]), cs[g], ci[g])
    sel = torch.empty(B, Tq, 16, dtype=torch.int32, device="cuda")
    msa.msa_dcp_merge(ranks[0], cs, ci, sel)
    po = torch.empty(G, B, Tq, Hq, D, dtype=torch.float32, device="cuda")
    pl = torch.empty(G, B, Tq, Hq, dtype=torch.float32, device="cuda")
    for g, (n0, n1) in enumerate(ranges):
        msa.msa_dcp_attend(ranks[g], n0, n1, sel, po[g], pl[g])
    out, lse, _ = msa.outputs(p)
    msa.msa_dcp_combine(ranks[-1], po, pl, out, lse)
    torch.cuda.synchronize()
    for r in ranks:
        assert status_of(r) == 0  # no page outside a rank's range was read
    assert np.array_equal(sel.cpu().numpy(), d["sel"])
    check_attention(out.cpu().numpy(), d["out"])
    # candidates: per rank, exactly the best min(15, c) blocks of its range other than the
    # query's own block by (score desc, id asc) -- checked against the pooled scores of the
    # whole-context indexer -- ascending by id, inside the range, scores equal to the pooled ones
    cs_h, ci_h = cs.cpu().numpy(), ci.cpu().numpy()
    bs = torch.empty(B, Tq, p.nbmax, dtype=torch.float32, device="cuda")
    msa.msa_index(p, bs)
    bs_h = bs.cpu().numpy()
    for g, (n0, n1) in enumerate(ranges):
        for b in range(B):
            for t in range(Tq):
                ids = ci_h[g, b, t]
                k = int((ids >= 0).sum())
                assert (ids[:k] >= 0).all() and (ids[k:] == -1).all() and ids[15] == -1
                assert ((ids[:k] >= n0) & (ids[:k] < n1)).all()
                assert list(ids[:k]) == sorted(ids[:k])
                assert np.array_equal(cs_h[g, b, t, :k], bs_h[b, t, ids[:k]])
                r = (inp.seq_lens[b] - Tq + t) // 128
                pool = [n for n in range(n0, min(n1, r + 1)) if n != r]
                best = sorted(pool, key=lambda n: (-bs_h[b, t, n], n))[:15]
                assert sorted(best) == list(ids[:k])


def test_full_size_speculative_verify_ranks():
    """The long-context verify workload (4 x 512K, 8 query tokens) over 2, 4 and 8 ranks:
    the selection equals msa_decode's; attention matches it within tolerance."""
    w = configs.SPEC_VERIFY_512K
    inp = synth.make_inputs(w, device="cuda")
    p = msa.MsaProblem(seq_lens=torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda"),
                       k=msa.encode_cache(inp.k, inp.s_k), v=msa.encode_cache(inp.v, inp.s_v),
                       ik=msa.encode_cache(inp.ik, inp.s_ik), q=inp.q.contiguous(), q_idx=inp.q_idx.contiguous(),
                       status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    del inp
    torch.cuda.empty_cache()
    d = run_decode(p)
    for G in (2, 4, 8):
        out, lse, _ = msa.outputs(p)
        sel = dcp.simulate_ranks(p, G, out, lse)
        torch.cuda.synchronize()
        assert status_of(p) == 0
        assert np.array_equal(sel.cpu().numpy(), d["sel"])
        check_attention(out.cpu().numpy(), d["out"])
        np.testing.assert_allclose(lse.cpu().numpy(), d["lse"], rtol=1e-5, atol=1e-5)


def test_argument_errors():
    inp = CASES["tq4_di64_causal"]()
    p = problem_from_inputs(inp)
    B, Tq, Hq, D = p.q.shape
    ws = dcp.CudaOps.workspace(p)
    cs = torch.empty(B, Tq, 16, device="cuda")
    ci = torch.empty(B, Tq, 16, dtype=torch.int32, device="cuda")
    for n0, n1 in ((5, 5), (-1, 3), (0, p.nbmax + 1), (7, 3)):
        with pytest.raises(msa.MsaError) as e:
            msa.msa_dcp_candidates(p, n0, n1, ws, cs, ci)
        assert e.value.code == 1
    with pytest.raises(msa.MsaError) as e:
        msa.msa_dcp_candidates(p, 0, 4, ws[:16], cs, ci)
    assert e.value.code == 4
    sel = torch.empty(B, Tq, 16, dtype=torch.int32, device="cuda")
    with pytest.raises(msa.MsaError) as e:
        msa.msa_dcp_merge(p, cs.expand(33, B, Tq, 16).contiguous(), ci.expand(33, B, Tq, 16).contiguous(), sel)
    assert e.value.code == 2
    with pytest.raises(ValueError):
        dcp.block_ranges(4, 5)
    pf = problem_from_inputs(_custom(1, 64, 8, 1, 8, 64, [3000], 3072))
    with pytest.raises(msa.MsaError) as e:
        msa.msa_dcp_candidates(pf, 0, 8, dcp.CudaOps.workspace(pf), torch.empty(1, 64, 16, device="cuda"),
                               torch.empty(1, 64, 16, dtype=torch.int32, device="cuda"))
    assert e.value.code == 2
