"""Chunked prefill (Tq * HI > 32): the tensor-core indexer (tcgen05) and the whole
msa_decode step against the oracle.

Small cases span several 128-row query tiles, a partial last tile, ragged
lengths, causal diagonals, HI 1..8, DI 64/128 and head weights; the full-size
workload (2 sequences, 4,096-token chunk on a 128K context) is checked on 256
sampled query tokens (chunk start and end, every block-boundary class, random),
each of which the oracle scores as a one-token step at its own position (causal
truncation; pinned in test_oracle_msa).
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_10_b200 import configs, msa, synth
from tests._common import (bf16_values, check_attention, check_selection, oracle_attend_rows,
                           oracle_caches, oracle_index_rows)
from tests._gpu import paged_problem, problem_from_inputs, run_decode

pytestmark = pytest.mark.gpu


def _custom(B, Tq, Hq, Hkv, HI, DI, lens, lmax, weights=False, seed=7):
    w = synth.Workload("pf", B=B, Tq=Tq, Hq=Hq, Hkv=Hkv, D=128, HI=HI, DI=DI, seq_len=max(lens), lmax=lmax,
                       seed=seed, weights=weights)
    inp = synth.make_inputs(w)
    inp.seq_lens = list(lens)
    for b, L in enumerate(lens):
        inp.k[b, :, L:] = 0
        inp.v[b, :, L:] = 0
        inp.ik[b, :, L:] = 0
    return inp


CASES = {
    "tq256_hi8_di128": lambda: _custom(2, 256, 32, 4, 8, 128, [2560, 1500], 2560),
    # blocks chosen by more than 16 tokens (several tiles per block), ragged lengths
    "tq1024_hi4_many_tiles": lambda: _custom(2, 1024, 16, 2, 4, 64, [3300, 1030], 3328),
    "tq100_hi4_di64_partial_tile": lambda: _custom(1, 100, 8, 1, 4, 64, [3000], 3072),
    "tq40_hi2_weights_ragged": lambda: _custom(3, 40, 16, 2, 2, 128, [5000, 40, 777], 5120, weights=True),
    "tq33_hi1_di64": lambda: _custom(2, 33, 8, 8, 1, 64, [129, 4100], 4224),
}


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    inp = CASES[request.param]()
    return request.param, inp, oracle_caches(inp)


def test_prefill_index_select_attend(case):
    name, inp, (k, v, ik) = case
    p = problem_from_inputs(inp)
    B, Tq = inp.w.B, inp.w.Tq
    bs = torch.full((B, Tq, p.nbmax), float("nan"), device="cuda")
    msa.msa_index(p, bs)
    sel = torch.empty(B, Tq, 16, dtype=torch.int32, device="cuda")
    msa.msa_select(p, bs, sel)
    out, lse, _ = msa.outputs(p)
    msa.msa_attend(p, sel, out, lse)
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    w = None if inp.w_idx is None else inp.w_idx.numpy()
    obs, _ = oracle.index(bf16_values(inp.q_idx), ik, inp.seq_lens, w)
    gbs = bs.cpu().numpy()
    fin = np.isfinite(obs)
    assert np.array_equal(fin, np.isfinite(gbs)), "visibility of blocks differs"
    scale = np.abs(obs[fin]).mean()
    np.testing.assert_allclose(gbs[fin], obs[fin], rtol=1e-4, atol=1e-5 * scale)
    ora_sel = oracle.select(obs, inp.seq_lens)
    check_selection(sel.cpu().numpy(), ora_sel, obs, inp.seq_lens, Tq)
    o, l = oracle.attend(bf16_values(inp.q), k, v, sel.cpu().numpy(), inp.seq_lens)
    check_attention(out.cpu().numpy(), o)
    np.testing.assert_allclose(lse.cpu().numpy(), l, rtol=1e-4, atol=1e-4)
    # msa_decode: block-major tensor-core attention when Hq / Hkv = 8, else the gather kernel
    d = run_decode(p)
    assert int(p.status.item()) == 0
    assert np.array_equal(d["sel"], sel.cpu().numpy())
    check_attention(d["out"], o)
    np.testing.assert_allclose(d["lse"], l, rtol=1e-4, atol=1e-4)
    d2 = run_decode(p)
    assert np.array_equal(d2["out"].view(np.uint32), d["out"].view(np.uint32))  # bitwise reproducible
    assert np.array_equal(d2["lse"].view(np.uint32), d["lse"].view(np.uint32))


def test_prefill_rejects_max_pooling_and_token_scores():
    inp = CASES["tq33_hi1_di64"]()
    p = problem_from_inputs(inp)
    bs = torch.empty(inp.w.B, inp.w.Tq, p.nbmax, device="cuda")
    p.pool_mode = 1
    with pytest.raises(msa.MsaError) as e:
        msa.msa_index(p, bs)
    assert e.value.code == 2
    p.pool_mode = 0
    ts = torch.empty(inp.w.B, inp.w.Tq, p.ik.data.shape[2], device="cuda")
    with pytest.raises(msa.MsaError) as e:
        msa.msa_index(p, bs, ts)
    assert e.value.code == 2


def _sample_tokens(Tq, L, n, seed):
    """n query tokens of the chunk: its first and last three, every token whose position is
    the first, second or last of a 128-token block, then seeded random tokens."""
    pos0 = L - Tq
    toks = {0, 1, 2, Tq - 3, Tq - 2, Tq - 1}
    toks |= {t for t in range(Tq) if (pos0 + t) % 128 in (0, 1, 127)}
    rng = np.random.default_rng(seed)
    while len(toks) < n:
        toks.add(int(rng.integers(0, Tq)))
    return sorted(toks)


@pytest.mark.parametrize("DI,HI,paged", [(128, 8, False), (64, 4, False), (128, 8, True)])
def test_prefill_indexer_many_units_per_cta(DI, HI, paged):
    """Every CTA of the tensor-core indexer runs several (sequence, 256-key, query-chunk) units
    here (2 x 256 key tiles x 1 chunk over 148 CTAs), and the shorter sequence's units past its
    length see no token, so live and dead units alternate within a CTA: the pooled scores of
    sampled rows must equal the oracle's over every block (each unit's keys come from the key
    tile written during the unit before it).  Both head dims, and a paged cache (bitwise equal
    to the contiguous one as well)."""
    inp = _custom(2, 512, 8, 1, HI, DI, [40000, 65536], 65536, seed=11)
    p = problem_from_inputs(inp)
    B, Tq = inp.w.B, inp.w.Tq
    bs = torch.full((B, Tq, p.nbmax), float("nan"), device="cuda")
    msa.msa_index(p, bs)
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    gbs = bs.cpu().numpy()
    if paged:
        pp = paged_problem(p, seed=5)
        bsp = torch.full((B, Tq, p.nbmax), float("nan"), device="cuda")
        msa.msa_index(pp, bsp)
        torch.cuda.synchronize()
        assert int(pp.status.item()) == 0
        gbsp = bsp.cpu().numpy()
        assert np.array_equal(np.nan_to_num(gbs).view(np.uint32), np.nan_to_num(gbsp).view(np.uint32))
        gbs = gbsp
    ik_all = oracle.nvfp4_encode(inp.ik.numpy(), inp.s_ik)
    for b, L in enumerate(inp.seq_lens):
        tokens = _sample_tokens(Tq, L, 40, seed=200 + b)
        pos = [L - Tq + t for t in tokens]
        ik = oracle.Nvfp4(ik_all.data[b:b + 1], ik_all.scale[b:b + 1], ik_all.tensor_scale)
        obs = oracle_index_rows(bf16_values(inp.q_idx[b])[tokens], ik, pos)
        got = gbs[b, tokens]
        fin = np.isfinite(obs)
        assert np.array_equal(fin, np.isfinite(got)), "visibility of blocks differs"
        scale = np.abs(obs[fin]).mean()
        np.testing.assert_allclose(got[fin], obs[fin], rtol=1e-4, atol=1e-5 * scale)


def test_prefill_full_size_sampled_tokens():
    """The full-size chunked-prefill workload in bench.py's launch configuration (one
    msa_decode over both sequences), checked on 128 sampled query tokens of each sequence
    (256 rows): pooled-score selection and attention against the oracle, which regenerates
    each sequence's caches on the CPU from the counter-based generator and encodes them with
    its own encoder."""
    w = configs.PREFILL_4K_ON_128K
    inp = synth.make_inputs(w, device="cuda")
    p = msa.MsaProblem(seq_lens=torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda"),
                       k=msa.encode_cache(inp.k, inp.s_k), v=msa.encode_cache(inp.v, inp.s_v),
                       ik=msa.encode_cache(inp.ik, inp.s_ik), q=inp.q.contiguous(), q_idx=inp.q_idx.contiguous(),
                       status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    s_k, s_v, s_ik = inp.s_k, inp.s_v, inp.s_ik
    del inp
    torch.cuda.empty_cache()
    ws = msa.alloc_workspace(p)
    out, lse, sel = msa.outputs(p)
    msa.msa_decode(p, ws, out, lse, sel)
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    sel_h, out_h, lse_h = sel.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()
    assert np.isfinite(out_h).all()
    L = w.seq_len
    rows = 0
    for b in range(w.B):
        tokens = _sample_tokens(w.Tq, L, 128, seed=100 + b)
        assert len(tokens) == 128
        pos = [L - w.Tq + t for t in tokens]
        q, qi, _ = synth.queries(w, [b])
        assert torch.equal(q[0], p.q[b].cpu()) and torch.equal(qi[0], p.q_idx[b].cpu())
        # the sequence's caches, generated and encoded on the CPU
        ik32 = np.zeros((1, 1, w.lmax, w.DI), np.float32)
        ik32[0, :, :L] = synth.kv_tokens(w, synth.TID_IK, b, 1, w.DI, 0, L).numpy()
        ik = oracle.nvfp4_encode(ik32, s_ik)
        del ik32
        assert np.array_equal(ik.data[0, 0], p.ik.data[b, 0].cpu().numpy())
        kv = []
        for tid, s in ((synth.TID_K, s_k), (synth.TID_V, s_v)):
            x = np.zeros((1, w.Hkv, w.lmax, w.D), np.float32)
            x[0, :, :L] = synth.kv_tokens(w, tid, b, w.Hkv, w.D, 0, L).numpy()
            kv.append(oracle.nvfp4_encode(x, s))
            del x
        K, V = kv
        assert np.array_equal(K.scale[0, :, :L], p.k.scale[b, :, :L].cpu().numpy())
        assert np.array_equal(V.data[0, :, L - 4096:L], p.v.data[b, :, L - 4096:L].cpu().numpy())
        # selection of every sampled row against the oracle's own pooled scores
        obs = oracle_index_rows(bf16_values(qi[0])[tokens], ik, pos)
        osel = oracle.select(obs[:, None], [x + 1 for x in pos])
        check_selection(sel_h[b, tokens][:, None], osel, obs[:, None], [x + 1 for x in pos], 1)
        # attention of every sampled row over the GPU's selection
        o, l = oracle_attend_rows(bf16_values(q[0])[tokens], K, V, sel_h[b, tokens], pos)
        check_attention(out_h[b, tokens], o)
        np.testing.assert_allclose(lse_h[b, tokens], l, rtol=1e-4, atol=1e-4)
        rows += len(tokens)
    assert rows >= 256
