"""GPU MSA steps (msa_index, msa_select, msa_attend, msa_decode) against the oracle.

Sizes span several tiles and a ragged tail; edge cases: one key, a context that
fits in 16 blocks (dense), partial last blocks, multi-token causal queries, GQA
groups 1..8, indexer heads 1..8, DI 64/128, max pooling, head weights, rows of more
than 1,024 blocks (separate two-level selection launch).
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_10_b200 import configs, msa, synth
from tests._common import (bf16_values, check_attention, check_attention_bf16, check_selection, oracle_caches)
from tests._gpu import problem_from_inputs, run_decode, run_steps, status_of

pytestmark = pytest.mark.gpu


def _custom(name, B, Tq, Hq, Hkv, HI, DI, lens, lmax, needles=0, weights=False, seed=99):
    w = synth.Workload(name, B=B, Tq=Tq, Hq=Hq, Hkv=Hkv, D=128, HI=HI, DI=DI, seq_len=max(lens), lmax=lmax,
                       needles=needles, seed=seed, weights=weights)
    inp = synth.make_inputs(w)
    # ragged lengths: zero the cache past each sequence's own length
    inp.seq_lens = list(lens)
    for b, L in enumerate(lens):
        inp.k[b, :, L:] = 0
        inp.v[b, :, L:] = 0
        inp.ik[b, :, L:] = 0
    return inp


CASES = {
    "tiny_config": lambda: synth.make_inputs(configs.TINY),
    "gqa8_di128_ragged": lambda: _custom("a", 3, 1, 32, 4, 8, 128, [5000, 777, 1280], 5120, needles=4),
    "tq8_di64_causal": lambda: _custom("b", 2, 8, 8, 1, 4, 64, [3000, 9001], 9088, needles=5),
    "g1_hi2_weights": lambda: _custom("c", 2, 4, 4, 4, 2, 64, [4, 2049], 2176, weights=True),
    "g2_hi1_single_key": lambda: _custom("d", 2, 1, 2, 1, 1, 128, [1, 130], 256),
    "tq32_hi1": lambda: _custom("e", 1, 32, 8, 2, 1, 128, [6000], 6016),
    "tq2_hi8_dense": lambda: _custom("f", 2, 2, 16, 2, 8, 128, [2048, 1100], 2048),
    "g4_hi4_tq4": lambda: _custom("g", 3, 4, 16, 4, 4, 64, [20000, 128, 129], 20096, needles=6),
    # rows of > 1,024 blocks: msa_decode selects in its own launch (two-level CTA kernel)
    "long_rows_tq2": lambda: _custom("h", 2, 2, 8, 1, 4, 64, [150000, 133333], 150016, needles=4),
}


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    inp = CASES[request.param]()
    k, v, ik = oracle_caches(inp)
    return request.param, inp, (k, v, ik)


@pytest.mark.parametrize("pool_mode", [0, 1])
def test_steps_match_oracle(case, pool_mode):
    name, inp, (k, v, ik) = case
    p = problem_from_inputs(inp)
    p.pool_mode = pool_mode
    got = run_steps(p)
    assert status_of(p) == 0
    # encoder parity on the same inputs (identical dequantised caches on both sides)
    assert np.array_equal(p.ik.data.cpu().numpy(), ik.data) and np.array_equal(p.ik.scale.cpu().numpy(), ik.scale)
    assert np.array_equal(p.k.data.cpu().numpy(), k.data) and np.array_equal(p.v.scale.cpu().numpy(), v.scale)
    w = None if inp.w_idx is None else inp.w_idx.numpy()
    qi = bf16_values(inp.q_idx)
    bs, ts = oracle.index(qi, ik, inp.seq_lens, w, pool_mode=pool_mode, token_scores=True)
    Tq = inp.w.Tq
    # pooled scores: fp32 tensor-core accumulation vs double
    fin = np.isfinite(bs)
    assert np.array_equal(fin, np.isfinite(got["block_scores"])), "visibility of blocks differs"
    scale = np.abs(bs[fin]).mean() + 1e-30
    np.testing.assert_allclose(got["block_scores"][fin], bs[fin], rtol=1e-4, atol=1e-5 * scale)
    vis = ~np.isnan(ts)
    assert np.array_equal(vis, ~np.isnan(got["token_scores"])), "visible token set differs"
    np.testing.assert_allclose(got["token_scores"][vis], ts[vis], rtol=1e-4, atol=1e-5 * scale)
    # selection (bit-exact up to near-ties at the cutoff)
    ora_sel = oracle.select(bs, inp.seq_lens)
    check_selection(got["sel"], ora_sel, bs, inp.seq_lens, Tq)
    # attention on the GPU's own selection
    out, lse = oracle.attend(bf16_values(inp.q), k, v, got["sel"], inp.seq_lens)
    check_attention(got["out"], out)
    np.testing.assert_allclose(got["lse"], lse, rtol=1e-4, atol=1e-4)


def test_decode_matches_steps(case):
    name, inp, (k, v, ik) = case
    p = problem_from_inputs(inp)
    a = run_steps(p)
    d = run_decode(p)
    assert np.array_equal(a["sel"], d["sel"])
    assert np.array_equal(a["out"].view(np.uint32), d["out"].view(np.uint32))  # same kernels, bitwise
    assert np.array_equal(a["lse"].view(np.uint32), d["lse"].view(np.uint32))
    d2 = run_decode(p)
    assert np.array_equal(d["out"].view(np.uint32), d2["out"].view(np.uint32))  # run-to-run deterministic


def test_tiny_needles_found():
    inp = synth.make_inputs(configs.TINY)
    p = problem_from_inputs(inp)
    d = run_decode(p)
    assert set(inp.needles[0]) <= set(d["sel"][0, 0].tolist())


def test_bf16_output_is_the_rounded_fp32_output(case):
    name, inp, _ = case
    p = problem_from_inputs(inp)
    ws = msa.alloc_workspace(p)
    out32, lse32, sel32 = msa.outputs(p)
    msa.msa_decode(p, ws, out32, lse32, sel32)
    p.out_bf16 = True
    out16, lse16, sel16 = msa.outputs(p)
    assert out16.dtype == torch.bfloat16
    msa.msa_decode(p, ws, out16, lse16, sel16)
    a16 = torch.empty_like(out16)
    msa.msa_attend(p, sel16, a16, None)
    torch.cuda.synchronize()
    assert status_of(p) == 0
    assert torch.equal(sel16, sel32) and torch.equal(lse16, lse32)
    assert torch.equal(out16.view(torch.int16), out32.to(torch.bfloat16).view(torch.int16))
    assert torch.equal(a16.view(torch.int16), out16.view(torch.int16))
    if msa.msa_workspace_size_single_launch(p) > 0:
        o1, _, _ = msa.outputs(p)
        msa.msa_decode_single_launch(p, msa.alloc_workspace_single_launch(p), o1)
        torch.cuda.synchronize()
        p.out_bf16 = False
        o2, _, _ = msa.outputs(p)
        msa.msa_decode_single_launch(p, msa.alloc_workspace_single_launch(p), o2)
        torch.cuda.synchronize()
        assert torch.equal(o1.view(torch.int16), o2.to(torch.bfloat16).view(torch.int16))


def test_bf16_output_matches_oracle(case):
    """bf16 attention output of msa_decode against the oracle rounded to bf16."""
    name, inp, (k, v, ik) = case
    p = problem_from_inputs(inp)
    p.out_bf16 = True
    d = run_decode(p)
    assert status_of(p) == 0
    out, _ = oracle.attend(bf16_values(inp.q), k, v, d["sel"], inp.seq_lens)
    check_attention_bf16(d["out"], out)
