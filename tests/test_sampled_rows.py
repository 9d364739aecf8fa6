"""The sampled-row helpers used by the full-size GPU parity tests give exactly what the
oracle gives on the whole problem: scoring rows one at a time at their own positions
equals scoring the chunk of consecutive query tokens, and attention over a row's
compact cache of selected blocks equals attention over the full cache."""
import numpy as np

import oracle
from block_sparse_attention_10_b200 import synth
from tests._common import bf16_values, oracle_attend_rows, oracle_caches, oracle_index_rows


def _inputs():
    w = synth.Workload("rows", B=1, Tq=40, Hq=8, Hkv=2, D=128, HI=2, DI=64, seq_len=3000, lmax=3072,
                       needles=3, seed=321)
    return synth.make_inputs(w)


def test_index_rows_equal_the_chunk():
    inp = _inputs()
    _, _, ik = oracle_caches(inp)
    L, Tq = inp.seq_lens[0], inp.w.Tq
    qi = bf16_values(inp.q_idx)
    full, _ = oracle.index(qi, ik, [L])
    toks = [0, 1, 7, 20, 39]
    rows = oracle_index_rows(qi[0, toks], ik, [L - Tq + t for t in toks], group=2)
    assert np.array_equal(rows, full[0, toks])


def test_attend_rows_equal_the_full_cache():
    inp = _inputs()
    k, v, ik = oracle_caches(inp)
    L, Tq = inp.seq_lens[0], inp.w.Tq
    full = oracle.decode(bf16_values(inp.q), bf16_values(inp.q_idx), k, v, ik, [L])
    toks = [0, 5, 38, 39]
    out, lse = oracle_attend_rows(bf16_values(inp.q)[0, toks], k, v, full["sel"][0, toks],
                                  [L - Tq + t for t in toks])
    np.testing.assert_allclose(out, full["out"][0, toks], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, full["lse"][0, toks], rtol=0, atol=1e-12)


def test_bf16_check_accepts_rounding_and_rejects_errors():
    import pytest
    import torch
    from tests._common import check_attention_bf16
    rng = np.random.default_rng(5)
    o = rng.normal(size=(4, 8, 128)) * 0.3
    g = torch.from_numpy(o.astype(np.float32)).to(torch.bfloat16).float().numpy()
    check_attention_bf16(g, o)
    bad = g.copy()
    bad[1, 2, 3] += 0.05
    with pytest.raises(AssertionError):
        check_attention_bf16(bad, o)
    with pytest.raises(AssertionError):
        check_attention_bf16(g * (1 + 4e-3), o)
