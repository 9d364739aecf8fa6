"""The largest batch the indexer takes: B = 4,096 sequences, whose per-sequence tables then
fill 32 KB of the decode indexer's shared memory in every CTA (one CTA per SM instead of
two), with short ragged lengths; selection and attention of every row against the oracle.
One sequence more is refused on the host before anything is enqueued (MSA_EUNSUPPORTED,
tests/test_abi_host.py)."""
import dataclasses

import numpy as np
import pytest

import oracle
from block_sparse_attention_10_b200 import synth
from tests._common import bf16_values, check_attention, check_selection, oracle_caches
from tests._gpu import problem_from_inputs, run_decode, status_of

pytestmark = pytest.mark.gpu


def test_largest_batch_every_row():
    w = synth.Workload("maxb", B=4096, Tq=1, Hq=8, Hkv=1, D=128, HI=4, DI=64, seq_len_range=(1, 384),
                       needles=0, seed=97)
    inp = synth.make_inputs(w, device="cuda")
    p = problem_from_inputs(inp)
    d = run_decode(p)
    assert status_of(p) == 0
    host = dataclasses.replace(inp, q=inp.q.cpu(), q_idx=inp.q_idx.cpu(), k=inp.k.cpu(), v=inp.v.cpu(),
                               ik=inp.ik.cpu())
    k, v, ik = oracle_caches(host)
    lens = host.seq_lens
    assert min(lens) < 128 < max(lens)
    bs, _ = oracle.index(bf16_values(host.q_idx), ik, lens)
    check_selection(d["sel"], oracle.select(bs, lens), bs, lens, 1)
    out, lse = oracle.attend(bf16_values(host.q), k, v, d["sel"], lens)
    check_attention(d["out"], out)
    np.testing.assert_allclose(d["lse"], lse, rtol=1e-4, atol=1e-4)
