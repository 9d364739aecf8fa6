"""The C ABI's documented error paths on the GPU (status bits of include/msa.h), each
checked against the corrected inputs bit for bit:

* a sequence length outside [Tq, lmax] is clamped into it and flags MSA_STATUS_SEQLEN
  (decode, multi-token rows and chunked prefill with the tensor-core paths);
* a selected block past the row's visible blocks is skipped and flags MSA_STATUS_SELECT.
"""
import dataclasses

import numpy as np
import pytest
import torch

from block_sparse_attention_10_b200 import msa, synth
from tests._gpu import problem_from_inputs, run_decode, status_of

pytestmark = pytest.mark.gpu

SEQLEN, SELECT = 1, 2


def _inputs(Tq, HI, DI, lmax, seed):
    w = synth.Workload("status", B=3, Tq=Tq, Hq=8, Hkv=1, D=128, HI=HI, DI=DI, seq_len=lmax, lmax=lmax,
                       needles=0, seed=seed)
    return synth.make_inputs(w)


@pytest.mark.parametrize("Tq,HI,DI", [(1, 4, 64), (4, 4, 128), (64, 8, 128)])
def test_out_of_range_lengths_are_clamped_and_flagged(Tq, HI, DI):
    lmax = 2048
    inp = _inputs(Tq, HI, DI, lmax, seed=71 + Tq)
    p = problem_from_inputs(inp)
    # above lmax, below Tq, in range
    p.seq_lens.copy_(torch.tensor([lmax + 300, Tq - 1, 1000], dtype=torch.int32))
    fixed = dataclasses.replace(p, seq_lens=torch.tensor([lmax, Tq, 1000], dtype=torch.int32, device="cuda"),
                                status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    got, ref = run_decode(p), run_decode(fixed)
    assert status_of(p) & SEQLEN
    assert status_of(fixed) == 0
    assert status_of(p) & ~SEQLEN == 0
    for key in ("sel", "out", "lse"):
        assert np.array_equal(got[key].view(np.uint32), ref[key].view(np.uint32)), key


def test_selected_block_past_the_row_is_skipped_and_flagged():
    inp = _inputs(1, 4, 64, 3072, seed=83)
    p = problem_from_inputs(inp)
    p.seq_lens.copy_(torch.tensor([1000, 3000, 129], dtype=torch.int32))
    B = 3
    bs = torch.full((B, 1, p.nbmax), float("nan"), device="cuda")
    msa.msa_index(p, bs)
    sel = torch.empty(B, 1, 16, dtype=torch.int32, device="cuda")
    msa.msa_select(p, bs, sel)
    torch.cuda.synchronize()
    assert status_of(p) == 0
    out, lse, _ = msa.outputs(p)
    msa.msa_attend(p, sel, out, lse)
    # rows 0 (8 visible blocks) and 2 (2 visible blocks) are padded with -1: one padding slot
    # of each gets a block id past the row's visible blocks (but inside the cache)
    bad = sel.clone()
    assert int(bad[0, 0, 10]) == -1 and int(bad[2, 0, 5]) == -1
    bad[0, 0, 10] = 20
    bad[2, 0, 5] = 2
    p2 = dataclasses.replace(p, status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    out2, lse2, _ = msa.outputs(p2)
    msa.msa_attend(p2, bad, out2, lse2)
    torch.cuda.synchronize()
    assert status_of(p) == 0
    assert status_of(p2) & SELECT
    assert np.array_equal(out.cpu().numpy().view(np.uint32), out2.cpu().numpy().view(np.uint32))
    assert np.array_equal(lse.cpu().numpy().view(np.uint32), lse2.cpu().numpy().view(np.uint32))
