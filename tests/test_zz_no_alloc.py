"""msa_decode_static: the decode step for callers that cannot allocate device memory
(e.g. a plugin that a host framework hands only its inputs and outputs).  Its scratch
is a fixed device array inside libmsa.so; this checks it against msa_decode, which
takes caller scratch, on calls in a row (a call must not be disturbed by what an earlier
call left in the shared array; one problem has rows of more than 1,024 blocks, so its
selection goes through the array's selection region), and that oversized problems are
refused.

Collected last on purpose, so a stop-at-first-failure run has already run every
other test before this one."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_10_b200 import configs, msa, synth
from tests._common import check_attention
from tests._gpu import problem_from_inputs, run_decode

pytestmark = pytest.mark.gpu


def _static(p):
    out, lse, sel = msa.outputs(p)
    msa.msa_decode_static(p, out, lse, sel)
    torch.cuda.synchronize()
    return dict(sel=sel.cpu().numpy(), out=out.cpu().numpy(), lse=lse.cpu().numpy())


def _ragged_case():
    w = synth.Workload("noalloc", B=3, Tq=2, Hq=16, Hkv=2, D=128, HI=8, DI=128, seq_len=6000, lmax=6016,
                       needles=4, seed=4242)
    inp = synth.make_inputs(w)
    inp.seq_lens = [6000, 333, 2500]
    for b, L in enumerate(inp.seq_lens):
        inp.k[b, :, L:] = 0
        inp.v[b, :, L:] = 0
        inp.ik[b, :, L:] = 0
    return inp


def _long_rows_case():
    # rows of more than 1,024 blocks: msa_decode runs the selection as its own launch, which
    # writes the selected ids into the second region of the scratch (after the block scores)
    w = synth.Workload("noalloc_long", B=2, Tq=1, Hq=8, Hkv=1, D=128, HI=4, DI=64, seq_len=163000,
                       lmax=163840, needles=6, seed=4243)
    inp = synth.make_inputs(w, device="cuda")
    inp.seq_lens = [163000, 140001]
    L = inp.seq_lens[1]
    inp.k[1, :, L:] = 0
    inp.v[1, :, L:] = 0
    inp.ik[1, :, L:] = 0
    return inp


def test_static_scratch_matches_msa_decode_twice():
    torch.cuda.set_device(0)
    # calls in a row over problems of different shapes (the long-row problem twice, the
    # second time after two other problems overwrote the shared array): stale scratch
    # from an earlier call must not matter
    for make in (_long_rows_case, _ragged_case, lambda: synth.make_inputs(configs.TINY), _long_rows_case):
        inp = make()
        p = problem_from_inputs(inp)
        assert msa.msa_workspace_size(p) <= msa.MSA_STATIC_SCRATCH_BYTES
        ref = run_decode(p)
        got = _static(p)
        assert int(p.status.item()) == 0
        assert np.array_equal(got["sel"], ref["sel"])
        check_attention(got["out"], ref["out"])
        np.testing.assert_allclose(got["lse"], ref["lse"], rtol=1e-5, atol=1e-5)


def test_static_scratch_rejects_oversized_problem():
    # 256 sequences x 1M-token capacity: 8 MiB of block scores > MSA_STATIC_SCRATCH_BYTES.
    # Rejected on the host before anything touches these (fake, never dereferenced) pointers.
    p = msa._Params(256, 1, 8, 1, 128, 4, 64, 1 << 20, 0x1000, msa._Cache(0x2000, 0x3000, 0.01),
                    msa._Cache(0x4000, 0x5000, 0.01), msa._Cache(0x6000, 0x7000, 0.01), 0x8000, 0x9000, None,
                    0.0, 0, None)
    assert msa.lib().msa_workspace_size(ctypes.byref(p)) > msa.MSA_STATIC_SCRATCH_BYTES
    r = msa.lib().msa_decode_static(ctypes.byref(p), ctypes.c_void_p(0x10000), None, None, None)
    assert r == 4  # MSA_EWORKSPACE
