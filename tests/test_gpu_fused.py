"""msa_decode_single_launch (decode_fused.cu) against msa_decode and the oracle: the
same selection, attention within the tolerance (the per-block partials are combined in
another order), workspace contents on entry do not matter (the counters are cleared on
the stream), repeated calls are bitwise identical, the optional outputs may be absent,
and every row of a ragged batch is right (sequences finish their index stream at
different times, so their selection and attention interleave with other sequences'
index work)."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_10_b200 import msa, synth
from tests._common import bf16_values, check_attention, check_selection, oracle_caches
from tests._gpu import problem_from_inputs, run_decode, status_of

pytestmark = pytest.mark.gpu


def _case(B, Tq, Hq, Hkv, HI, DI, lens, lmax, needles=3, seed=5):
    w = synth.Workload("fused", B=B, Tq=Tq, Hq=Hq, Hkv=Hkv, D=128, HI=HI, DI=DI, seq_len=max(lens), lmax=lmax,
                       needles=needles, seed=seed)
    inp = synth.make_inputs(w)
    inp.seq_lens = list(lens)
    for b, L in enumerate(lens):
        inp.k[b, :, L:] = 0
        inp.v[b, :, L:] = 0
        inp.ik[b, :, L:] = 0
    return inp


def test_many_ragged_sequences_match_oracle():
    # 12 sequences from 1 key to 40 blocks: partial last blocks, dense short rows, more
    # sequences than list steps between a sequence's index items and its attention
    lens = [1, 129, 5000, 128, 2047, 2048, 2049, 777, 4096, 3333, 5120, 64]
    inp = _case(12, 1, 16, 2, 8, 128, lens, 5120, needles=2, seed=17)
    p = problem_from_inputs(inp)
    d = run_decode(p, single_launch=True)
    assert status_of(p) == 0
    k, v, ik = oracle_caches(inp)
    bs, _ = oracle.index(bf16_values(inp.q_idx), ik, inp.seq_lens)
    check_selection(d["sel"], oracle.select(bs, inp.seq_lens), bs, inp.seq_lens, 1)
    o, l = oracle.attend(bf16_values(inp.q), k, v, d["sel"], inp.seq_lens)
    check_attention(d["out"], o)
    np.testing.assert_allclose(d["lse"], l, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("DI,HI,Tq,G", [(64, 4, 1, 8), (128, 8, 2, 4), (64, 1, 16, 2), (128, 2, 4, 1)])
def test_single_launch_matches_msa_decode(DI, HI, Tq, G):
    inp = _case(3, Tq, 8, 8 // G, HI, DI, [3000, 9000, 257], 9088, seed=DI + HI + Tq)
    p = problem_from_inputs(inp)
    s = run_decode(p)
    d = run_decode(p, single_launch=True)
    assert status_of(p) == 0
    assert np.array_equal(s["sel"], d["sel"])
    # P is rounded to fp16 after subtracting a running max that depends on how the keys
    # are split between warps: the paths agree to ~1e-4 relative, within the tolerance
    check_attention(d["out"], s["out"])
    assert np.abs(d["out"] - s["out"]).max() <= 1e-3 * np.abs(s["out"]).max()
    np.testing.assert_allclose(d["lse"], s["lse"], rtol=1e-4, atol=1e-4)


def test_garbage_workspace_and_repeats_are_bitwise_stable():
    inp = _case(4, 1, 32, 4, 8, 128, [6000, 6100, 300, 4097], 6144, seed=23)
    p = problem_from_inputs(inp)
    ws = msa.alloc_workspace_single_launch(p)
    ref = run_decode(p, single_launch=True, ws=ws.zero_())
    ws.fill_(0xFF)  # every counter, score, selection and partial slot is garbage on entry
    got = run_decode(p, single_launch=True, ws=ws)
    assert np.array_equal(ref["sel"], got["sel"])
    assert np.array_equal(ref["out"].view(np.uint32), got["out"].view(np.uint32))
    out, lse, sel = msa.outputs(p)
    for _ in range(50):
        msa.msa_decode_single_launch(p, ws, out, lse, sel)
    torch.cuda.synchronize()
    assert status_of(p) == 0
    assert np.array_equal(ref["out"].view(np.uint32), out.cpu().numpy().view(np.uint32))
    assert np.array_equal(ref["lse"].view(np.uint32), lse.cpu().numpy().view(np.uint32))
    assert np.array_equal(ref["sel"], sel.cpu().numpy())


def test_optional_outputs_absent():
    inp = _case(2, 1, 8, 1, 4, 64, [4000, 1000], 4096, seed=31)
    p = problem_from_inputs(inp)
    ref = run_decode(p, single_launch=True)
    ws = msa.alloc_workspace_single_launch(p)
    out, _, _ = msa.outputs(p)
    msa.msa_decode_single_launch(p, ws, out, None, None)
    torch.cuda.synchronize()
    assert status_of(p) == 0
    assert np.array_equal(ref["out"].view(np.uint32), out.cpu().numpy().view(np.uint32))


def test_unsupported_shape_is_refused():
    inp = _case(1, 8, 8, 1, 4, 64, [2000], 2048, needles=0)
    p = problem_from_inputs(inp)
    assert msa.msa_workspace_size_single_launch(p) == 0
    out, _, _ = msa.outputs(p)
    with pytest.raises(msa.MsaError) as e:
        msa.msa_decode_single_launch(p, torch.empty(1 << 20, dtype=torch.uint8, device="cuda"), out)
    assert e.value.code == 2


def test_maximum_batch():
    # B = 4096 (the library's limit): 4,096 ragged short sequences; per-CTA prefix arrays of
    # 2 x 4,097 ints (one CTA per SM for the indexers), a 16,384-CTA attention grid.  The
    # inputs are generated on the GPU (the same bits as on the host) and copied back for
    # the oracle.
    B = 4096
    rng = np.random.default_rng(4096)
    lens = [int(x) for x in rng.integers(1, 641, B)]
    w = synth.Workload("maxb", B=B, Tq=1, Hq=8, Hkv=1, D=128, HI=4, DI=64, seq_len=max(lens), lmax=640,
                       needles=0, seed=41)
    inp = synth.make_inputs(w, device="cuda")
    inp.seq_lens = lens
    for name in ("k", "v", "ik"):  # zero past each sequence's own length, then to the host
        t = getattr(inp, name)
        mask = torch.arange(640, device="cuda")[None, :] < torch.tensor(lens, device="cuda")[:, None]
        t.mul_(mask[:, None, :, None])
        setattr(inp, name, t.cpu())
    inp.q, inp.q_idx = inp.q.cpu(), inp.q_idx.cpu()
    p = problem_from_inputs(inp)
    d = run_decode(p)
    assert status_of(p) == 0
    k, v, ik = oracle_caches(inp)
    bs, _ = oracle.index(bf16_values(inp.q_idx), ik, inp.seq_lens)
    check_selection(d["sel"], oracle.select(bs, inp.seq_lens), bs, inp.seq_lens, 1)
    o, l = oracle.attend(bf16_values(inp.q), k, v, d["sel"], inp.seq_lens)
    check_attention(d["out"], o)
    np.testing.assert_allclose(d["lse"], l, rtol=1e-4, atol=1e-4)
    s = run_decode(p, single_launch=True)
    assert status_of(p) == 0
    assert np.array_equal(s["sel"], d["sel"])
    check_attention(s["out"], o)
