"""The seeded input generator: determinism, sub-range consistency, shapes of the workloads."""
import numpy as np
import torch

from block_sparse_attention_10_b200 import configs, synth


def test_counter_based_subranges_agree():
    full = synth.normal_tensor(7, synth.TID_K, 3, 4096)
    part = synth.normal_tensor(7, synth.TID_K, 2, 1000, row0=1, col0=3000)
    assert torch.equal(full[1:3, 3000:4000], part)
    other = synth.normal_tensor(8, synth.TID_K, 3, 4096)
    assert not torch.equal(full, other)


def test_normal_statistics():
    x = synth.normal_tensor(3, synth.TID_V, 1, 1 << 20).view(-1).double()
    assert abs(x.mean().item()) < 5e-3
    assert abs(x.std().item() - 1) < 5e-3
    assert x.abs().max().item() < 6.67  # Box-Muller bound sqrt(-2 ln 2^-32)
    m4 = ((x - x.mean()) ** 4).mean() / x.var() ** 2
    assert abs(m4.item() - 3) < 0.05


def test_lowbias32_known_values():
    # integer arithmetic in int64 tensors agrees with plain Python ints
    xs = [0, 1, 2, 0xDEADBEEF, 0xFFFFFFFF, 123456789]
    t = synth.lowbias32(torch.tensor(xs, dtype=torch.int64)).tolist()
    assert t == [synth.lowbias32_int(x) for x in xs]


def test_ragged_lengths_and_needles():
    w = configs.LONG_RAGGED_256K
    lens = synth.seq_lens_for(w)
    assert len(lens) == w.B
    assert all(196608 <= L <= 262144 and L % 128 != 0 for L in lens)
    needles = synth.needle_blocks_for(w, lens)
    for L, nd in zip(lens, needles):
        assert len(nd) == w.needles == len(set(nd))
        assert all(0 <= n and (n + 1) * 128 <= L - w.Tq for n in nd)  # full, before the query's block


def test_small_inputs_shapes_and_needle_shift():
    w = configs.TINY
    inp = synth.make_inputs(w)
    assert inp.q.shape == (1, 1, 8, 128) and inp.q.dtype == torch.bfloat16
    assert inp.q_idx.shape == (1, 1, 4, 64)
    assert inp.ik.shape == (1, 1, 4096, 64) and inp.k.shape == (1, 1, 4096, 128)
    base = synth.kv_tokens(w, synth.TID_IK, 0, 1, 64, 0, 4096)
    qb = synth.qbar(inp.q_idx[0])
    for n in inp.needles[0]:
        blk = slice(n * 128, (n + 1) * 128)
        assert torch.equal(inp.ik[0, :, blk], base[:, blk] + qb * 0.5)
    other = [n for n in range(32) if n not in inp.needles[0]]
    assert torch.equal(inp.ik[0, :, other[0] * 128:(other[0] + 1) * 128], base[:, other[0] * 128:(other[0] + 1) * 128])
