"""End-to-end oracle runs on the tiny workload: invariants of the pages and needle recall."""
import numpy as np

from block_sparse_attention_10_b200 import configs, synth
from tests._common import oracle_decode_inputs


def test_tiny_workload_needles_recalled_and_invariants():
    w = configs.TINY
    inp = synth.make_inputs(w)
    res = oracle_decode_inputs(inp)
    sel = res["sel"][0, 0]
    L = inp.seq_lens[0]
    assert (L - 1) // 128 in sel  # recent block kept
    assert (sel >= 0).sum() == 16  # 32 blocks visible -> 16 selected
    assert set(inp.needles[0]) <= set(sel.tolist())  # planted needles found
    assert np.isfinite(res["out"]).all()
    # needle blocks score clearly above the rest
    bs = res["block_scores"][0, 0]
    others = [n for n in range(32) if n not in inp.needles[0] and n != (L - 1) // 128]
    assert min(bs[n] for n in inp.needles[0]) > max(bs[n] for n in others)
