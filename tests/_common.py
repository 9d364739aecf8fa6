"""Shared test helpers: golden fixture parsing and oracle-side input preparation."""
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def golden_dict(name):
    return {p[0]: p[1:] for p in golden_lines(name)}


def bf16_values(t: torch.Tensor) -> np.ndarray:
    """fp32 numpy copy of a bf16 tensor's values (exact)."""
    return t.detach().to("cpu", torch.float32).numpy()


def oracle_caches(inp):
    """Encode the fp32 caches of a synth.Inputs with the oracle's NVFP4 encoder."""
    import oracle
    k = oracle.nvfp4_encode(inp.k.numpy(), inp.s_k) if inp.k is not None else None
    v = oracle.nvfp4_encode(inp.v.numpy(), inp.s_v) if inp.v is not None else None
    ik = oracle.nvfp4_encode(inp.ik.numpy(), inp.s_ik)
    return k, v, ik


def oracle_decode_inputs(inp, pool_mode=0):
    import oracle
    k, v, ik = oracle_caches(inp)
    w = None if inp.w_idx is None else inp.w_idx.numpy()
    res = oracle.decode(bf16_values(inp.q), bf16_values(inp.q_idx), k, v, ik, inp.seq_lens, w, pool_mode)
    res["caches"] = (k, v, ik)
    return res


# ----------------------------------------------------------------------------- parity helpers

SEL_EXEMPT_REL = 1e-4     # selection: blocks within 1e-4 relative of the cutoff are exempt
ATT_MAX_ABS = 5e-3        # attention: max-abs vs the oracle
ATT_REL_L2 = 1e-3         # attention: relative L2 vs the oracle


def check_selection(gpu_sel, ora_sel, ora_scores, seq_lens, Tq):
    """GPU selection == oracle selection except for blocks whose oracle pooled score lies
    within SEL_EXEMPT_REL (relative) of the cutoff (lowest selected non-forced oracle score).
    Returns the number of exempted differences."""
    gpu_sel = np.asarray(gpu_sel)
    ora_sel = np.asarray(ora_sel)
    B = gpu_sel.shape[0]
    exempt = 0
    for b in range(B):
        for t in range(Tq):
            pos = seq_lens[b] - Tq + t
            r = pos // 128
            nvis = r + 1
            gs = [int(x) for x in gpu_sel[b, t] if x >= 0]
            os_ = [int(x) for x in ora_sel[b, t] if x >= 0]
            assert gs == sorted(gs) and len(set(gs)) == len(gs), (b, t, gs)
            assert r in gs, (b, t, "recent block missing")
            assert len(gs) == min(16, nvis), (b, t, len(gs))
            assert all(0 <= x < nvis for x in gs)
            assert list(gpu_sel[b, t, len(gs):]) == [-1] * (16 - len(gs))
            diff = set(gs) ^ set(os_)
            if not diff:
                continue
            s = ora_scores[b, t]
            others = [x for x in os_ if x != r]
            cut = min(s[x] for x in others)
            for n in diff:
                assert abs(s[n] - cut) <= SEL_EXEMPT_REL * abs(cut), (b, t, n, s[n], cut)
                exempt += 1
    return exempt


def check_attention(gpu_out, ora_out):
    g = np.asarray(gpu_out, dtype=np.float64)
    o = np.asarray(ora_out, dtype=np.float64)
    assert np.isfinite(g).all()
    max_abs = np.abs(g - o).max()
    rel = np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30)
    assert max_abs <= ATT_MAX_ABS, max_abs
    assert rel <= ATT_REL_L2, rel
    return max_abs, rel
