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



def check_attention_bf16(gpu_out, ora_out):
    """bf16 attention output (given as its fp32 values) against the fp64 oracle: the fp32
    bounds above plus bf16 rounding.  Element-wise, |gpu - bf16(oracle)| <= ATT_MAX_ABS + one
    bf16 ulp of the oracle value (a GPU value within the fp32 tolerance may round to the
    neighbouring bf16 value); overall, rel-L2(gpu - oracle) <= ATT_REL_L2 + 2^-9, since
    round-to-nearest-even to bf16 moves every element by at most 2^-9 of its magnitude."""
    g = np.asarray(gpu_out, dtype=np.float64)
    o = np.asarray(ora_out, dtype=np.float64)
    assert np.isfinite(g).all()
    o16 = torch.from_numpy(o.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(o), 1e-38))) - 7)
    err = np.abs(g - o16)
    assert (err <= ATT_MAX_ABS + ulp).all(), float((err - ulp).max())
    rel = np.linalg.norm(g - o) / max(np.linalg.norm(o), 1e-30)
    assert rel <= ATT_REL_L2 + 2.0 ** -9, rel
    return float(err.max()), rel

# ----------------------------------------------------------------------------- sampled query rows

def oracle_index_rows(q_idx_rows, ik_seq, positions, group=16):
    """Oracle pooled block scores of single query rows of one sequence at arbitrary positions.

    q_idx_rows fp32 [n, HI, DI]; ik_seq: the sequence's NVFP4 index-key cache [1, 1, lmax, DI/2];
    row i sits at positions[i] and sees keys 0..positions[i] (a one-token step with context
    length positions[i] + 1, which is how the method treats a query at that position).  The rows
    go to the oracle in groups of `group` (the cache repeated once per row of the group).
    Returns float64 [n, lmax / 128]."""
    import oracle
    q_idx_rows = np.ascontiguousarray(q_idx_rows, dtype=np.float32)
    n = q_idx_rows.shape[0]
    nbmax = ik_seq.data.shape[2] // 128
    out = np.empty((n, nbmax), np.float64)
    for i0 in range(0, n, group):
        m = min(group, n - i0)
        ik = oracle.Nvfp4(np.repeat(ik_seq.data, m, 0), np.repeat(ik_seq.scale, m, 0), ik_seq.tensor_scale)
        bs, _ = oracle.index(q_idx_rows[i0:i0 + m, None], ik, [p + 1 for p in positions[i0:i0 + m]])
        out[i0:i0 + m] = bs[:, 0]
    return out


def oracle_attend_rows(q_rows, k_seq, v_seq, sel_rows, positions):
    """Oracle attention of single query rows of one sequence over their own selected blocks.

    q_rows fp32 [n, Hq, D]; k_seq, v_seq: the sequence's NVFP4 caches [1, Hkv, lmax, ...];
    sel_rows int32 [n, 16] (ascending, -1 padded, the row's own block last); row i sits at
    positions[i].  Each row gets a compact cache holding only its selected blocks, in the same
    ascending order, with its own block last and cut at the row's position: the oracle then
    attends over exactly the row's key set, in the same order as over the full cache.
    Returns float64 out [n, Hq, D] and lse [n, Hq]."""
    import oracle
    q_rows = np.ascontiguousarray(q_rows, dtype=np.float32)
    n = q_rows.shape[0]
    Hkv = k_seq.data.shape[1]
    kd = np.zeros((n, Hkv, 16 * 128, k_seq.data.shape[3]), np.uint8)
    ks = np.zeros((n, Hkv, 16 * 128, k_seq.scale.shape[3]), np.uint8)
    vd, vs = np.zeros_like(kd), np.zeros_like(ks)
    sel = np.full((n, 1, 16), -1, np.int32)
    lens = []
    for i in range(n):
        ids = [int(x) for x in sel_rows[i] if x >= 0]
        r = positions[i] // 128
        assert ids == sorted(ids) and ids[-1] == r
        for j, blk in enumerate(ids):
            a, c = blk * 128, blk * 128 + 128
            kd[i, :, j * 128:(j + 1) * 128] = k_seq.data[0, :, a:c]
            ks[i, :, j * 128:(j + 1) * 128] = k_seq.scale[0, :, a:c]
            vd[i, :, j * 128:(j + 1) * 128] = v_seq.data[0, :, a:c]
            vs[i, :, j * 128:(j + 1) * 128] = v_seq.scale[0, :, a:c]
        sel[i, 0, :len(ids)] = np.arange(len(ids))
        lens.append((len(ids) - 1) * 128 + positions[i] - r * 128 + 1)
    out, lse = oracle.attend(q_rows[:, None], oracle.Nvfp4(kd, ks, k_seq.tensor_scale),
                             oracle.Nvfp4(vd, vs, v_seq.tensor_scale), sel, lens)
    return out[:, 0], lse[:, 0]
