"""One rank's share of a context-parallel decode step, timed on one GPU.

    python -m block_sparse_attention_10_b200.dcp_bench [--workload spec_verify_b4_512k_tq8] [--ranks 1 2 4 8]

For each G, rank G - 1 (which holds the queries' own blocks at the end of the context)
runs its steps on its block range: msa_dcp_candidates (indexer over the range + its best
15 blocks), msa_dcp_merge over G ranks' candidates (all ranks' candidates computed once
beforehand), msa_dcp_attend on its range and msa_dcp_combine of G partials.  Each step is
replayed 50 times from a CUDA graph and timed with CUDA events; the exchanges between ranks
(two NCCL all-gathers) are not part of this single-GPU measurement.  The whole-context
msa_index and msa_decode are timed the same way for reference.  Prints one JSON line per G.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import configs, dcp, msa
from .profile_case import build


def graph_time(fn, n=50, reps=5):
    """Mean ms per call of fn(), replayed from a CUDA graph of n calls; best of reps."""
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for _ in range(3):
            fn(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for _ in range(n):
            fn(s)
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            a.record(s)
            g.replay()
            b.record(s)
        torch.cuda.synchronize()
        best = min(best, a.elapsed_time(b) / n)
    del g
    return best


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default=configs.SPEC_VERIFY_512K.name, choices=sorted(configs.BY_NAME))
    ap.add_argument("--ranks", type=int, nargs="+", default=[1, 2, 4, 8])
    a = ap.parse_args(argv)
    torch.cuda.set_device(0)
    msa.lib()
    w = configs.BY_NAME[a.workload]
    p = build(w, with_kv=True)
    B, Tq, Hq, D = p.q.shape
    out, lse, _ = msa.outputs(p)
    ws = msa.alloc_workspace(p)
    bs = torch.empty(B, Tq, p.nbmax, dtype=torch.float32, device="cuda")
    full_index = graph_time(lambda s: msa.msa_index(p, bs, None, stream=s))
    full_decode = graph_time(lambda s: msa.msa_decode(p, ws, out, lse, None, stream=s))
    wsd = dcp.CudaOps.workspace(p)
    for G in a.ranks:
        ranges = dcp.block_ranges(p.nbmax, G)
        cs = torch.empty(G, B, Tq, 16, dtype=torch.float32, device="cuda")
        ci = torch.empty(G, B, Tq, 16, dtype=torch.int32, device="cuda")
        for g, (n0, n1) in enumerate(ranges):
            msa.msa_dcp_candidates(p, n0, n1, wsd, cs[g], ci[g])
        sel = torch.empty(B, Tq, 16, dtype=torch.int32, device="cuda")
        po = torch.empty(G, B, Tq, Hq, D, dtype=torch.float32, device="cuda")
        pl = torch.empty(G, B, Tq, Hq, dtype=torch.float32, device="cuda")
        msa.msa_dcp_merge(p, cs, ci, sel)
        for g, (n0, n1) in enumerate(ranges):
            msa.msa_dcp_attend(p, n0, n1, sel, po[g], pl[g])
        n0, n1 = ranges[-1]
        t_cand = graph_time(lambda s: msa.msa_dcp_candidates(p, n0, n1, wsd, cs[G - 1], ci[G - 1], stream=s))
        t_merge = graph_time(lambda s: msa.msa_dcp_merge(p, cs, ci, sel, stream=s))
        t_att = graph_time(lambda s: msa.msa_dcp_attend(p, n0, n1, sel, po[G - 1], pl[G - 1], stream=s))
        t_comb = graph_time(lambda s: msa.msa_dcp_combine(p, po, pl, out, lse, stream=s))
        torch.cuda.synchronize()
        assert int(p.status.item()) == 0
        print(json.dumps({"workload": w.name, "ranks": G, "rank": G - 1, "blocks": [n0, n1],
                          "candidates_us": 1e3 * t_cand, "merge_us": 1e3 * t_merge, "attend_us": 1e3 * t_att,
                          "combine_us": 1e3 * t_comb,
                          "rank_step_us": 1e3 * (t_cand + t_merge + t_att + t_comb),
                          "whole_context_index_us": 1e3 * full_index, "whole_context_decode_us": 1e3 * full_decode,
                          "indexer_speedup": full_index / t_cand}), flush=True)
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
