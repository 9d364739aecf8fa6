"""The exchange of context-parallel decode (block_sparse_attention_10_b200.dcp) on CPU
ranks with gloo: every rank ends with the oracle's single-rank decode result.

The CUDA kernels cannot run here, so the four steps are stand-ins written in this test
on top of the oracle (candidates: the best 15 blocks of the rank's range by (score desc,
id asc) from the oracle's pooled scores; merge: the forced block plus the best 15 of all
ranks' pairs; attend: the oracle's attention restricted to the range; combine: the
log-sum-exp merge).  What is under test is DcpDecoder: the split of the context into
ranges, the order and shapes of the all-gathers, and that every rank issues the same
collectives."""
import os
import sys
import types

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleOps:
    """CPU stand-ins for the four steps (test infrastructure)."""

    @staticmethod
    def workspace(p):
        return None

    @staticmethod
    def candidates(p, n0, n1, ws, cand_score, cand_id):
        bs = p.block_scores
        B, Tq, _ = bs.shape
        cand_score.fill_(float("-inf"))
        cand_id.fill_(-1)
        for b in range(B):
            for t in range(Tq):
                pos = p.seq_lens[b] - Tq + t
                r = pos // 128
                ids = [n for n in range(n0, min(n1, r + 1)) if n != r]
                ids.sort(key=lambda n: (-bs[b, t, n], n))
                for i, n in enumerate(ids[:15]):
                    cand_score[b, t, i] = float(np.float32(bs[b, t, n]))
                    cand_id[b, t, i] = n

    @staticmethod
    def merge(p, cs, ci, sel):
        G, B, Tq, _ = cs.shape
        sel.fill_(-1)
        for b in range(B):
            for t in range(Tq):
                r = (p.seq_lens[b] - Tq + t) // 128
                pairs = {(float(cs[g, b, t, i]), int(ci[g, b, t, i])) for g in range(G) for i in range(16)
                         if 0 <= int(ci[g, b, t, i]) <= r and int(ci[g, b, t, i]) != r}
                best = sorted(pairs, key=lambda x: (-x[0], x[1]))[:min(15, r)]
                ids = sorted([n for _, n in best] + [r])
                sel[b, t, :len(ids)] = torch.tensor(ids, dtype=torch.int32)

    @staticmethod
    def attend(p, n0, n1, sel, part_out, part_lse):
        import oracle
        s = np.full(sel.shape, -1, np.int32)  # the selection restricted to [n0, n1), still ascending
        for b in range(s.shape[0]):
            for t in range(s.shape[1]):
                ids = [int(x) for x in sel[b, t] if n0 <= int(x) < n1]
                s[b, t, :len(ids)] = ids
        out = np.zeros(part_out.shape)
        lse = np.full(part_lse.shape, -np.inf)
        B, Tq = s.shape[:2]
        for b in range(B):
            for t in range(Tq):
                if (s[b, t] >= 0).any():
                    qb = p.q32[b:b + 1, t:t + 1]
                    o, l = oracle.attend(qb, p.kb[b], p.vb[b], s[b:b + 1, t:t + 1],
                                         [p.seq_lens[b] - Tq + t + 1])
                    out[b, t], lse[b, t] = o[0, 0], l[0, 0]
        part_out.copy_(torch.from_numpy(out))
        part_lse.copy_(torch.from_numpy(lse))

    @staticmethod
    def combine(p, po, pl, out, lse):
        po, pl = po.double().numpy(), pl.double().numpy()
        M = pl.max(axis=0)
        w = np.where(np.isfinite(pl), np.exp(pl - M), 0.0)
        L = w.sum(axis=0)
        out.copy_(torch.from_numpy((w[..., None] * po).sum(axis=0) / L[..., None]))
        if lse is not None:
            lse.copy_(torch.from_numpy(M + np.log(L)))


def _problem():
    import oracle
    from block_sparse_attention_10_b200 import synth
    from tests._common import bf16_values, oracle_caches
    w = synth.Workload("dcp_cpu", B=2, Tq=2, Hq=4, Hkv=2, D=128, HI=2, DI=64, seq_len=3000, lmax=3072, needles=3,
                       seed=808)
    inp = synth.make_inputs(w)
    inp.seq_lens = [3000, 1000]
    for tensor in (inp.k, inp.v, inp.ik):
        tensor[1, :, 1000:] = 0
    k, v, ik = oracle_caches(inp)
    q32, qi32 = bf16_values(inp.q), bf16_values(inp.q_idx)
    ref = oracle.decode(q32, qi32, k, v, ik, inp.seq_lens)

    def one(c, b):
        return oracle.Nvfp4(c.data[b:b + 1], c.scale[b:b + 1], c.tensor_scale)

    p = types.SimpleNamespace(q=inp.q, nbmax=w.lmax // 128, seq_lens=inp.seq_lens, q32=q32,
                              block_scores=ref["block_scores"], kb=[one(k, b) for b in range(2)],
                              vb=[one(v, b) for b in range(2)])
    return p, ref


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    from block_sparse_attention_10_b200 import dcp
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        p, ref = _problem()
        dec = dcp.DcpDecoder(p, rank, world, ops=OracleOps)
        B, Tq, Hq, D = p.q.shape
        out = torch.empty(B, Tq, Hq, D, dtype=torch.float64)
        lse = torch.empty(B, Tq, Hq, dtype=torch.float64)
        dec.part_out = dec.part_out.double()
        dec.part_lse = dec.part_lse.double()
        sel = dec.step(out, lse)
        ok = (np.array_equal(sel.numpy(), ref["sel"]),
              float(np.abs(out.numpy() - ref["out"]).max()),
              float(np.abs(lse.numpy() - ref["lse"]).max()),
              (dec.n0, dec.n1))
        res = [None] * world
        dist.all_gather_object(res, ok)
        if rank == 0:
            q.put(res)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 3])
def test_ranks_reach_the_single_rank_result(world):
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = 29700 + world * 10 + (os.getpid() % 500)
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(200)
        assert pr.exitcode == 0
    res = q.get()
    ranges = [r[3] for r in res]
    assert ranges[0][0] == 0 and ranges[-1][1] == 24
    assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
    for same_sel, err_out, err_lse, _ in res:
        assert same_sel
        assert err_out < 1e-9 and err_lse < 1e-9


def test_block_ranges_cover_without_overlap():
    from block_sparse_attention_10_b200 import dcp
    for nb in (1, 7, 512, 4096):
        for G in range(1, min(nb, 9) + 1):
            r = dcp.block_ranges(nb, G)
            assert r[0][0] == 0 and r[-1][1] == nb and all(a < b for a, b in r)
            assert all(r[i][1] == r[i + 1][0] for i in range(G - 1))
