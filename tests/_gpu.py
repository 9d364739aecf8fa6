"""GPU-side setup for the parity tests: builds an MsaProblem from synth inputs with the
library's own NVFP4 encoder, runs the C ABI, returns host copies."""
import numpy as np
import torch

from block_sparse_attention_10_b200 import msa


def problem_from_inputs(inp, status=True, dev="cuda"):
    w = inp.w
    k = msa.encode_cache(inp.k.to(dev), inp.s_k)
    v = msa.encode_cache(inp.v.to(dev), inp.s_v)
    ik = msa.encode_cache(inp.ik.to(dev), inp.s_ik)
    return msa.MsaProblem(
        seq_lens=torch.tensor(inp.seq_lens, dtype=torch.int32, device=dev), k=k, v=v, ik=ik,
        q=inp.q.to(dev).contiguous(), q_idx=inp.q_idx.to(dev).contiguous(),
        w_idx=None if inp.w_idx is None else inp.w_idx.to(dev).contiguous(),
        status=torch.zeros(1, dtype=torch.int32, device=dev) if status else None)


def run_steps(p):
    """msa_index -> msa_select -> msa_attend as separate calls."""
    B, Tq = p.q.shape[:2]
    bs = torch.full((B, Tq, p.nbmax), float("nan"), dtype=torch.float32, device=p.q.device)
    lmax = p.k.data.shape[2]
    ts = torch.full((B, Tq, lmax), float("nan"), dtype=torch.float32, device=p.q.device)
    msa.msa_index(p, bs, ts)
    sel = torch.empty(B, Tq, 16, dtype=torch.int32, device=p.q.device)
    msa.msa_select(p, bs, sel)
    out, lse, _ = msa.outputs(p)
    msa.msa_attend(p, sel, out, lse)
    torch.cuda.synchronize()
    return dict(block_scores=bs.cpu().numpy(), token_scores=ts.cpu().numpy(), sel=sel.cpu().numpy(),
                out=out.cpu().numpy(), lse=lse.cpu().numpy())


def run_decode(p, single_launch=False, ws=None):
    if ws is None:
        ws = msa.alloc_workspace_single_launch(p) if single_launch else msa.alloc_workspace(p)
    out, lse, sel = msa.outputs(p)
    (msa.msa_decode_single_launch if single_launch else msa.msa_decode)(p, ws, out, lse, sel)
    torch.cuda.synchronize()
    return dict(sel=sel.cpu().numpy(), out=out.cpu().numpy(), lse=lse.cpu().numpy())


def status_of(p):
    return 0 if p.status is None else int(p.status.item())
