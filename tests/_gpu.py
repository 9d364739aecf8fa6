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
    lmax = p.nbmax * 128
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
    return dict(sel=sel.cpu().numpy(), out=out.float().cpu().numpy(), lse=lse.cpu().numpy())


def status_of(p):
    return 0 if p.status is None else int(p.status.item())


def paged_problem(p, extra_pages=7, seed=0, fill=0xAB):
    """The same problem with its caches scattered into shuffled page pools (one page = one
    128-token block of every head) and a block table; unused pages hold garbage."""
    B, nb = p.q.shape[0], p.nbmax
    g = torch.Generator().manual_seed(seed)
    npages = B * nb + extra_pages
    perm = torch.randperm(npages, generator=g)[:B * nb]
    dev = p.q.device
    idx = perm.to(dev)

    def scatter(t):
        H, x = t.shape[1], t.shape[-1]
        blocks = t.view(B, H, nb, 128, x).permute(0, 2, 1, 3, 4).reshape(B * nb, H, 128, x)
        out = torch.full((npages, H, 128, x), fill, dtype=torch.uint8, device=dev)
        out[idx] = blocks
        return out

    def pool(c):
        return msa.Nvfp4Cache(scatter(c.data), scatter(c.scale), c.tensor_scale)

    return msa.MsaProblem(seq_lens=p.seq_lens, k=pool(p.k), v=pool(p.v), ik=pool(p.ik), q=p.q, q_idx=p.q_idx,
                          w_idx=p.w_idx, softmax_scale=p.softmax_scale, pool_mode=p.pool_mode,
                          status=torch.zeros(1, dtype=torch.int32, device=dev),
                          block_table=perm.view(B, nb).to(torch.int32).to(dev))
