"""Run a few launches of one MSA kernel on a synthetic workload, for profilers.

    python -m block_sparse_attention_10_b200.profile_case --workload decode_b32_64k --kernel index --launches 3

Builds the workload's NVFP4 caches on the GPU (library encoder), releases every
temporary so only the kernel's own operands stay allocated, then launches the
chosen step ``--launches`` times on one stream (index = msa_index, select =
msa_select, attend = msa_attend, decode = msa_decode, single =
msa_decode_single_launch) and checks the device status word.  Used to make the ncu summaries under profiles/.
"""
from __future__ import annotations

import argparse
import sys

import torch

from . import configs, msa, synth


def build(w: synth.Workload, with_kv: bool, device="cuda"):
    inp = synth.make_inputs(w, device=device, with_kv=with_kv)
    ik = msa.encode_cache(inp.ik, inp.s_ik)
    if with_kv:
        k = msa.encode_cache(inp.k, inp.s_k)
        v = msa.encode_cache(inp.v, inp.s_v)
    else:  # 1-token placeholders: the indexer never reads K/V
        k = msa.Nvfp4Cache.empty(w.B, w.Hkv, 128, w.D, inp.s_k, device)
        v = msa.Nvfp4Cache.empty(w.B, w.Hkv, 128, w.D, inp.s_v, device)
    p = msa.MsaProblem(seq_lens=torch.tensor(inp.seq_lens, dtype=torch.int32, device=device), k=k, v=v, ik=ik,
                       q=inp.q.contiguous(), q_idx=inp.q_idx.contiguous(), w_idx=None,
                       status=torch.zeros(1, dtype=torch.int32, device=device))
    torch.cuda.synchronize()
    del inp
    return p


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default=configs.DECODE_B32_64K.name, choices=sorted(configs.BY_NAME))
    ap.add_argument("--kernel", default="index", choices=["index", "select", "attend", "decode", "single"])
    ap.add_argument("--launches", type=int, default=3)
    a = ap.parse_args(argv)
    w = configs.BY_NAME[a.workload]
    torch.cuda.set_device(0)
    msa.lib()
    p = build(w, with_kv=a.kernel in ("attend", "decode", "single"))
    lmax = p.ik.data.shape[2]
    B, Tq = w.B, w.Tq
    bs = torch.empty(B, Tq, lmax // 128, dtype=torch.float32, device="cuda")
    sel = torch.empty(B, Tq, 16, dtype=torch.int32, device="cuda")
    out, lse, _ = msa.outputs(p)
    ws = None
    if a.kernel == "decode":
        ws = msa.alloc_workspace(p)
    elif a.kernel == "single":
        ws = msa.alloc_workspace_single_launch(p)
    torch.cuda.empty_cache()
    s = torch.cuda.current_stream()
    if a.kernel in ("select", "attend"):
        msa.msa_index(p, bs, None)
        msa.msa_select(p, bs, sel)
    for _ in range(a.launches):
        if a.kernel == "index":
            msa.msa_index(p, bs, None)
        elif a.kernel == "select":
            msa.msa_select(p, bs, sel)
        elif a.kernel == "attend":
            msa.msa_attend(p, sel, out, lse)
        elif a.kernel == "decode":
            msa.msa_decode(p, ws, out, lse, None)
        else:
            msa.msa_decode_single_launch(p, ws, out, lse, None)
    s.synchronize()
    st = int(p.status.item())
    print(f"profile_case {a.workload} {a.kernel} x{a.launches}: status={st}, "
          f"allocated={torch.cuda.memory_allocated() / 1e9:.2f} GB")
    return 0 if st == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
