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
