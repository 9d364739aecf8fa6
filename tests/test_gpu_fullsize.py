"""Full-size decode workloads on the GPU (the launch configuration bench.py times:
one msa_decode call over the whole batch), checked on sampled sequences against
the oracle, which regenerates those sequences' inputs on the CPU from the same
counter-based generator.

Per sampled sequence: the oracle scans every index key of the sequence (pooled
scores, selection); attention is compared on the GPU's own selection, for which
the oracle encodes only the selected blocks' K/V (NVFP4 groups are independent,
and the tensor scale is the workload's fixed calibrated scale, so these bytes
equal those of a whole-cache encode).
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_10_b200 import configs, msa, synth
from tests._common import bf16_values, check_attention, check_selection

pytestmark = pytest.mark.gpu


def _gpu_problem(w):
    inp = synth.make_inputs(w, device="cuda")
    p = msa.MsaProblem(seq_lens=torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda"),
                       k=msa.encode_cache(inp.k, inp.s_k), v=msa.encode_cache(inp.v, inp.s_v),
                       ik=msa.encode_cache(inp.ik, inp.s_ik), q=inp.q.contiguous(), q_idx=inp.q_idx.contiguous(),
                       status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    meta = (inp.seq_lens, inp.needles, inp.s_k, inp.s_v, inp.s_ik)
    del inp
    torch.cuda.empty_cache()
    return p, meta


def _check_sequence(w, p, meta, b, sel_gpu, out_gpu):
    seq_lens, needles, s_k, s_v, s_ik = meta
    L = seq_lens[b]
    q, qi, _ = synth.queries(w, [b])
    assert torch.equal(q, p.q[b:b + 1].cpu()) and torch.equal(qi, p.q_idx[b:b + 1].cpu())
    # index keys of the whole sequence, regenerated on the CPU
    ik32 = torch.zeros(1, 1, w.lmax, w.DI)
    ik32[0, :, :L] = synth.index_key_tokens(w, b, 0, L, needles[b], synth.qbar(qi[0]))
    ik = oracle.nvfp4_encode(ik32.numpy(), s_ik)
    # the CPU generator and the GPU generator + GPU encoder agree bit for bit
    assert np.array_equal(ik.data[0, 0, :L], p.ik.data[b, 0, :L].cpu().numpy())
    assert np.array_equal(ik.scale[0, 0, :L], p.ik.scale[b, 0, :L].cpu().numpy())
    bs, _ = oracle.index(bf16_values(qi), ik, [L])
    ora_sel = oracle.select(bs, [L])
    check_selection(sel_gpu[b:b + 1], ora_sel, bs, [L], w.Tq)
    # K/V of the blocks the GPU selected (any token of this sequence)
    blocks = sorted({int(n) for n in sel_gpu[b].reshape(-1) if n >= 0})
    kd = np.zeros((1, w.Hkv, w.lmax, w.D // 2), np.uint8)
    ksc = np.zeros((1, w.Hkv, w.lmax, w.D // 16), np.uint8)
    vd, vsc = kd.copy(), ksc.copy()
    for n in blocks:
        t0, t1 = n * 128, min(L, (n + 1) * 128)
        kb = oracle.nvfp4_encode(synth.kv_tokens(w, synth.TID_K, b, w.Hkv, w.D, t0, t1).numpy(), s_k)
        vb = oracle.nvfp4_encode(synth.kv_tokens(w, synth.TID_V, b, w.Hkv, w.D, t0, t1).numpy(), s_v)
        kd[0, :, t0:t1], ksc[0, :, t0:t1] = kb.data, kb.scale
        vd[0, :, t0:t1], vsc[0, :, t0:t1] = vb.data, vb.scale
        assert np.array_equal(kb.data, p.k.data[b, :, t0:t1].cpu().numpy())
        assert np.array_equal(vb.scale, p.v.scale[b, :, t0:t1].cpu().numpy())
    out, _ = oracle.attend(bf16_values(q), oracle.Nvfp4(kd, ksc, s_k), oracle.Nvfp4(vd, vsc, s_v),
                           sel_gpu[b:b + 1], [L])
    check_attention(out_gpu[b:b + 1], out)
    # needle recall of the committed token: 15 non-forced slots
    found = len(set(needles[b]) & set(int(x) for x in sel_gpu[b, 0]))
    return found >= min(len(needles[b]), 15)


@pytest.mark.parametrize("w,samples", [
    (configs.DECODE_B32_64K, [0, 5, 9, 14, 17, 22, 27, 31]),
    (configs.LONG_RAGGED_256K, list(range(8))),
    (configs.SPEC_VERIFY_512K, list(range(4))),
])
def test_full_size_decode_sampled(w, samples):
    p, meta = _gpu_problem(w)
    ws = msa.alloc_workspace(p)
    out, lse, sel = msa.outputs(p)
    msa.msa_decode(p, ws, out, lse, sel)
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    sel_h, out_h = sel.cpu().numpy(), out.cpu().numpy()
    assert np.isfinite(out_h).all()
    # invariants on every sequence: recent block kept, 16 blocks, <= 2,048 keys
    for b, L in enumerate(meta[0]):
        for t in range(w.Tq):
            pos = L - w.Tq + t
            s = sel_h[b, t]
            assert (s >= 0).sum() == 16 and pos // 128 in s
    recalled = [_check_sequence(w, p, meta, b, sel_h, out_h) for b in samples]
    assert all(recalled), "planted needle blocks not all selected"


def test_repeated_decode_is_deterministic_and_never_times_out():
    """300 back-to-back decode steps on the 32 x 64K workload: every in-kernel wait
    completes (status word stays 0) and every step gives the same bits."""
    w = configs.DECODE_B32_64K
    p, meta = _gpu_problem(w)
    ws = msa.alloc_workspace(p)
    out, lse, sel = msa.outputs(p)
    msa.msa_decode(p, ws, out, lse, sel)
    ref = out.clone()
    acc = torch.zeros_like(out, dtype=torch.int32)
    for _ in range(300):
        msa.msa_decode(p, ws, out, lse, sel)
        acc |= (out.view(torch.int32) ^ ref.view(torch.int32))
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    assert int(acc.abs().max().item()) == 0
