"""Chunked prefill (Tq * HI > 32): the tensor-core indexer (tcgen05) and the whole
msa_decode step against the oracle.

Small cases span several 128-row query tiles, a partial last tile, ragged
lengths, causal diagonals, HI 1..8, DI 64/128 and head weights; the full-size
workload (2 sequences, 4,096-token chunk on a 128K context) is checked on
sampled query tokens, each of which the oracle scores as a one-token step at its
own position (causal truncation; pinned in test_oracle_msa).
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_10_b200 import configs, msa, synth
from tests._common import bf16_values, check_attention, check_selection, oracle_caches
from tests._gpu import problem_from_inputs, run_decode

pytestmark = pytest.mark.gpu


def _custom(B, Tq, Hq, Hkv, HI, DI, lens, lmax, weights=False, seed=7):
    w = synth.Workload("pf", B=B, Tq=Tq, Hq=Hq, Hkv=Hkv, D=128, HI=HI, DI=DI, seq_len=max(lens), lmax=lmax,
                       seed=seed, weights=weights)
    inp = synth.make_inputs(w)
    inp.seq_lens = list(lens)
    for b, L in enumerate(lens):
        inp.k[b, :, L:] = 0
        inp.v[b, :, L:] = 0
        inp.ik[b, :, L:] = 0
    return inp


CASES = {
    "tq256_hi8_di128": lambda: _custom(2, 256, 32, 4, 8, 128, [2560, 1500], 2560),
    "tq100_hi4_di64_partial_tile": lambda: _custom(1, 100, 8, 1, 4, 64, [3000], 3072),
    "tq40_hi2_weights_ragged": lambda: _custom(3, 40, 16, 2, 2, 128, [5000, 40, 777], 5120, weights=True),
    "tq33_hi1_di64": lambda: _custom(2, 33, 8, 8, 1, 64, [129, 4100], 4224),
}


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    inp = CASES[request.param]()
    return request.param, inp, oracle_caches(inp)


def test_prefill_index_select_attend(case):
    name, inp, (k, v, ik) = case
    p = problem_from_inputs(inp)
    B, Tq = inp.w.B, inp.w.Tq
    bs = torch.full((B, Tq, p.nbmax), float("nan"), device="cuda")
    msa.msa_index(p, bs)
    sel = torch.empty(B, Tq, 16, dtype=torch.int32, device="cuda")
    msa.msa_select(p, bs, sel)
    out, lse, _ = msa.outputs(p)
    msa.msa_attend(p, sel, out, lse)
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    w = None if inp.w_idx is None else inp.w_idx.numpy()
    obs, _ = oracle.index(bf16_values(inp.q_idx), ik, inp.seq_lens, w)
    gbs = bs.cpu().numpy()
    fin = np.isfinite(obs)
    assert np.array_equal(fin, np.isfinite(gbs)), "visibility of blocks differs"
    scale = np.abs(obs[fin]).mean()
    np.testing.assert_allclose(gbs[fin], obs[fin], rtol=1e-4, atol=1e-5 * scale)
    ora_sel = oracle.select(obs, inp.seq_lens)
    check_selection(sel.cpu().numpy(), ora_sel, obs, inp.seq_lens, Tq)
    o, l = oracle.attend(bf16_values(inp.q), k, v, sel.cpu().numpy(), inp.seq_lens)
    check_attention(out.cpu().numpy(), o)
    np.testing.assert_allclose(lse.cpu().numpy(), l, rtol=1e-4, atol=1e-4)
    d = run_decode(p)
    assert np.array_equal(d["sel"], sel.cpu().numpy())


def test_prefill_rejects_max_pooling_and_token_scores():
    inp = CASES["tq33_hi1_di64"]()
    p = problem_from_inputs(inp)
    bs = torch.empty(inp.w.B, inp.w.Tq, p.nbmax, device="cuda")
    p.pool_mode = 1
    with pytest.raises(msa.MsaError) as e:
        msa.msa_index(p, bs)
    assert e.value.code == 2
    p.pool_mode = 0
    ts = torch.empty(inp.w.B, inp.w.Tq, p.ik.data.shape[2], device="cuda")
    with pytest.raises(msa.MsaError) as e:
        msa.msa_index(p, bs, ts)
    assert e.value.code == 2


def test_prefill_full_size_sampled_tokens():
    w = configs.PREFILL_4K_ON_128K
    inp = synth.make_inputs(w, device="cuda")
    p = msa.MsaProblem(seq_lens=torch.tensor(inp.seq_lens, dtype=torch.int32, device="cuda"),
                       k=msa.encode_cache(inp.k, inp.s_k), v=msa.encode_cache(inp.v, inp.s_v),
                       ik=msa.encode_cache(inp.ik, inp.s_ik), q=inp.q.contiguous(), q_idx=inp.q_idx.contiguous(),
                       status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    s_k, s_v, s_ik = inp.s_k, inp.s_v, inp.s_ik
    del inp
    torch.cuda.empty_cache()
    ws = msa.alloc_workspace(p)
    out, lse, sel = msa.outputs(p)
    msa.msa_decode(p, ws, out, lse, sel)
    torch.cuda.synchronize()
    assert int(p.status.item()) == 0
    sel_h, out_h = sel.cpu().numpy(), out.cpu().numpy()
    assert np.isfinite(out_h).all()
    L = w.seq_len
    tokens = [0, 1, 127, 128, 2047, 2048, 4000, 4095]
    for b in range(w.B):
        qi = bf16_values(p.q_idx[b])                      # [Tq, HI, DI]
        ik32 = torch.zeros(1, 1, w.lmax, w.DI)
        ik32[0, :, :L] = synth.kv_tokens(w, synth.TID_IK, b, 1, w.DI, 0, L)
        ik = oracle.nvfp4_encode(ik32.numpy(), s_ik)
        assert np.array_equal(ik.data[0, 0], p.ik.data[b, 0].cpu().numpy())
        n = len(tokens)
        ikb = oracle.Nvfp4(np.repeat(ik.data, n, 0), np.repeat(ik.scale, n, 0), s_ik)
        pos = [L - w.Tq + t for t in tokens]
        obs, _ = oracle.index(qi[tokens][:, None], ikb, [x + 1 for x in pos])
        osel = oracle.select(obs, [x + 1 for x in pos])
        check_selection(sel_h[b, tokens][:, None], osel, obs, [x + 1 for x in pos], 1)
        # attention for the sampled tokens on the GPU's selection
        blocks = sorted({int(x) for t in tokens for x in sel_h[b, t] if x >= 0})
        kd = np.zeros((1, w.Hkv, w.lmax, w.D // 2), np.uint8)
        ksc = np.zeros((1, w.Hkv, w.lmax, w.D // 16), np.uint8)
        vd, vsc = kd.copy(), ksc.copy()
        for nblk in blocks:
            t0, t1 = nblk * 128, min(L, (nblk + 1) * 128)
            kb = oracle.nvfp4_encode(synth.kv_tokens(w, synth.TID_K, b, w.Hkv, w.D, t0, t1).numpy(), s_k)
            vb = oracle.nvfp4_encode(synth.kv_tokens(w, synth.TID_V, b, w.Hkv, w.D, t0, t1).numpy(), s_v)
            kd[0, :, t0:t1], ksc[0, :, t0:t1] = kb.data, kb.scale
            vd[0, :, t0:t1], vsc[0, :, t0:t1] = vb.data, vb.scale
        K = oracle.Nvfp4(np.repeat(kd, n, 0), np.repeat(ksc, n, 0), s_k)
        V = oracle.Nvfp4(np.repeat(vd, n, 0), np.repeat(vsc, n, 0), s_v)
        q = bf16_values(p.q[b])[tokens][:, None]
        o, _ = oracle.attend(q, K, V, sel_h[b, tokens][:, None], [x + 1 for x in pos])
        check_attention(out_h[b, tokens][:, None], o)
