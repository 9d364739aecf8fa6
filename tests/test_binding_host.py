"""The Python binding without a GPU: the ctypes parameter block mirrors the problem
(contiguous and paged caches, output type), is built once and rebuilt after any field is
reassigned, and the output buffers follow the output type."""
import ctypes

import torch

from block_sparse_attention_10_b200 import msa


def _cache(B, H, L, dim):
    return msa.Nvfp4Cache(torch.zeros(B, H, L, dim // 2, dtype=torch.uint8),
                          torch.zeros(B, H, L, dim // 16, dtype=torch.uint8), 0.5)


def _problem(**kw):
    B, Tq, Hq, Hkv, HI, DI, L = 3, 2, 8, 2, 4, 64, 1024
    base = dict(seq_lens=torch.full((B,), L, dtype=torch.int32), k=_cache(B, Hkv, L, 128),
                v=_cache(B, Hkv, L, 128), ik=_cache(B, 1, L, DI),
                q=torch.zeros(B, Tq, Hq, 128, dtype=torch.bfloat16),
                q_idx=torch.zeros(B, Tq, HI, DI, dtype=torch.bfloat16))
    base.update(kw)
    return msa.MsaProblem(**base)


def test_params_mirror_a_contiguous_problem():
    p = _problem()
    prm = p.params()
    assert (prm.B, prm.Tq, prm.Hq, prm.Hkv, prm.D, prm.HI, prm.DI) == (3, 2, 8, 2, 128, 4, 64)
    assert prm.lmax == 1024 and p.nbmax == 8
    assert prm.k.data == p.k.data.data_ptr() and prm.ik.scale == p.ik.scale.data_ptr()
    assert prm.k.tensor_scale == 0.5
    assert prm.block_table is None and prm.num_pages == 0 and prm.out_bf16 == 0


def test_params_mirror_a_paged_problem():
    pages, nb = 40, 16  # pools of 40 pages; 16 blocks (2,048 tokens) per sequence
    table = torch.arange(3 * nb, dtype=torch.int32).view(3, nb) % pages
    p = _problem(k=_cache(pages, 2, 128, 128), v=_cache(pages, 2, 128, 128), ik=_cache(pages, 1, 128, 64),
                 block_table=table)
    prm = p.params()
    assert p.nbmax == nb and prm.lmax == nb * 128
    assert prm.block_table == table.data_ptr() and prm.num_pages == pages


def test_params_are_cached_and_invalidated():
    p = _problem()
    a = p.params()
    assert p.params() is a  # reused while nothing changes
    p.pool_mode = 1
    b = p.params()
    assert b is not a and b.pool_mode == 1
    p.q_idx = torch.zeros(3, 2, 4, 64, dtype=torch.bfloat16)
    c = p.params()
    assert c is not b and c.q_idx == p.q_idx.data_ptr()


def test_output_type_follows_the_flag():
    p = _problem()
    out, lse, sel = msa.outputs(p)
    assert out.dtype == torch.float32 and lse.dtype == torch.float32 and sel.dtype == torch.int32
    p.out_bf16 = True
    assert p.params().out_bf16 == 1
    out, _, _ = msa.outputs(p)
    assert out.dtype == torch.bfloat16 and tuple(out.shape) == (3, 2, 8, 128)


def test_caches_are_immutable():
    c = _cache(1, 1, 128, 64)
    try:
        c.tensor_scale = 2.0
    except Exception as e:  # dataclasses.FrozenInstanceError
        assert "cannot assign" in str(e)
    else:
        raise AssertionError("Nvfp4Cache must be immutable")
    assert ctypes.sizeof(msa._Params) > 0
