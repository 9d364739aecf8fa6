"""The C ABI without a GPU: the library loads, exports every function include/msa.h
declares, and rejects bad arguments on the host before anything is enqueued."""
import ctypes
import os
import re

import pytest

from block_sparse_attention_10_b200 import build, msa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return msa.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "msa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\**\s+\**(msa_\w+)\s*\(", src, re.M)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert "msa_decode" in names and "msa_nvfp4_encode" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(msa.EXPORTS)


def test_status_strings(L):
    for code in range(6):
        assert msa.status_string(code).startswith("MSA_")
    assert "unknown" in msa.status_string(99)


def _params(**kw):
    base = dict(B=2, Tq=1, Hq=8, Hkv=1, D=128, HI=4, DI=64, lmax=4096, seq_lens=0x1000,
                k=msa._Cache(0x2000, 0x3000, 0.01), v=msa._Cache(0x4000, 0x5000, 0.01),
                ik=msa._Cache(0x6000, 0x7000, 0.01), q=0x8000, q_idx=0x9000, w_idx=None,
                softmax_scale=0.0, pool_mode=0, status=None)
    base.update(kw)
    return msa._Params(**base)


def _r256(x):
    return (x + 255) // 256 * 256


def test_workspace_size_host_only(L):
    p = _params()
    B, Tq, Hkv, nb = 2, 1, 1, 4096 // 128
    n = L.msa_workspace_size(ctypes.byref(p))
    assert n == _r256(B * Tq * nb * 4) + _r256(B * Tq * 16 * 4)
    assert L.msa_workspace_size(None) == 0
    bad = _params(lmax=4000)
    assert L.msa_workspace_size(ctypes.byref(bad)) == 0
    # the single-launch path: counters, pooled scores, selection, and 8 partials of
    # (8 x 128 + 16) floats per (query row, KV head)
    n1 = L.msa_workspace_size_single_launch(ctypes.byref(p))
    assert n1 == (_r256((4 + B + B * Tq + B * Tq * Hkv) * 4) + _r256(B * Tq * nb * 4) + _r256(B * Tq * 16 * 4) +
                  _r256(B * Tq * Hkv * 8 * 1040 * 4))
    assert L.msa_workspace_size_single_launch(ctypes.byref(_params(Tq=8))) == 0  # Tq * HI > 16
    assert L.msa_workspace_size_single_launch(ctypes.byref(bad)) == 0


def test_block_table_arguments(L):
    # a block table needs a positive page count; the single launch does not take paged caches
    p = _params(block_table=0xA000, num_pages=0)
    assert L.msa_workspace_size(ctypes.byref(p)) == 0
    r = L.msa_decode(ctypes.byref(p), ctypes.c_void_p(0x10000), 1 << 20, ctypes.c_void_p(0x20000), None, None, None)
    assert r == 1
    p = _params(block_table=0xA000, num_pages=64)
    assert L.msa_workspace_size(ctypes.byref(p)) == L.msa_workspace_size(ctypes.byref(_params()))
    assert L.msa_workspace_size_single_launch(ctypes.byref(p)) == 0
    r = L.msa_decode_single_launch(ctypes.byref(p), ctypes.c_void_p(0x10000), 1 << 30, ctypes.c_void_p(0x20000),
                                   None, None, None)
    assert r == 2


def test_params_struct_layout(L):
    # the Python mirror of msa_params_t ends with the block table, the page count and the
    # output type (int, padded to the struct's 8-byte alignment)
    names = [f[0] for f in msa._Params._fields_]
    assert names[-4:] == ["status", "block_table", "num_pages", "out_bf16"]
    assert msa._Params.out_bf16.offset == msa._Params.num_pages.offset + 8
    assert ctypes.sizeof(msa._Params) == msa._Params.out_bf16.offset + 8


def test_out_type_argument(L):
    p = _params(out_bf16=2)
    r = L.msa_decode(ctypes.byref(p), ctypes.c_void_p(0x10000), 1 << 20, ctypes.c_void_p(0x20000), None, None, None)
    assert r == 1


def test_single_launch_rejects_before_enqueueing(L):
    out = ctypes.c_void_p(0x20000)
    r = L.msa_decode_single_launch(ctypes.byref(_params(Tq=8)), ctypes.c_void_p(0x10000), 1 << 30, out, None, None,
                                   None)
    assert r == 2  # MSA_EUNSUPPORTED
    p = _params()
    assert L.msa_decode_single_launch(ctypes.byref(p), ctypes.c_void_p(0x10000), 1024, out, None, None, None) == 4
    assert L.msa_decode_single_launch(ctypes.byref(p), None, 1 << 30, out, None, None, None) == 4
    assert L.msa_decode_single_launch(ctypes.byref(_params(HI=3)), ctypes.c_void_p(0x10000), 1 << 30, out, None,
                                      None, None) == 2


@pytest.mark.parametrize("field,value,code", [
    ("lmax", 4000, 1), ("B", 0, 1), ("Tq", 0, 1), ("seq_lens", None, 1), ("pool_mode", 2, 1),
    ("D", 64, 2), ("DI", 96, 2), ("HI", 3, 2), ("Hq", 24, 2), ("B", 4097, 2), ("B", 5000, 2),
    ("q", 0x8001, 3), ("q_idx", 0x9008, 3),
])
def test_decode_rejects_bad_params(L, field, value, code):
    p = _params(**{field: value})
    ws = ctypes.c_void_p(0x10000)
    r = L.msa_decode(ctypes.byref(p), ws, 1 << 20, ctypes.c_void_p(0x20000), None, None, None)
    assert r == code, (field, r)


def test_prefill_path_is_mean_pooling_only(L):
    # Tq * HI > 32 selects the tensor-core prefill indexer, which pools by mean only
    p = _params(Tq=9, pool_mode=1)
    r = L.msa_decode(ctypes.byref(p), ctypes.c_void_p(0x10000), 1 << 20, ctypes.c_void_p(0x20000), None, None, None)
    assert r == 2
    p = _params(Tq=9)
    assert L.msa_workspace_size(ctypes.byref(p)) > 0


def test_bad_cache_and_workspace(L):
    p = _params(k=msa._Cache(0x2000, 0x3000, 0.0))
    assert L.msa_decode(ctypes.byref(p), ctypes.c_void_p(0x10000), 1 << 20, ctypes.c_void_p(0x20000), None, None,
                        None) == 1
    p = _params(v=msa._Cache(0x4004, 0x5000, 0.01))
    assert L.msa_attend(ctypes.byref(p), ctypes.c_void_p(0x100), ctypes.c_void_p(0x200), None, None) == 3
    p = _params()
    assert L.msa_decode(ctypes.byref(p), ctypes.c_void_p(0x10000), 16, ctypes.c_void_p(0x20000), None, None,
                        None) == 4
    assert L.msa_decode(ctypes.byref(p), None, 1 << 20, ctypes.c_void_p(0x20000), None, None, None) == 4
    assert L.msa_decode(ctypes.byref(p), ctypes.c_void_p(0x10010), 1 << 20, ctypes.c_void_p(0x20000), None, None,
                        None) == 4
    assert L.msa_index(ctypes.byref(p), None, None, None) == 1
    assert L.msa_select(ctypes.byref(p), None, None, None) == 1


def test_codec_rejects_bad_args(L):
    assert L.msa_nvfp4_encode(ctypes.c_void_p(0x100), 4, 24, ctypes.c_float(1.0), ctypes.c_void_p(0x200),
                              ctypes.c_void_p(0x300), None) == 1
    assert L.msa_nvfp4_encode(ctypes.c_void_p(0x100), 4, 32, ctypes.c_float(-1.0), ctypes.c_void_p(0x200),
                              ctypes.c_void_p(0x300), None) == 1
    assert L.msa_nvfp4_encode(ctypes.c_void_p(0x104), 4, 32, ctypes.c_float(1.0), ctypes.c_void_p(0x200),
                              ctypes.c_void_p(0x300), None) == 3
    assert L.msa_nvfp4_encode(None, 0, 32, ctypes.c_float(1.0), None, None, None) == 0  # empty: no-op
    assert L.msa_nvfp4_decode(ctypes.c_void_p(0x100), ctypes.c_void_p(0x100), 4, 32, ctypes.c_float(1.0), None,
                              None) == 1
