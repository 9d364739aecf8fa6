"""CPU oracle for MSA decode over an NVFP4 KV cache (ctypes wrapper of msa_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``.  The CUDA path never imports it,
and it imports nothing from the CUDA path.

Functions take and return numpy arrays.  Definitions and the passages they
follow are in msa_oracle.c.  Parity status of each function:
  nvfp4 codec, indexer, pooling, selection, attention: pinned by the
  `-m "not gpu"` tests (hand-built values, library routines, brute force and
  closed forms).  The readings themselves (indexer form, mean pooling, NVFP4
  layout) are not fixed by the pages: results are checked against these
  documented readings, not against MiniMax's model.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
MSA_BLOCK = 128
MSA_TOPK = 16


def build(force: bool = False) -> str:
    """Compile liboracle.so with gcc (plain C11, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "msa_oracle.h"))):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11",
               "-Wall", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class _Nvfp4(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("tensor_scale", ctypes.c_float),
                ("heads", ctypes.c_int), ("dim", ctypes.c_int), ("lmax", ctypes.c_int64)]


_lib = None


def configure(L):
    """Declare the C signatures on a loaded oracle library."""
    L.orc_e2m1_value.restype = ctypes.c_double
    L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_value.restype = ctypes.c_double
    L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
    L.orc_e4m3_encode.restype = ctypes.c_uint8
    L.orc_e4m3_encode.argtypes = [ctypes.c_float]
    L.orc_e2m1_encode.restype = ctypes.c_uint8
    L.orc_e2m1_encode.argtypes = [ctypes.c_float]
    L.orc_tensor_scale.restype = ctypes.c_float
    L.orc_tensor_scale.argtypes = [ctypes.c_void_p, ctypes.c_int64]
    L.orc_nvfp4_encode.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                                   ctypes.c_void_p, ctypes.c_void_p]
    L.orc_nvfp4_decode.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                   ctypes.c_float, ctypes.c_void_p]
    L.orc_index.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 3 + [ctypes.POINTER(_Nvfp4), ctypes.c_int,
                                                                          ctypes.c_void_p, ctypes.c_void_p]
    L.orc_select.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                             ctypes.c_void_p]
    L.orc_attend.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(_Nvfp4),
                                                  ctypes.POINTER(_Nvfp4), ctypes.c_void_p, ctypes.c_double,
                                                  ctypes.c_void_p, ctypes.c_void_p]
    L.orc_num_threads.restype = ctypes.c_int
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().orc_num_threads()


# --- element formats --------------------------------------------------------

def e2m1_value(code: int) -> float:
    return lib().orc_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return lib().orc_e4m3_value(code)


def e4m3_encode(x: float) -> int:
    return lib().orc_e4m3_encode(x)


def e2m1_encode(x: float) -> int:
    return lib().orc_e2m1_encode(x)


# --- NVFP4 codec ------------------------------------------------------------

class Nvfp4:
    """NVFP4 cache planes: data u8 [..., dim/2], scale u8 [..., dim/16] (E4M3), fp32 tensor scale."""

    def __init__(self, data: np.ndarray, scale: np.ndarray, tensor_scale: float):
        self.data = np.ascontiguousarray(data, dtype=np.uint8)
        self.scale = np.ascontiguousarray(scale, dtype=np.uint8)
        self.tensor_scale = float(np.float32(tensor_scale))

    @property
    def dim(self) -> int:
        return self.data.shape[-1] * 2

    def struct(self) -> _Nvfp4:
        # caches are [B][heads][lmax][...]
        B, H, lmax = self.data.shape[:3]
        return _Nvfp4(self.data.ctypes.data, self.scale.ctypes.data, self.tensor_scale, H, self.dim, lmax)


def tensor_scale(x: np.ndarray) -> float:
    """amax / (6 * 448) in fp32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    return lib().orc_tensor_scale(_ptr(x), x.size)


def nvfp4_encode(x: np.ndarray, s_tensor: float) -> Nvfp4:
    """Quantise fp32 x [..., dim] (dim % 16 == 0) to NVFP4 planes."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    dim = x.shape[-1]
    assert dim % 16 == 0
    nvec = x.size // dim
    data = np.zeros(x.shape[:-1] + (dim // 2,), dtype=np.uint8)
    scale = np.zeros(x.shape[:-1] + (dim // 16,), dtype=np.uint8)
    lib().orc_nvfp4_encode(_ptr(x), nvec, dim, np.float32(s_tensor), _ptr(data), _ptr(scale))
    return Nvfp4(data, scale, s_tensor)


def nvfp4_decode(c: Nvfp4) -> np.ndarray:
    dim = c.dim
    nvec = c.data.size // (dim // 2)
    out = np.empty(c.data.shape[:-1] + (dim,), dtype=np.float32)
    lib().orc_nvfp4_decode(_ptr(c.data), _ptr(c.scale), nvec, dim, np.float32(c.tensor_scale), _ptr(out))
    return out


# --- MSA steps --------------------------------------------------------------

def _seq_lens(seq_lens) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))


def index(q_idx: np.ndarray, ik: Nvfp4, seq_lens, w_idx=None, pool_mode: int = 0, token_scores: bool = False):
    """Indexer scores + block pooling.

    q_idx fp32 [B, Tq, HI, DI] (values of the bf16 queries); ik NVFP4 [B, 1, lmax, DI/2].
    Returns (block_scores float64 [B, Tq, NBmax] with -inf for invisible blocks,
             token_scores float64 [B, Tq, lmax] or None).
    """
    q_idx = np.ascontiguousarray(q_idx, dtype=np.float32)
    B, Tq, HI, DI = q_idx.shape
    assert ik.dim == DI and ik.data.shape[0] == B and ik.data.shape[1] == 1
    lmax = ik.data.shape[2]
    nbmax = (lmax + MSA_BLOCK - 1) // MSA_BLOCK
    sl = _seq_lens(seq_lens)
    bs = np.empty((B, Tq, nbmax), dtype=np.float64)
    ts = np.full((B, Tq, lmax), np.nan, dtype=np.float64) if token_scores else None
    w = None if w_idx is None else np.ascontiguousarray(w_idx, dtype=np.float32)
    st = ik.struct()
    lib().orc_index(B, Tq, HI, DI, _ptr(sl), _ptr(q_idx), None if w is None else _ptr(w), ctypes.byref(st),
                    pool_mode, None if ts is None else _ptr(ts), _ptr(bs))
    return bs, ts


def select(block_scores: np.ndarray, seq_lens) -> np.ndarray:
    """int32 [B, Tq, 16]: forced recent block + best 15 others, ascending, -1 padded."""
    bs = np.ascontiguousarray(block_scores, dtype=np.float64)
    B, Tq, nbmax = bs.shape
    sl = _seq_lens(seq_lens)
    sel = np.empty((B, Tq, MSA_TOPK), dtype=np.int32)
    lib().orc_select(B, Tq, nbmax, _ptr(sl), _ptr(bs), _ptr(sel))
    return sel


def attend(q: np.ndarray, k: Nvfp4, v: Nvfp4, sel: np.ndarray, seq_lens, scale: float = 0.0):
    """Exact softmax attention over the selected visible keys.

    q fp32 [B, Tq, Hq, D]; k, v NVFP4 [B, Hkv, lmax, D/2]; sel int32 [B, Tq, 16].
    Returns (out float64 [B, Tq, Hq, D], lse float64 [B, Tq, Hq]).
    """
    q = np.ascontiguousarray(q, dtype=np.float32)
    B, Tq, Hq, D = q.shape
    Hkv = k.data.shape[1]
    assert Hq % Hkv == 0 and k.dim == D and v.dim == D
    if scale == 0.0:
        scale = 1.0 / np.sqrt(D)
    sl = _seq_lens(seq_lens)
    sel = np.ascontiguousarray(sel, dtype=np.int32)
    out = np.empty((B, Tq, Hq, D), dtype=np.float64)
    lse = np.empty((B, Tq, Hq), dtype=np.float64)
    ks, vs = k.struct(), v.struct()
    lib().orc_attend(B, Tq, Hq, Hkv, D, _ptr(sl), _ptr(q), ctypes.byref(ks), ctypes.byref(vs), _ptr(sel),
                     float(scale), _ptr(out), _ptr(lse))
    return out, lse


def decode(q, q_idx, k: Nvfp4, v: Nvfp4, ik: Nvfp4, seq_lens, w_idx=None, pool_mode=0, scale=0.0):
    """The whole MSA decode step: index -> pool -> select -> attend."""
    bs, _ = index(q_idx, ik, seq_lens, w_idx, pool_mode)
    sel = select(bs, seq_lens)
    out, lse = attend(q, k, v, sel, seq_lens, scale)
    return dict(block_scores=bs, sel=sel, out=out, lse=lse)
