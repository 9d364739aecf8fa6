"""Thin ctypes binding of libmsa.so (include/msa.h): argument marshalling only.

Every function here has the name of the C entry point it calls and does no
arithmetic of the method: it turns torch tensors into device pointers, builds
the ``msa_params_t`` struct, passes the current CUDA stream, and raises
:class:`MsaError` on a non-zero status.  There is no fallback: if libmsa.so is
missing or cannot be loaded, importing the library fails loudly.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmsa.so")

MSA_BLOCK_TOKENS = 128
MSA_TOPK_BLOCKS = 16
MSA_STATUS_SEQLEN = 1
MSA_STATUS_SELECT = 2
MSA_STATUS_TIMEOUT = 4

# names exported by the C ABI (include/msa.h)
EXPORTS = ("msa_status_string", "msa_version", "msa_nvfp4_encode", "msa_nvfp4_decode", "msa_nvfp4_amax",
           "msa_workspace_size", "msa_index", "msa_select", "msa_attend", "msa_decode", "msa_decode_static",
           "msa_workspace_size_single_launch", "msa_decode_single_launch", "msa_dcp_workspace_size",
           "msa_dcp_candidates", "msa_dcp_merge", "msa_dcp_attend", "msa_dcp_combine")
MSA_STATIC_SCRATCH_BYTES = 4 << 20


class MsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (code {code})")


class _Cache(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("tensor_scale", ctypes.c_float)]


class _Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Tq", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("D", ctypes.c_int), ("HI", ctypes.c_int), ("DI", ctypes.c_int), ("lmax", ctypes.c_int64),
                ("seq_lens", ctypes.c_void_p), ("k", _Cache), ("v", _Cache), ("ik", _Cache),
                ("q", ctypes.c_void_p), ("q_idx", ctypes.c_void_p), ("w_idx", ctypes.c_void_p),
                ("softmax_scale", ctypes.c_float), ("pool_mode", ctypes.c_int), ("status", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("num_pages", ctypes.c_int64), ("out_bf16", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmsa.so (built in-tree by ``block_sparse_attention_10_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmsa.so not found at {LIB_PATH}: build it with "
                              f"`python -m block_sparse_attention_10_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        L.msa_status_string.restype = ctypes.c_char_p
        L.msa_status_string.argtypes = [i32]
        L.msa_version.restype = ctypes.c_char_p
        L.msa_nvfp4_encode.argtypes = [vp, i64, i32, f32, vp, vp, vp]
        L.msa_nvfp4_decode.argtypes = [vp, vp, i64, i32, f32, vp, vp]
        L.msa_nvfp4_amax.argtypes = [vp, i64, vp, vp]
        P = ctypes.POINTER(_Params)
        L.msa_workspace_size.restype = ctypes.c_size_t
        L.msa_workspace_size.argtypes = [P]
        L.msa_index.argtypes = [P, vp, vp, vp]
        L.msa_select.argtypes = [P, vp, vp, vp]
        L.msa_attend.argtypes = [P, vp, vp, vp, vp]
        L.msa_decode.argtypes = [P, vp, ctypes.c_size_t, vp, vp, vp, vp]
        L.msa_workspace_size_single_launch.restype = ctypes.c_size_t
        L.msa_workspace_size_single_launch.argtypes = [P]
        L.msa_decode_single_launch.argtypes = [P, vp, ctypes.c_size_t, vp, vp, vp, vp]
        L.msa_decode_static.argtypes = [P, vp, vp, vp, vp]
        L.msa_dcp_workspace_size.restype = ctypes.c_size_t
        L.msa_dcp_workspace_size.argtypes = [P]
        L.msa_dcp_candidates.argtypes = [P, i64, i64, vp, ctypes.c_size_t, vp, vp, vp]
        L.msa_dcp_merge.argtypes = [P, i32, vp, vp, vp, vp]
        L.msa_dcp_attend.argtypes = [P, i64, i64, vp, vp, vp, vp]
        L.msa_dcp_combine.argtypes = [P, i32, vp, vp, vp, vp, vp]
        for name in (n for n in EXPORTS
                     if n not in ("msa_status_string", "msa_version", "msa_workspace_size",
                                  "msa_workspace_size_single_launch", "msa_dcp_workspace_size")):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().msa_status_string(code).decode()


def _check(code: int, where: str):
    if code != 0:
        raise MsaError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass(frozen=True)
class Nvfp4Cache:
    """An NVFP4 cache tensor: data uint8 [B, H, lmax, dim/2], scale uint8 [B, H, lmax, dim/16], fp32 scale.
    Immutable (a new cache is a new object), so a problem's cached parameter block stays valid."""
    data: torch.Tensor
    scale: torch.Tensor
    tensor_scale: float

    @staticmethod
    def empty(B: int, H: int, lmax: int, dim: int, tensor_scale: float, device="cuda") -> "Nvfp4Cache":
        return Nvfp4Cache(torch.zeros(B, H, lmax, dim // 2, dtype=torch.uint8, device=device),
                          torch.zeros(B, H, lmax, dim // 16, dtype=torch.uint8, device=device), tensor_scale)

    def _c(self) -> _Cache:
        return _Cache(self.data.data_ptr(), self.scale.data_ptr(), self.tensor_scale)


@dataclass
class MsaProblem:
    """Python view of ``msa_params_t``; tensors must live on the current CUDA device."""
    seq_lens: torch.Tensor          # int32 [B]
    k: Nvfp4Cache
    v: Nvfp4Cache
    ik: Nvfp4Cache
    q: torch.Tensor                 # bf16 [B, Tq, Hq, D]
    q_idx: torch.Tensor             # bf16 [B, Tq, HI, DI]
    w_idx: Optional[torch.Tensor] = None  # fp32 [B, Tq, HI]
    softmax_scale: float = 0.0
    pool_mode: int = 0
    status: Optional[torch.Tensor] = None  # int32/uint32 [1]
    # paged caches: int32 [B, lmax / 128] page of each block; k, v, ik are then page pools
    # [num_pages, H, 128, dim/2] (+ scales)
    block_table: Optional[torch.Tensor] = None
    out_bf16: bool = False  # attention output as bf16 instead of fp32

    def __setattr__(self, name, value):
        # any change of a field invalidates the cached parameter block
        object.__setattr__(self, name, value)
        if name != "_prm":
            object.__setattr__(self, "_prm", None)

    def params(self) -> _Params:
        """The ``msa_params_t`` of this problem, built once and reused while no field is
        reassigned (tensors changed in place keep their addresses)."""
        prm = getattr(self, "_prm", None)
        if prm is None:
            prm = self._build_params()
            object.__setattr__(self, "_prm", prm)
        return prm

    def _build_params(self) -> _Params:
        B, Tq, Hq, D = self.q.shape
        HI, DI = self.q_idx.shape[2], self.q_idx.shape[3]
        Hkv = self.k.data.shape[1]
        paged = self.block_table is not None
        return _Params(B, Tq, Hq, Hkv, D, HI, DI, self.nbmax * MSA_BLOCK_TOKENS, self.seq_lens.data_ptr(),
                       self.k._c(), self.v._c(), self.ik._c(), self.q.data_ptr(), self.q_idx.data_ptr(),
                       None if self.w_idx is None else self.w_idx.data_ptr(), self.softmax_scale, self.pool_mode,
                       None if self.status is None else self.status.data_ptr(),
                       self.block_table.data_ptr() if paged else None, self.ik.data.shape[0] if paged else 0,
                       1 if self.out_bf16 else 0)

    @property
    def nbmax(self) -> int:
        """Blocks per sequence: the cache capacity (contiguous) or the block-table width (paged)."""
        if self.block_table is not None:
            return self.block_table.shape[1]
        return self.ik.data.shape[2] // MSA_BLOCK_TOKENS


# --------------------------------------------------------------------------- codec

def msa_nvfp4_encode(x: torch.Tensor, tensor_scale: float, data: torch.Tensor, scale: torch.Tensor, stream=None):
    dim = x.shape[-1]
    _check(lib().msa_nvfp4_encode(_ptr(x), x.numel() // dim, dim, tensor_scale, _ptr(data), _ptr(scale),
                                  _stream(stream)), "msa_nvfp4_encode")


def msa_nvfp4_decode(data: torch.Tensor, scale: torch.Tensor, tensor_scale: float, out: torch.Tensor, stream=None):
    dim = out.shape[-1]
    _check(lib().msa_nvfp4_decode(_ptr(data), _ptr(scale), out.numel() // dim, dim, tensor_scale, _ptr(out),
                                  _stream(stream)), "msa_nvfp4_decode")


def msa_nvfp4_amax(x: torch.Tensor, out: torch.Tensor, stream=None):
    _check(lib().msa_nvfp4_amax(_ptr(x), x.numel(), _ptr(out), _stream(stream)), "msa_nvfp4_amax")


def encode_cache(x: torch.Tensor, tensor_scale: float, stream=None) -> Nvfp4Cache:
    """Allocate NVFP4 planes for fp32 x [..., dim] (on x's device) and fill them with msa_nvfp4_encode."""
    dim = x.shape[-1]
    data = torch.empty(*x.shape[:-1], dim // 2, dtype=torch.uint8, device=x.device)
    scale = torch.empty(*x.shape[:-1], dim // 16, dtype=torch.uint8, device=x.device)
    msa_nvfp4_encode(x.contiguous(), tensor_scale, data, scale, stream)
    return Nvfp4Cache(data, scale, tensor_scale)


# --------------------------------------------------------------------------- MSA steps

def msa_workspace_size(p: MsaProblem) -> int:
    prm = p.params()
    return int(lib().msa_workspace_size(ctypes.byref(prm)))


def msa_index(p: MsaProblem, block_scores: torch.Tensor, token_scores: Optional[torch.Tensor] = None, stream=None):
    prm = p.params()
    _check(lib().msa_index(ctypes.byref(prm), _ptr(block_scores), _ptr(token_scores), _stream(stream)), "msa_index")


def msa_select(p: MsaProblem, block_scores: torch.Tensor, sel: torch.Tensor, stream=None):
    prm = p.params()
    _check(lib().msa_select(ctypes.byref(prm), _ptr(block_scores), _ptr(sel), _stream(stream)), "msa_select")


def msa_attend(p: MsaProblem, sel: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
               stream=None):
    prm = p.params()
    _check(lib().msa_attend(ctypes.byref(prm), _ptr(sel), _ptr(out), _ptr(lse), _stream(stream)), "msa_attend")


def msa_decode(p: MsaProblem, ws: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
               sel_out: Optional[torch.Tensor] = None, stream=None):
    prm = p.params()
    _check(lib().msa_decode(ctypes.byref(prm), _ptr(ws), ws.numel() * ws.element_size(), _ptr(out), _ptr(lse),
                            _ptr(sel_out), _stream(stream)), "msa_decode")


def msa_workspace_size_single_launch(p: MsaProblem) -> int:
    prm = p.params()
    return int(lib().msa_workspace_size_single_launch(ctypes.byref(prm)))


def msa_decode_single_launch(p: MsaProblem, ws: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                             sel_out: Optional[torch.Tensor] = None, stream=None):
    """The decode step as one persistent launch (same results as msa_decode; see msa.h)."""
    prm = p.params()
    _check(lib().msa_decode_single_launch(ctypes.byref(prm), _ptr(ws), ws.numel() * ws.element_size(), _ptr(out),
                                          _ptr(lse), _ptr(sel_out), _stream(stream)), "msa_decode_single_launch")


def alloc_workspace_single_launch(p: MsaProblem) -> torch.Tensor:
    n = msa_workspace_size_single_launch(p)
    if n == 0:
        raise MsaError(2, "msa_workspace_size_single_launch")
    return torch.empty(n, dtype=torch.uint8, device=p.q.device)


def msa_decode_static(p: MsaProblem, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                      sel_out: Optional[torch.Tensor] = None, stream=None):
    """msa_decode with the library's own static device scratch (no allocation anywhere).

    For callers that cannot allocate device memory; calls that overlap on the GPU race
    (they share one scratch array), and the first call on a device should precede any
    stream capture."""
    prm = p.params()
    _check(lib().msa_decode_static(ctypes.byref(prm), _ptr(out), _ptr(lse), _ptr(sel_out), _stream(stream)),
           "msa_decode_static")


def alloc_workspace(p: MsaProblem) -> torch.Tensor:
    n = msa_workspace_size(p)
    if n == 0:
        raise MsaError(1, "msa_workspace_size")
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(n, dtype=torch.uint8, device=p.q.device)


def outputs(p: MsaProblem):
    """(out [B, Tq, Hq, D] fp32 or bf16 per p.out_bf16, lse fp32 [B, Tq, Hq], sel int32 [B, Tq, 16])."""
    B, Tq, Hq, D = p.q.shape
    dev = p.q.device
    return (torch.empty(B, Tq, Hq, D, dtype=torch.bfloat16 if p.out_bf16 else torch.float32, device=dev),
            torch.empty(B, Tq, Hq, dtype=torch.float32, device=dev),
            torch.empty(B, Tq, MSA_TOPK_BLOCKS, dtype=torch.int32, device=dev))


# --------------------------------------------------------------------------- context-parallel decode

def msa_dcp_workspace_size(p: MsaProblem) -> int:
    prm = p.params()
    return int(lib().msa_dcp_workspace_size(ctypes.byref(prm)))


def msa_dcp_candidates(p: MsaProblem, n0: int, n1: int, ws: torch.Tensor, cand_score: torch.Tensor,
                       cand_id: torch.Tensor, stream=None):
    """This rank's candidates from blocks [n0, n1): fp32 / int32 [B, Tq, 16] (see msa.h)."""
    prm = p.params()
    _check(lib().msa_dcp_candidates(ctypes.byref(prm), n0, n1, _ptr(ws), ws.numel() * ws.element_size(),
                                    _ptr(cand_score), _ptr(cand_id), _stream(stream)), "msa_dcp_candidates")


def msa_dcp_merge(p: MsaProblem, cand_score: torch.Tensor, cand_id: torch.Tensor, sel: torch.Tensor, stream=None):
    """Merge of the G ranks' candidates [G, B, Tq, 16] into the selection [B, Tq, 16]."""
    prm = p.params()
    _check(lib().msa_dcp_merge(ctypes.byref(prm), cand_score.shape[0], _ptr(cand_score), _ptr(cand_id), _ptr(sel),
                               _stream(stream)), "msa_dcp_merge")


def msa_dcp_attend(p: MsaProblem, n0: int, n1: int, sel: torch.Tensor, part_out: torch.Tensor,
                   part_lse: torch.Tensor, stream=None):
    """Attention over the selected blocks in [n0, n1): fp32 partial out [B, Tq, Hq, D] and lse [B, Tq, Hq]."""
    prm = p.params()
    _check(lib().msa_dcp_attend(ctypes.byref(prm), n0, n1, _ptr(sel), _ptr(part_out), _ptr(part_lse),
                                _stream(stream)), "msa_dcp_attend")


def msa_dcp_combine(p: MsaProblem, part_out: torch.Tensor, part_lse: torch.Tensor, out: torch.Tensor,
                    lse: Optional[torch.Tensor] = None, stream=None):
    """Combine of G partials [G, B, Tq, Hq, D] / [G, B, Tq, Hq] into out (fp32 or bf16) and lse."""
    prm = p.params()
    _check(lib().msa_dcp_combine(ctypes.byref(prm), part_out.shape[0], _ptr(part_out), _ptr(part_lse), _ptr(out),
                                 _ptr(lse), _stream(stream)), "msa_dcp_combine")
