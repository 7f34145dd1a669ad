"""CPU oracle for InfLLM v2 block-sparse attention -- test infrastructure only.

The arithmetic lives in ``infllmv2_oracle.c`` (plain C, double precision, OpenMP over
independent rows); this module only compiles it and marshals numpy arrays.  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may use it.
It shares nothing with the CUDA library, and the CUDA library never calls it.

bf16 tensors are passed as ``uint16`` bit patterns (``tensor.view(torch.int16)``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "infllmv2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_infllmv2.so")
_lib = None


class _Params(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("kernel_size", ctypes.c_int32),
        ("kernel_stride", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("n_init", ctypes.c_int32),
        ("n_local", ctypes.c_int32),
        ("softmax_scale", ctypes.c_double),
        ("score_mode", ctypes.c_int32),
        ("pool_mode", ctypes.c_int32),
    ]


@dataclass
class Params:
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int = 128
    block_size: int = 64
    kernel_size: int = 32
    kernel_stride: int = 16
    topk: int = 16
    n_init: int = 1
    n_local: int = 2
    softmax_scale: float = 0.0
    score_mode: int = 0  # 0 softmax-sum, 1 logit-sum
    pool_mode: int = 0   # 0 overlapping kernels, 1 kernels inside the block

    def _c(self) -> _Params:
        return _Params(self.batch, self.num_q_heads, self.num_kv_heads, self.head_dim,
                       self.block_size, self.kernel_size, self.kernel_stride, self.topk,
                       self.n_init, self.n_local, float(self.softmax_scale), int(self.score_mode),
                       int(self.pool_mode))


def build(force: bool = False) -> str:
    """Compile the oracle into a shared library next to its source."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC",
                               "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER(_Params)
        vp = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.oracle_bf16_round.argtypes = [vp, vp, i64]
        lib.oracle_num_kernels.argtypes = [P, i64]
        lib.oracle_num_kernels.restype = i64
        lib.oracle_num_blocks.argtypes = [P, i64]
        lib.oracle_num_blocks.restype = i64
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_compress.argtypes = [P, vp, vp, i64, vp]
        lib.oracle_select.argtypes = [P, vp, i64, vp, i64, vp, i64, vp, i64, vp, vp, i64]
        lib.oracle_select.restype = ctypes.c_int
        lib.oracle_attn.argtypes = [P, vp, i64, vp, vp, vp, i64, vp, vp, i64, vp, vp]
        lib.oracle_attn.restype = i64
        lib.oracle_attn_backward.argtypes = [P, vp, i64, vp, vp, vp, i64, vp, vp, vp, vp, vp, vp]
        lib.oracle_attn_backward.restype = i64
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16, a.dtype
    return a


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def num_kernels(p: Params, n: int) -> int:
    return int(_load().oracle_num_kernels(ctypes.byref(p._c()), n))


def num_blocks(p: Params, n: int) -> int:
    return int(_load().oracle_num_blocks(ctypes.byref(p._c()), n))


def bf16_round(x) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even); returns uint16 patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_bf16_round(_ptr(x), _ptr(out), x.size)
    return out


def compress(p: Params, k, lens=None) -> np.ndarray:
    """Semantic kernels: k [B,Hkv,Lmax,d] bf16 -> kc [B,Hkv,NK(Lmax),d] bf16 (uint16)."""
    k = _u16(k)
    B, H, Lmax, d = k.shape
    nk = num_kernels(p, Lmax)
    kc = np.zeros((B, H, nk, d), dtype=np.uint16)
    lens_a = None if lens is None else np.ascontiguousarray(lens, dtype=np.int32)
    _load().oracle_compress(ctypes.byref(p._c()), _ptr(k), _ptr(lens_a), Lmax, _ptr(kc))
    return kc


def _rows(rows, Lq):
    if rows is None:
        rows = np.arange(Lq, dtype=np.int64)
    return np.ascontiguousarray(rows, dtype=np.int64)


def select(p: Params, q, kc, lens=None, Lmax=None, rows=None, want_scores=False):
    """Block selection.  q [B,Lq,Hq,d], kc [B,Hkv,NK,d] (bf16 as uint16).

    Queries are the last Lq tokens of each sequence (lens[b] tokens, or Lmax when lens is
    None).  Returns idx [B,Hkv,R,topk] int32 and, if asked, scores [B,Hkv,R,nblk] float64
    (-inf marks an ineligible block)."""
    q = _u16(q)
    kc = _u16(kc)
    B, Lq, Hq, d = q.shape
    nkmax = kc.shape[2]
    if Lmax is None:
        Lmax = Lq if lens is None else int(np.max(lens))
    rows = _rows(rows, Lq)
    lens_a = None if lens is None else np.ascontiguousarray(lens, dtype=np.int32)
    H = p.num_kv_heads
    idx = np.empty((B, H, len(rows), p.topk), dtype=np.int32)
    nblk = num_blocks(p, Lmax)
    scores = np.empty((B, H, len(rows), nblk), dtype=np.float64) if want_scores else None
    rc = _load().oracle_select(ctypes.byref(p._c()), _ptr(q), Lq, _ptr(kc), nkmax, _ptr(lens_a),
                               Lmax, _ptr(rows), len(rows), _ptr(idx), _ptr(scores), nblk)
    if rc != 0:
        raise ValueError("oracle_select: a query position lies outside its sequence")
    return (idx, scores) if want_scores else idx


def attn(p: Params, q, k, v, idx, lens=None, rows=None):
    """Sparse attention.  q [B,Lq,Hq,d]; k, v [B,Hkv,Lmax,d]; idx [B,Hkv,R,topk] for the
    evaluated rows.  Returns o [B,R,Hq,d] float64 and lse [B,Hq,R] float64."""
    q = _u16(q)
    k = _u16(k)
    v = _u16(v)
    B, Lq, Hq, d = q.shape
    Lmax = k.shape[2]
    rows = _rows(rows, Lq)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    assert idx.shape == (B, p.num_kv_heads, len(rows), p.topk), idx.shape
    lens_a = None if lens is None else np.ascontiguousarray(lens, dtype=np.int32)
    o = np.empty((B, len(rows), Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq, len(rows)), dtype=np.float64)
    rc = _load().oracle_attn(ctypes.byref(p._c()), _ptr(q), Lq, _ptr(k), _ptr(v), _ptr(lens_a),
                             Lmax, _ptr(idx), _ptr(rows), len(rows), _ptr(o), _ptr(lse))
    if rc < 0:
        raise ValueError("oracle_attn: a query position lies outside its sequence")
    if rc > 0:
        raise ValueError(f"oracle_attn: {rc} selected block indices lie outside [0, t/block]")
    return o, lse


def attn_backward(p: Params, q, k, v, idx, d_o, lens=None, o=None):
    """Gradients of the sparse attention (block lists fixed).  q, d_o [B,Lq,Hq,d]; k, v
    [B,Hkv,Lmax,d] (bf16 as uint16); idx [B,Hkv,Lq,topk] for every query row; o: the
    forward output [B,Lq,Hq,d] (float64) when the backward takes it as an input, else
    None (exact).  Returns dq [B,Lq,Hq,d], dk and dv [B,Hkv,Lmax,d] as float64."""
    q = _u16(q)
    k = _u16(k)
    v = _u16(v)
    d_o = _u16(d_o)
    B, Lq, Hq, d = q.shape
    Lmax = k.shape[2]
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    assert idx.shape == (B, p.num_kv_heads, Lq, p.topk), idx.shape
    assert d_o.shape == q.shape
    lens_a = None if lens is None else np.ascontiguousarray(lens, dtype=np.int32)
    o_a = None if o is None else np.ascontiguousarray(o, dtype=np.float64)
    if o_a is not None:
        assert o_a.shape == q.shape, o_a.shape
    dq = np.empty((B, Lq, Hq, d), dtype=np.float64)
    dk = np.empty(k.shape, dtype=np.float64)
    dv = np.empty(v.shape, dtype=np.float64)
    rc = _load().oracle_attn_backward(ctypes.byref(p._c()), _ptr(q), Lq, _ptr(k), _ptr(v), _ptr(lens_a), Lmax,
                                      _ptr(idx), _ptr(d_o), _ptr(o_a), _ptr(dq), _ptr(dk), _ptr(dv))
    if rc < 0:
        raise ValueError("oracle_attn_backward: a query position lies outside its sequence")
    if rc > 0:
        raise ValueError(f"oracle_attn_backward: {rc} selected block indices lie outside [0, t/block]")
    return dq, dk, dv
