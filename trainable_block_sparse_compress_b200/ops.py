"""Python binding of the InfLLM v2 C ABI: the same calls, taking torch tensors.

PyTorch provides device memory and the current CUDA stream; the binding checks shapes,
dtypes and devices, allocates outputs and workspaces with the caching allocator, and
passes raw pointers to the library.  No arithmetic of the method runs here.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

from . import _lib


@dataclass(frozen=True)
class Params:
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int = 128
    block_size: int = 64
    kernel_size: int = 32
    kernel_stride: int = 16
    topk: int = 96
    n_init: int = 1
    n_local: int = 2
    softmax_scale: float = 0.0
    score_mode: int = 0  # 0 softmax-sum, 1 logit-sum (the block score)
    pool_mode: int = 0   # 0 overlapping kernels, 1 kernels inside the block (the pooling)

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def c(self) -> _lib.CParams:
        return _lib.CParams(self.batch, self.num_q_heads, self.num_kv_heads, self.head_dim, self.block_size,
                            self.kernel_size, self.kernel_stride, self.topk, self.n_init, self.n_local,
                            float(self.softmax_scale), int(self.score_mode), int(self.pool_mode))

    @staticmethod
    def from_workload(wl, batch: Optional[int] = None) -> "Params":
        return Params(batch if batch is not None else wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim,
                      wl.block_size, wl.kernel_size, wl.kernel_stride, wl.topk, wl.n_init, wl.n_local)


def num_kernels(p: Params, n: int) -> int:
    return int(_lib.load().infllmv2_num_kernels(ctypes.byref(p.c()), n))


def num_blocks(p: Params, n: int) -> int:
    return (n + p.block_size - 1) // p.block_size


def workspace_size(p: Params, op: int, L: int) -> int:
    v = int(_lib.load().infllmv2_workspace_size(ctypes.byref(p.c()), op, L))
    if v == ctypes.c_size_t(-1).value:
        raise _lib.InfLLMv2Error("infllmv2_workspace_size", _lib.ERR_INVALID_ARG)
    return v


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device.index != torch.cuda.current_device():
        # the library launches on the current device: another device's pointer is not its memory
        raise ValueError(f"{name} is on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _workspace(p: Params, op: int, L: int, ws: Optional[torch.Tensor], device) -> Optional[torch.Tensor]:
    n = workspace_size(p, op, L)
    if n == 0:
        return ws
    if ws is None or ws.numel() * ws.element_size() < n:
        ws = torch.empty(n, dtype=torch.uint8, device=device)
    return ws


def compress_keys(p: Params, k: torch.Tensor, lens: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Semantic kernels: k bf16 [B, Hkv, Lmax, d] -> kc bf16 [B, Hkv, NK(Lmax), d]."""
    B, H, Lmax, d = k.shape
    _need(k, "k", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    if lens is not None:
        _need(lens, "lens", torch.int32, (p.batch,))
    nk = num_kernels(p, Lmax)
    if out is None:
        out = torch.empty((B, H, nk, d), dtype=torch.bfloat16, device=k.device)
    _need(out, "kc", torch.bfloat16, (B, H, nk, d))
    st = _lib.load().infllmv2_compress_keys(ctypes.byref(p.c()), _ptr(k), _ptr(lens), Lmax, _ptr(out), _stream())
    _lib.check("infllmv2_compress_keys", st)
    return out


def select_blocks_prefill(p: Params, q: torch.Tensor, kc: torch.Tensor,
                          out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """q bf16 [B, L, Hq, d], kc [B, Hkv, NK(L), d] -> block_idx int32 [B, Hkv, L, topk]."""
    B, L, Hq, d = q.shape
    _need(q, "q", torch.bfloat16, (p.batch, L, p.num_q_heads, p.head_dim))
    _need(kc, "kc", torch.bfloat16, (p.batch, p.num_kv_heads, num_kernels(p, L), p.head_dim))
    if out is None:
        out = torch.empty((B, p.num_kv_heads, L, p.topk), dtype=torch.int32, device=q.device)
    _need(out, "block_idx", torch.int32, (B, p.num_kv_heads, L, p.topk))
    st = _lib.load().infllmv2_select_blocks(ctypes.byref(p.c()), _lib.MODE_PREFILL, _ptr(q), _ptr(kc), None, L,
                                            _ptr(out), None, 0, _stream())
    _lib.check("infllmv2_select_blocks", st)
    return out


def select_blocks_chunk(p: Params, q: torch.Tensor, kc: torch.Tensor, Lmax: int,
                        q_lens: Optional[torch.Tensor] = None, kv_lens: Optional[torch.Tensor] = None,
                        out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Selection for a chunk of queries against existing caches.  q bf16 [B, Lq, Hq, d]: rows
    0..q_lens[b]-1 are the last q_lens[b] of kv_lens[b] cached tokens of sequence b (None:
    Lq and Lmax); kc [B, Hkv, NK(Lmax), d] -> block_idx int32 [B, Hkv, Lq, topk] (padding
    rows are not written)."""
    B, Lq, Hq, d = q.shape
    _need(q, "q", torch.bfloat16, (p.batch, Lq, p.num_q_heads, p.head_dim))
    _need(kc, "kc", torch.bfloat16, (p.batch, p.num_kv_heads, num_kernels(p, Lmax), p.head_dim))
    for t, name in ((q_lens, "q_lens"), (kv_lens, "kv_lens")):
        if t is not None:
            _need(t, name, torch.int32, (p.batch,))
    if out is None:
        out = torch.empty((B, p.num_kv_heads, Lq, p.topk), dtype=torch.int32, device=q.device)
    _need(out, "block_idx", torch.int32, (B, p.num_kv_heads, Lq, p.topk))
    st = _lib.load().infllmv2_select_blocks_chunk(ctypes.byref(p.c()), _ptr(q), Lq, _ptr(kc), _ptr(q_lens),
                                                  _ptr(kv_lens), Lmax, _ptr(out), None, 0, _stream())
    _lib.check("infllmv2_select_blocks_chunk", st)
    return out


def select_blocks_decode(p: Params, q: torch.Tensor, kc: torch.Tensor, lens: torch.Tensor, Lmax: int,
                         out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """q bf16 [B, Hq, d], kc [B, Hkv, NK(Lmax), d], lens int32 [B] -> int32 [B, Hkv, 1, topk]."""
    _need(q, "q", torch.bfloat16, (p.batch, p.num_q_heads, p.head_dim))
    _need(kc, "kc", torch.bfloat16, (p.batch, p.num_kv_heads, num_kernels(p, Lmax), p.head_dim))
    _need(lens, "lens", torch.int32, (p.batch,))
    if out is None:
        out = torch.empty((p.batch, p.num_kv_heads, 1, p.topk), dtype=torch.int32, device=q.device)
    _need(out, "block_idx", torch.int32, (p.batch, p.num_kv_heads, 1, p.topk))
    ws = _workspace(p, _lib.OP_SELECT_DECODE, Lmax, ws, q.device)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    st = _lib.load().infllmv2_select_blocks(ctypes.byref(p.c()), _lib.MODE_DECODE, _ptr(q), _ptr(kc), _ptr(lens),
                                            Lmax, _ptr(out), _ptr(ws), nbytes, _stream())
    _lib.check("infllmv2_select_blocks", st)
    return out


def sparse_attn_prefill(p: Params, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_idx: torch.Tensor,
                        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                        want_lse: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """O bf16 [B, L, Hq, d] and lse fp32 [B, Hq, L] over the selected blocks."""
    B, L, Hq, d = q.shape
    _need(q, "q", torch.bfloat16, (p.batch, L, p.num_q_heads, p.head_dim))
    _need(k, "k", torch.bfloat16, (p.batch, p.num_kv_heads, L, p.head_dim))
    _need(v, "v", torch.bfloat16, (p.batch, p.num_kv_heads, L, p.head_dim))
    _need(block_idx, "block_idx", torch.int32, (p.batch, p.num_kv_heads, L, p.topk))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "o", torch.bfloat16, tuple(q.shape))
    if want_lse and lse is None:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Hq, L))
    st = _lib.load().infllmv2_sparse_attn_prefill(ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(block_idx),
                                                  L, _ptr(out), _ptr(lse), None, 0, _stream())
    _lib.check("infllmv2_sparse_attn_prefill", st)
    return out, lse


def sparse_attn_chunk(p: Params, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block_idx: torch.Tensor,
                      q_lens: Optional[torch.Tensor] = None, kv_lens: Optional[torch.Tensor] = None,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                      want_lse: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Attention of a chunk of queries (as select_blocks_chunk) over caches k, v bf16
    [B, Hkv, Lmax, d]: O bf16 [B, Lq, Hq, d], lse fp32 [B, Hq, Lq] (padding rows not written)."""
    B, Lq, Hq, d = q.shape
    Lmax = k.shape[2]
    _need(q, "q", torch.bfloat16, (p.batch, Lq, p.num_q_heads, p.head_dim))
    _need(k, "k", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    _need(v, "v", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    _need(block_idx, "block_idx", torch.int32, (p.batch, p.num_kv_heads, Lq, p.topk))
    for t, name in ((q_lens, "q_lens"), (kv_lens, "kv_lens")):
        if t is not None:
            _need(t, name, torch.int32, (p.batch,))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "o", torch.bfloat16, tuple(q.shape))
    if want_lse and lse is None:
        lse = torch.empty((B, Hq, Lq), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Hq, Lq))
    st = _lib.load().infllmv2_sparse_attn_chunk(ctypes.byref(p.c()), _ptr(q), Lq, _ptr(k), _ptr(v), _ptr(q_lens),
                                                _ptr(kv_lens), Lmax, _ptr(block_idx), _ptr(out), _ptr(lse), None, 0,
                                                _stream())
    _lib.check("infllmv2_sparse_attn_chunk", st)
    return out, lse


def sparse_attn_backward(p: Params, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
                         lse: torch.Tensor, d_o: torch.Tensor, block_idx: torch.Tensor,
                         ws: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients of the prefill sparse attention with the block lists fixed: q, o, d_o bf16
    [B, L, Hq, d], k, v bf16 [B, Hkv, L, d], lse fp32 [B, Hq, L] from the forward ->
    dq [B, L, Hq, d], dk, dv [B, Hkv, L, d] (bf16)."""
    B, L, Hq, d = q.shape
    for t, name in ((q, "q"), (o, "o"), (d_o, "d_o")):
        _need(t, name, torch.bfloat16, (p.batch, L, p.num_q_heads, p.head_dim))
    for t, name in ((k, "k"), (v, "v")):
        _need(t, name, torch.bfloat16, (p.batch, p.num_kv_heads, L, p.head_dim))
    _need(lse, "lse", torch.float32, (p.batch, p.num_q_heads, L))
    _need(block_idx, "block_idx", torch.int32, (p.batch, p.num_kv_heads, L, p.topk))
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    ws = _workspace(p, _lib.OP_ATTN_BACKWARD, L, ws, q.device)
    nbytes = ws.numel() * ws.element_size()
    st = _lib.load().infllmv2_sparse_attn_backward(ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                                   _ptr(d_o), _ptr(block_idx), L, _ptr(dq), _ptr(dk), _ptr(dv),
                                                   _ptr(ws), nbytes, _stream())
    _lib.check("infllmv2_sparse_attn_backward", st)
    return dq, dk, dv


def sparse_attn_decode(p: Params, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                       lens: torch.Tensor, block_idx: torch.Tensor, out: Optional[torch.Tensor] = None,
                       lse: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                       want_lse: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """O bf16 [B, Hq, d] and lse fp32 [B, Hq] for one query per sequence at lens[b]-1."""
    Lmax = k_cache.shape[2]
    _need(q, "q", torch.bfloat16, (p.batch, p.num_q_heads, p.head_dim))
    _need(k_cache, "k_cache", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    _need(v_cache, "v_cache", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    _need(lens, "lens", torch.int32, (p.batch,))
    _need(block_idx, "block_idx", torch.int32, (p.batch, p.num_kv_heads, 1, p.topk))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "o", torch.bfloat16, tuple(q.shape))
    if want_lse and lse is None:
        lse = torch.empty((p.batch, p.num_q_heads), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (p.batch, p.num_q_heads))
    ws = _workspace(p, _lib.OP_ATTN_DECODE, Lmax, ws, q.device)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    st = _lib.load().infllmv2_sparse_attn_decode(ctypes.byref(p.c()), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                                 _ptr(lens), Lmax, _ptr(block_idx), _ptr(out), _ptr(lse),
                                                 _ptr(ws), nbytes, _stream())
    _lib.check("infllmv2_sparse_attn_decode", st)
    return out, lse


def sparse_attn_decode_noalloc(p: Params, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                               lens: torch.Tensor, block_idx: torch.Tensor, out: torch.Tensor,
                               lse: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Decode attention for callers that cannot allocate device memory at call time: the
    caller passes preallocated outputs and the library uses its own fixed scratch array
    (no workspace).  Calls that overlap on the GPU race on that array."""
    Lmax = k_cache.shape[2]
    _need(q, "q", torch.bfloat16, (p.batch, p.num_q_heads, p.head_dim))
    _need(k_cache, "k_cache", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    _need(v_cache, "v_cache", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    _need(lens, "lens", torch.int32, (p.batch,))
    _need(block_idx, "block_idx", torch.int32, (p.batch, p.num_kv_heads, 1, p.topk))
    _need(out, "o", torch.bfloat16, tuple(q.shape))
    if lse is not None:
        _need(lse, "lse", torch.float32, (p.batch, p.num_q_heads))
    st = _lib.load().infllmv2_sparse_attn_decode_noalloc(ctypes.byref(p.c()), _ptr(q), _ptr(k_cache),
                                                         _ptr(v_cache), _ptr(lens), Lmax, _ptr(block_idx),
                                                         _ptr(out), _ptr(lse), _stream())
    _lib.check("infllmv2_sparse_attn_decode_noalloc", st)
    return out, lse


def append_kv(p: Params, k_new: torch.Tensor, v_new: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
              lens: torch.Tensor, kc: torch.Tensor) -> None:
    """Appends one token per sequence: k_new / v_new bf16 [B, Hkv, d] go to position lens[b]
    of the caches [B, Hkv, Lmax, d], a completed semantic kernel goes to kc
    [B, Hkv, NK(Lmax), d], and lens (int32 [B], on the GPU) is incremented in place."""
    Lmax = k_cache.shape[2]
    _need(k_new, "k_new", torch.bfloat16, (p.batch, p.num_kv_heads, p.head_dim))
    _need(v_new, "v_new", torch.bfloat16, (p.batch, p.num_kv_heads, p.head_dim))
    _need(k_cache, "k_cache", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    _need(v_cache, "v_cache", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    _need(lens, "lens", torch.int32, (p.batch,))
    _need(kc, "kc", torch.bfloat16, (p.batch, p.num_kv_heads, num_kernels(p, Lmax), p.head_dim))
    st = _lib.load().infllmv2_append_kv(ctypes.byref(p.c()), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                        _ptr(lens), Lmax, _ptr(kc), _stream())
    _lib.check("infllmv2_append_kv", st)


def device_error(clear: bool = True) -> int:
    v = int(_lib.load().infllmv2_device_error(1 if clear else 0))
    if v < 0:
        raise _lib.InfLLMv2Error("infllmv2_device_error", v)
    return v


def prefill(p: Params, q, k, v):
    """Whole prefill path: compress -> select -> sparse attention.  Returns (o, lse, idx, kc)."""
    kc = compress_keys(p, k)
    idx = select_blocks_prefill(p, q, kc)
    o, lse = sparse_attn_prefill(p, q, k, v, idx)
    return o, lse, idx, kc


def prefill_chunk(p: Params, q, k_cache, v_cache, kc, q_lens=None, kv_lens=None):
    """A chunk of queries against filled caches (keys, values and semantic kernels of
    kv_lens[b] tokens each): select -> sparse attention.  Returns (o, lse, idx)."""
    Lmax = k_cache.shape[2]
    idx = select_blocks_chunk(p, q, kc, Lmax, q_lens=q_lens, kv_lens=kv_lens)
    o, lse = sparse_attn_chunk(p, q, k_cache, v_cache, idx, q_lens=q_lens, kv_lens=kv_lens)
    return o, lse, idx


def decode_step(p: Params, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, kc: torch.Tensor,
                lens: torch.Tensor, k_new: Optional[torch.Tensor] = None, v_new: Optional[torch.Tensor] = None,
                lens_out: Optional[torch.Tensor] = None, block_idx: Optional[torch.Tensor] = None,
                out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None, want_lse: bool = True):
    """One decode step in one launch.  With k_new / v_new [B, Hkv, d]: the new token is
    appended at lens[b] (caches and kc updated in place) and lens_out[b] = lens[b] + 1
    (lens_out allocated when None); without: the query sits at lens[b]-1.  Then block
    selection and sparse attention over the selected blocks.  Returns (o, lse, block_idx)
    and, when appending, lens_out as a fourth element."""
    Lmax = k_cache.shape[2]
    _need(q, "q", torch.bfloat16, (p.batch, p.num_q_heads, p.head_dim))
    _need(k_cache, "k_cache", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    _need(v_cache, "v_cache", torch.bfloat16, (p.batch, p.num_kv_heads, Lmax, p.head_dim))
    _need(kc, "kc", torch.bfloat16, (p.batch, p.num_kv_heads, num_kernels(p, Lmax), p.head_dim))
    _need(lens, "lens", torch.int32, (p.batch,))
    appending = k_new is not None or v_new is not None
    if appending:
        _need(k_new, "k_new", torch.bfloat16, (p.batch, p.num_kv_heads, p.head_dim))
        _need(v_new, "v_new", torch.bfloat16, (p.batch, p.num_kv_heads, p.head_dim))
        if lens_out is None:
            lens_out = torch.empty_like(lens)
        _need(lens_out, "lens_out", torch.int32, (p.batch,))
        if lens_out.data_ptr() == lens.data_ptr():
            raise ValueError("lens_out must not be lens")
    if block_idx is None:
        block_idx = torch.empty((p.batch, p.num_kv_heads, 1, p.topk), dtype=torch.int32, device=q.device)
    _need(block_idx, "block_idx", torch.int32, (p.batch, p.num_kv_heads, 1, p.topk))
    if out is None:
        out = torch.empty_like(q)
    _need(out, "o", torch.bfloat16, tuple(q.shape))
    if want_lse and lse is None:
        lse = torch.empty((p.batch, p.num_q_heads), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (p.batch, p.num_q_heads))
    st = _lib.load().infllmv2_decode_step(ctypes.byref(p.c()), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                          _ptr(v_cache), _ptr(kc), _ptr(lens), _ptr(lens_out), Lmax, _ptr(block_idx),
                                          _ptr(out), _ptr(lse), _stream())
    _lib.check("infllmv2_decode_step", st)
    if appending:
        return out, lse, block_idx, lens_out
    return out, lse, block_idx


def decode(p: Params, q, k_cache, v_cache, kc, lens, Lmax):
    """One decode step over a filled cache (Lmax = the caches' length): select -> sparse
    attention, fused in one launch.  Returns (o, lse, idx)."""
    assert k_cache.shape[2] == Lmax, "Lmax is the caches' length"
    return decode_step(p, q, k_cache, v_cache, kc, lens)
