"""The no-allocation decode entry point (collected last on purpose).

Some callers cannot allocate device memory when they run attention -- an engine plugin
whose execute step must not allocate, or a service that reserves its memory budget at
start-up.  infllmv2_sparse_attn_decode_noalloc serves them from a fixed scratch array
inside the library.  These tests call it through the C ABI and check that it gives the
same result as the workspace-taking entry point and as the CPU oracle's exact attention
over the same block lists, on two calls in a row (the second call reuses the scratch the
first one left behind)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity import O_MAX_ABS, O_MEAN_ABS, compare_attention
from trainable_block_sparse_compress_b200 import _lib, build, ops
from trainable_block_sparse_compress_b200.synthetic import Workload, as_u16, make_inputs


def _check_noalloc_against_entry_point(wl, lens, seed):
    build.build()
    lib = _lib.load()
    x = make_inputs(wl, seed=seed)
    x.lens = torch.tensor(lens, dtype=torch.int32)
    p = ops.Params.from_workload(wl)
    assert ops.workspace_size(p, _lib.OP_ATTN_DECODE, wl.seq_len) <= _lib.NOALLOC_SCRATCH_BYTES
    q, k, v, lens = x.q.cuda(), x.k.cuda(), x.v.cuda(), x.lens.cuda()
    kc = ops.compress_keys(p, k, lens=lens)
    idx = ops.select_blocks_decode(p, q, kc, lens, wl.seq_len)
    o_ref, lse_ref = ops.sparse_attn_decode(p, q, k, v, lens, idx)
    op = oracle.Params(p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim, p.block_size, p.kernel_size,
                       p.kernel_stride, p.topk, p.n_init, p.n_local, p.softmax_scale)
    o_ora, lse_ora = oracle.attn(op, as_u16(x.q)[:, None], as_u16(x.k), as_u16(x.v), idx.cpu().numpy(),
                                 lens=np.array(lens.cpu().numpy(), np.int32))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        o = torch.full_like(q, float("nan"))
        lse = torch.full((p.batch, p.num_q_heads), float("nan"), device=q.device)
        st = lib.infllmv2_sparse_attn_decode_noalloc(ctypes.byref(p.c()), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                     lens.data_ptr(), wl.seq_len, idx.data_ptr(), o.data_ptr(),
                                                     lse.data_ptr(), stream)
        assert st == _lib.OK, lib.infllmv2_status_string(st)
        torch.cuda.synchronize()
        diff = (o.float() - o_ref.float()).abs()
        assert torch.isfinite(o).all() and torch.isfinite(lse).all()
        assert float(diff.max()) <= O_MAX_ABS and float(diff.mean()) <= O_MEAN_ABS, call
        assert float((lse - lse_ref).abs().max()) <= 1e-3, call
        compare_attention(o.float().cpu().numpy(), o_ora[:, 0], lse.cpu().numpy(), lse_ora[:, :, 0])
    assert ops.device_error(clear=True) == 0


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_entry_point():
    # 24 (sequence, kv-head) items: one thread-block cluster each, no scratch needed
    assert torch.cuda.is_available(), "GPU test"
    wl = Workload("noalloc", "decode", 12, 20000, 32, 2, 96)
    _check_noalloc_against_entry_point(
        wl, [20000, 1, 64, 65, 3001, 12345, 19999, 31, 640, 7000, 16384, 9999], seed=11)


@pytest.mark.gpu
def test_noalloc_decode_small_batch_uses_the_scratch():
    # 2 items: split finer than a cluster, partials merged through the fixed scratch
    assert torch.cuda.is_available(), "GPU test"
    wl = Workload("noalloc_b1", "decode", 1, 20000, 32, 2, 96)
    p = ops.Params.from_workload(wl)
    assert ops.workspace_size(p, _lib.OP_ATTN_DECODE, wl.seq_len) > 0
    _check_noalloc_against_entry_point(wl, [19999], seed=12)


def test_noalloc_scratch_covers_every_split_configuration():
    # The split path serves fewer (sequence, kv-head) items than SMs / 16 with at most
    # two blocks per split; its partials must fit the library's fixed scratch array for
    # every head count and top-k, so the no-allocation entry point never refuses a valid
    # call.  Host-only: infllmv2_workspace_size launches nothing.
    worst = 0
    for hkv in (1, 2, 4, 8):
        for batch in range(1, 17):
            for topk in (3, 16, 96, 255, 256):
                p = ops.Params(batch=batch, num_q_heads=16 * hkv, num_kv_heads=hkv, topk=topk)
                worst = max(worst, ops.workspace_size(p, _lib.OP_ATTN_DECODE, 131072))
    assert 0 < worst <= _lib.NOALLOC_SCRATCH_BYTES
