"""The no-allocation decode entry point (collected last on purpose).

Some callers cannot allocate device memory when they run attention -- an engine plugin
whose execute step must not allocate, or a service that reserves its memory budget at
start-up.  infllmv2_sparse_attn_decode_noalloc serves them from a fixed scratch array
inside the library.  These tests call it through the C ABI and check that it gives the
same result as the workspace-taking entry point, on two calls in a row (the second call
reuses the scratch the first one left behind)."""
import ctypes

import numpy as np
import pytest
import torch

from parity import O_MAX_ABS, O_MEAN_ABS
from trainable_block_sparse_compress_b200 import _lib, build, ops
from trainable_block_sparse_compress_b200.synthetic import Workload, make_inputs


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_entry_point():
    assert torch.cuda.is_available(), "GPU test"
    build.build()
    lib = _lib.load()
    wl = Workload("noalloc", "decode", 12, 20000, 32, 2, 96)
    x = make_inputs(wl, seed=11)
    x.lens = torch.tensor([20000, 1, 64, 65, 3001, 12345, 19999, 31, 640, 7000, 16384, 9999], dtype=torch.int32)
    p = ops.Params.from_workload(wl)
    assert ops.workspace_size(p, _lib.OP_ATTN_DECODE, wl.seq_len) <= _lib.NOALLOC_SCRATCH_BYTES
    q, k, v, lens = x.q.cuda(), x.k.cuda(), x.v.cuda(), x.lens.cuda()
    kc = ops.compress_keys(p, k, lens=lens)
    idx = ops.select_blocks_decode(p, q, kc, lens, wl.seq_len)
    o_ref, lse_ref = ops.sparse_attn_decode(p, q, k, v, lens, idx)
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
    assert ops.device_error(clear=True) == 0


@pytest.mark.gpu
def test_noalloc_decode_rejects_problems_beyond_its_scratch():
    build.build()
    lib = _lib.load()
    p = ops.Params(batch=1024, num_q_heads=32, num_kv_heads=2, topk=96)
    need = ops.workspace_size(p, _lib.OP_ATTN_DECODE, 4096)
    assert need > _lib.NOALLOC_SCRATCH_BYTES
    fake = 4096  # never dereferenced: the size check comes first
    st = lib.infllmv2_sparse_attn_decode_noalloc(ctypes.byref(p.c()), fake, fake, fake, fake, 4096, fake, fake,
                                                 None, None)
    assert st == _lib.ERR_WORKSPACE
