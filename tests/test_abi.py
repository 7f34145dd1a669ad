"""Host-side checks of the C ABI: the library loads, exports every declared symbol,
and rejects bad arguments before touching the GPU (no kernel is launched here)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from trainable_block_sparse_compress_b200 import _lib, build
from trainable_block_sparse_compress_b200.ops import Params

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "infllmv2.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"INFLLMV2_API\s+[\w\s\*]+?\b(infllmv2_\w+)\s*\(", text)))


def test_header_declares_the_four_calls():
    names = declared_symbols()
    for n in ("infllmv2_compress_keys", "infllmv2_select_blocks", "infllmv2_sparse_attn_prefill",
              "infllmv2_sparse_attn_decode", "infllmv2_workspace_size", "infllmv2_status_string"):
        assert n in names
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\bT\s+(\w+)", out.stdout))
    for name in declared_symbols():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # nothing but the API leaks out of the library
    assert {s for s in exported if s.startswith("infllmv2_")} == set(declared_symbols())


def test_version_and_status_strings(lib):
    assert lib.infllmv2_version() >= 100
    assert lib.infllmv2_status_string(0) == b"ok"
    assert b"workspace" in lib.infllmv2_status_string(-3)
    assert lib.infllmv2_status_string(12345) == b"unknown status"


def cp(**kw):
    base = dict(batch=1, num_q_heads=32, num_kv_heads=2, topk=96)
    base.update(kw)
    return ctypes.byref(Params(**base).c())


def test_param_validation(lib):
    f = lib.infllmv2_check_params
    assert f(cp()) == _lib.OK
    assert f(None) == _lib.ERR_INVALID_ARG
    assert f(cp(num_q_heads=31)) == _lib.ERR_INVALID_ARG  # not a multiple of Hkv
    assert f(cp(topk=2)) == _lib.ERR_INVALID_ARG  # n_init + n_local > topk
    assert f(cp(n_init=-1)) == _lib.ERR_INVALID_ARG
    assert f(cp(batch=0)) == _lib.ERR_INVALID_ARG
    assert f(cp(head_dim=64)) == _lib.ERR_UNSUPPORTED
    assert f(cp(block_size=128)) == _lib.ERR_UNSUPPORTED
    assert f(cp(kernel_size=64)) == _lib.ERR_UNSUPPORTED
    assert f(cp(num_q_heads=64, num_kv_heads=2)) == _lib.ERR_UNSUPPORTED  # G = 32
    assert f(cp(num_q_heads=6, num_kv_heads=2)) == _lib.ERR_UNSUPPORTED  # G = 3
    assert f(cp(topk=257)) == _lib.ERR_UNSUPPORTED
    assert f(cp(num_q_heads=8, num_kv_heads=1, topk=16)) == _lib.OK


def test_num_kernels(lib):
    for n, want in ((0, 0), (31, 0), (32, 1), (47, 1), (48, 2), (2048, 127), (131072, 8191)):
        assert lib.infllmv2_num_kernels(cp(), n) == want


def test_append_rejects_bad_arguments_before_launch(lib):
    good = 4096  # a fake, 16-byte aligned "device address": never dereferenced
    f = lib.infllmv2_append_kv
    assert f(cp(), None, good, good, good, good, 1024, good, None) == _lib.ERR_INVALID_ARG
    assert f(cp(), good, good, good, good, None, 1024, good, None) == _lib.ERR_INVALID_ARG
    assert f(cp(), good, good, good, good, good + 2, 1024, good, None) == _lib.ERR_INVALID_ARG
    assert f(cp(), good, good + 8, good, good, good, 1024, good, None) == _lib.ERR_INVALID_ARG
    assert f(cp(), good, good, good, good, good, 1024, None, None) == _lib.ERR_INVALID_ARG  # kc needed
    assert f(cp(), good, good, good, good, good, 0, good, None) == _lib.ERR_INVALID_ARG
    assert f(cp(head_dim=64), good, good, good, good, good, 1024, good, None) == _lib.ERR_UNSUPPORTED


def test_workspace_sizes(lib):
    ws = lib.infllmv2_workspace_size
    assert ws(cp(), _lib.OP_COMPRESS, 4096) == 0
    assert ws(cp(), _lib.OP_SELECT_PREFILL, 4096) == 0
    assert ws(cp(), _lib.OP_ATTN_PREFILL, 4096) == 0
    # decode selection merges its partials inside a thread-block cluster: no workspace
    assert ws(cp(batch=32), _lib.OP_SELECT_DECODE, 131072) == 0
    # decode attention: a cluster per (sequence, kv-head) when there are enough of them to
    # fill the GPU (no workspace); with very few, finer splits merged through the workspace
    assert ws(cp(batch=32), _lib.OP_ATTN_DECODE, 131072) == 0
    assert ws(cp(batch=1), _lib.OP_ATTN_DECODE, 131072) > 0
    assert ws(cp(), 99, 4096) == ctypes.c_size_t(-1).value
    assert ws(cp(), _lib.OP_COMPRESS, 0) == ctypes.c_size_t(-1).value
    assert ws(cp(), _lib.OP_COMPRESS, _lib.MAX_SEQ_LEN + 1) == ctypes.c_size_t(-1).value


def test_calls_reject_bad_arguments_before_launch(lib):
    # every failure below is detected on the host; nothing reaches the GPU
    good = 4096  # a fake, 16-byte aligned "device address": never dereferenced
    assert lib.infllmv2_compress_keys(cp(), None, None, 128, good, None) == _lib.ERR_INVALID_ARG
    assert lib.infllmv2_compress_keys(cp(), good, None, 128, None, None) == _lib.ERR_INVALID_ARG
    assert lib.infllmv2_compress_keys(cp(), good + 2, None, 128, good, None) == _lib.ERR_INVALID_ARG
    assert lib.infllmv2_compress_keys(cp(), good, None, 0, good, None) == _lib.ERR_INVALID_ARG
    assert lib.infllmv2_compress_keys(cp(head_dim=64), good, None, 128, good, None) == _lib.ERR_UNSUPPORTED
    assert lib.infllmv2_select_blocks(cp(), 0, None, good, None, 128, good, None, 0, None) == _lib.ERR_INVALID_ARG
    assert lib.infllmv2_select_blocks(cp(), 0, good, good, good, 128, good, None, 0, None) == _lib.ERR_INVALID_ARG
    assert lib.infllmv2_select_blocks(cp(), 7, good, good, None, 16, good, None, 0, None) == _lib.ERR_INVALID_ARG
    assert lib.infllmv2_sparse_attn_prefill(cp(), good, good, None, good, 128, good, None, None, 0,
                                            None) == _lib.ERR_INVALID_ARG
    assert lib.infllmv2_sparse_attn_prefill(cp(), good, good, good, good, 128, good, good + 1, None, 0,
                                            None) == _lib.ERR_INVALID_ARG
    # decode needs a workspace of the advertised size
    need = lib.infllmv2_workspace_size(cp(batch=4), _lib.OP_ATTN_DECODE, 1024)
    assert need > 0  # 8 items: the workspace path (the calls below must stop at the size check)
    assert lib.infllmv2_sparse_attn_decode(cp(batch=4), good, good, good, good, 1024, good, good, None, None, 0,
                                           None) == _lib.ERR_WORKSPACE
    assert lib.infllmv2_sparse_attn_decode(cp(batch=4), good, good, good, good, 1024, good, good, None, good,
                                           need - 1, None) == _lib.ERR_WORKSPACE
    # decode selection needs lens
    assert lib.infllmv2_select_blocks(cp(batch=4), 1, good, good, None, 1024, good, None, 0,
                                      None) == _lib.ERR_INVALID_ARG


def test_binding_rejects_host_tensors_before_calling_the_library():
    # the binding checks device, dtype and shape itself; nothing reaches the library
    from trainable_block_sparse_compress_b200 import ops
    p = ops.Params(batch=1, num_q_heads=16, num_kv_heads=1, topk=4)
    k = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.compress_keys(p, k)
    with pytest.raises(ValueError, match="CUDA tensor"):
        ops.append_kv(p, k[:, :, 0], k[:, :, 0], k, k, torch.zeros(1, dtype=torch.int32), k)


def test_chunk_calls_reject_bad_arguments_before_launch(lib):
    good = 4096  # a fake, 16-byte aligned "device address": never dereferenced
    sel = lib.infllmv2_select_blocks_chunk
    att = lib.infllmv2_sparse_attn_chunk
    # Lq in [1, Lmax], Lmax in [1, MAX_SEQ_LEN]
    assert sel(cp(), good, 0, good, None, None, 128, good, None, 0, None) == _lib.ERR_INVALID_ARG
    assert sel(cp(), good, 129, good, None, None, 128, good, None, 0, None) == _lib.ERR_INVALID_ARG
    assert sel(cp(), good, 8, good, None, None, _lib.MAX_SEQ_LEN + 1, good, None, 0, None) == _lib.ERR_INVALID_ARG
    # pointers: q, block_idx (and kc once a kernel exists) 16-byte aligned; length arrays 4-byte aligned
    assert sel(cp(), None, 8, good, None, None, 128, good, None, 0, None) == _lib.ERR_INVALID_ARG
    assert sel(cp(), good, 8, None, None, None, 128, good, None, 0, None) == _lib.ERR_INVALID_ARG
    assert sel(cp(), good, 8, good, good + 2, None, 128, good, None, 0, None) == _lib.ERR_INVALID_ARG
    assert sel(cp(), good, 8, good, None, good + 1, 128, good, None, 0, None) == _lib.ERR_INVALID_ARG
    assert sel(cp(head_dim=64), good, 8, good, None, None, 128, good, None, 0, None) == _lib.ERR_UNSUPPORTED
    assert att(cp(), good, 8, None, good, None, None, 128, good, good, None, None, 0, None) == _lib.ERR_INVALID_ARG
    assert att(cp(), good, 8, good, good, None, None, 128, good, None, None, None, 0, None) == _lib.ERR_INVALID_ARG
    assert att(cp(), good, 8, good, good, None, None, 128, good, good, good + 2, None, 0,
               None) == _lib.ERR_INVALID_ARG
    assert att(cp(), good, 200, good, good, None, None, 128, good, good, None, None, 0, None) == _lib.ERR_INVALID_ARG
    assert att(cp(), good, 8, good, good, good + 3, None, 128, good, good, None, None, 0,
               None) == _lib.ERR_INVALID_ARG


def test_score_and_pool_modes_are_checked(lib):
    f = lib.infllmv2_check_params
    for s, pm in ((0, 0), (1, 0), (0, 1), (1, 1)):
        assert f(cp(score_mode=s, pool_mode=pm)) == _lib.OK
    assert f(cp(score_mode=2)) == _lib.ERR_INVALID_ARG
    assert f(cp(pool_mode=-1)) == _lib.ERR_INVALID_ARG
    assert ctypes.sizeof(_lib.CParams) == 13 * 4  # the C struct: 10 int32, a float, 2 int32


def test_backward_rejects_bad_arguments_before_launch(lib):
    good = 4096  # a fake, 16-byte aligned "device address": never dereferenced
    f = lib.infllmv2_sparse_attn_backward
    need = lib.infllmv2_workspace_size(cp(), _lib.OP_ATTN_BACKWARD, 1024)
    assert need > 0
    args = [good] * 7 + [1024] + [good] * 3
    assert f(cp(), *args, None, 0, None) == _lib.ERR_WORKSPACE
    assert f(cp(), *args, good, need - 1, None) == _lib.ERR_WORKSPACE
    bad = list(args)
    bad[4] = good + 2  # lse must be 4-byte aligned
    assert f(cp(), *bad, good, need, None) == _lib.ERR_INVALID_ARG
    bad = list(args)
    bad[0] = None
    assert f(cp(), *bad, good, need, None) == _lib.ERR_INVALID_ARG
    bad = list(args)
    bad[7] = 0
    assert f(cp(), *bad, good, need, None) == _lib.ERR_INVALID_ARG


def test_decode_step_rejects_bad_arguments_before_launch(lib):
    good = 4096  # a fake, 16-byte aligned "device address": never dereferenced
    other = 8192
    f = lib.infllmv2_decode_step
    # q, k_new, v_new, k_cache, v_cache, kc, lens, lens_out, Lmax, block_idx, o, lse
    args = [good, None, None, good, good, good, good, None, 1024, good, good, None]
    for i in (0, 3, 4, 6, 9, 10):  # required pointers
        bad = list(args)
        bad[i] = None
        assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG, i
    for i in (0, 3, 4, 5, 9, 10):  # 16-byte aligned
        bad = list(args)
        bad[i] = good + 8
        assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG, i
    bad = list(args)
    bad[6] = good + 2  # lens 4-byte aligned
    assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG
    bad = list(args)
    bad[11] = good + 1  # lse 4-byte aligned
    assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG
    bad = list(args)
    bad[5] = None  # kc is needed once a semantic kernel exists
    assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG
    bad = list(args)
    bad[8] = 0
    assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG
    assert f(cp(head_dim=64), *args, None) == _lib.ERR_UNSUPPORTED
    # appending: both new rows, 16-byte aligned, and a lens_out distinct from lens
    app = list(args)
    app[1], app[2], app[7] = good, good, other
    bad = list(app)
    bad[2] = None
    assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG
    bad = list(app)
    bad[1] = good + 8
    assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG
    bad = list(app)
    bad[7] = None
    assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG
    bad = list(app)
    bad[7] = good  # == lens
    assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG
    bad = list(app)
    bad[7] = other + 2
    assert f(cp(), *bad, None) == _lib.ERR_INVALID_ARG
