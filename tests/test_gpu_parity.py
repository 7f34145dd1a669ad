"""Parity of the CUDA library (called through its C ABI) with the CPU oracle.

Each step is first checked in isolation on inputs the oracle produced (the GPU selection
is fed the oracle's kernels, the GPU attention the oracle's block lists), then the whole
path runs on the five benchmark workloads and is compared on sampled rows.
"""
import json
import os
import warnings

import numpy as np
import pytest
import torch

import oracle
from parity import (bf16_to_f64, bf16_ulp_diff, check_row_selection, compare_attention, compare_grad,
                    compare_selection, u16)
from trainable_block_sparse_compress_b200 import build, ops
from trainable_block_sparse_compress_b200.synthetic import WORKLOADS, Workload, as_u16, make_inputs

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def cuda_library():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    assert ops.device_error(clear=True) == 0
    yield
    assert ops.device_error(clear=True) == 0, "a kernel hit its wait time limit"


def oparams(p: ops.Params) -> oracle.Params:
    return oracle.Params(p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim, p.block_size, p.kernel_size,
                         p.kernel_stride, p.topk, p.n_init, p.n_local, p.softmax_scale, p.score_mode, p.pool_mode)


def inputs(B, L, Hq, Hkv, seed, mode="prefill", lens=None):
    wl = Workload("t", mode, B, L, Hq, Hkv, 16)
    x = make_inputs(wl, seed)
    if lens is not None:
        x.lens = torch.tensor(lens, dtype=torch.int32)
    return x


# ------------------------------------------------------------------ compression

@pytest.mark.parametrize("B,H,L,lens", [(2, 2, 4500, None), (3, 1, 1000, [1000, 31, 517]), (1, 2, 32, None),
                                        (1, 1, 31, None), (2, 2, 5000, [48, 4999])])
def test_compress_matches_oracle(B, H, L, lens):
    x = inputs(B, L, H, H, seed=100 + L, mode="decode" if lens else "prefill", lens=lens)
    p = ops.Params(B, H, H, topk=16)
    lens_t = None if lens is None else x.lens.cuda()
    kc_g = u16(ops.compress_keys(p, x.k.cuda(), lens=lens_t))
    kc_o = oracle.compress(oparams(p), as_u16(x.k), lens=None if lens is None else np.array(lens, np.int32))
    nks = [oracle.num_kernels(oparams(p), n) for n in (lens or [L] * B)]
    # the mean is exact on both sides and rounded once: bit-exact
    for b in range(B):
        a, o = kc_g[b, :, :nks[b]], kc_o[b, :, :nks[b]]
        assert np.array_equal(a, o), f"{int((a != o).sum())} kernel values differ, max {bf16_ulp_diff(a, o).max()} ulp"


def test_compress_closed_form_exact():
    c = np.array([1, -3, 2.5, 0, 7, -1.25, 6, 6, -8, 0.5, 3, -2] * 30, dtype=np.float32)
    L = 16 * len(c)
    k = torch.from_numpy(np.repeat(c, 16)).view(1, 1, L, 1).expand(1, 1, L, 128).contiguous().to(torch.bfloat16)
    p = ops.Params(1, 1, 1, topk=16)
    kc = bf16_to_f64(u16(ops.compress_keys(p, k.cuda())))
    want = (c[:-1].astype(np.float64) + c[1:]) / 2
    assert np.array_equal(kc[0, 0], np.repeat(want[:, None], 128, 1))


# -------------------------------------------------------------------- selection

GOLDEN_CASES = [c for f in ("select_closed_form.json", "select_variants.json")
                for c in json.load(open(os.path.join(GOLDEN, f)))["cases"]]


@pytest.mark.parametrize("case", GOLDEN_CASES, ids=lambda c: c["name"])
@pytest.mark.parametrize("mode", ["prefill", "decode", "step"])
def test_select_closed_form_cases(case, mode):
    L, Hq = case["seq_len"], case["num_q_heads"]
    k = torch.zeros((1, 1, L, 128))
    for comp, key in ((0, "u"), (1, "w")):
        k[0, 0, :, comp] = case.get(key + "_default", 0.0)
        for j, val in case[key].items():
            k[0, 0, int(j) * 64:(int(j) + 1) * 64, comp] = val
    q = torch.zeros((1, L, Hq, 128))
    if not case.get("zero_query"):
        for h in range(Hq):
            q[0, :, h, h] = 8.0
    p = ops.Params(1, Hq, 1, topk=case["topk"], n_init=case["n_init"], n_local=case["n_local"],
                   softmax_scale=0.125, score_mode=case.get("score_mode", 0), pool_mode=case.get("pool_mode", 0))
    t = case["query_pos"]
    if mode == "prefill":
        kc = ops.compress_keys(p, k.to(torch.bfloat16).cuda())
        idx = ops.select_blocks_prefill(p, q.to(torch.bfloat16).cuda(), kc).cpu().numpy()
        assert idx[0, 0, t].tolist() == case["expected"]
    else:  # the same row as a decode query over a cache of t + 1 tokens (alone, or in the fused step)
        lens = torch.tensor([t + 1], dtype=torch.int32).cuda()
        kg = k.to(torch.bfloat16).cuda()
        kc = ops.compress_keys(p, kg, lens=lens)
        qd = q[:, t].to(torch.bfloat16).contiguous().cuda()
        if mode == "decode":
            idx = ops.select_blocks_decode(p, qd, kc, lens, L)
        else:
            _, _, idx = ops.decode_step(p, qd, kg, torch.zeros_like(kg), kc, lens)
        assert idx.cpu().numpy()[0, 0, 0].tolist() == case["expected"]


SELECT_CASES = [
    # B, L, Hq, Hkv, topk, n_init, n_local
    (1, 4500, 32, 2, 16, 1, 2),   # 5 kernel tiles, ragged tail (4500 % 64 = 20, % 8 = 4)
    (2, 1000, 8, 1, 6, 1, 2),     # G = 8, two sequences
    (1, 777, 2, 2, 5, 2, 1),      # G = 1, two initial blocks, one local block
    (1, 2000, 16, 1, 256, 1, 2),  # topk larger than the number of blocks
    (1, 20, 16, 1, 4, 1, 2),      # no complete kernel: forced blocks only
    (1, 1100, 4, 1, 3, 0, 0),     # nothing forced
    (1, 1500, 4, 2, 8, 1, 2),     # G = 2
    (1, 14000, 2, 2, 24, 1, 2),   # G = 1 past the tensor-core kernel's key storage: m16n8k16 kernel
]


def prefill_rows(L):
    if L <= 1200:
        return np.arange(L)
    return np.unique(np.concatenate([np.arange(200), np.arange(200, L - 200, 13), np.arange(L - 200, L)]))


@pytest.mark.parametrize("B,L,Hq,Hkv,topk,ni,nl", SELECT_CASES)
def test_select_prefill_matches_oracle(B, L, Hq, Hkv, topk, ni, nl):
    x = inputs(B, L, Hq, Hkv, seed=200 + L)
    p = ops.Params(B, Hq, Hkv, topk=topk, n_init=ni, n_local=nl)
    op = oparams(p)
    kc_o = oracle.compress(op, as_u16(x.k))
    kc_t = torch.from_numpy(kc_o.view(np.int16)).view(torch.bfloat16).cuda()
    idx_g = ops.select_blocks_prefill(p, x.q.cuda(), kc_t).cpu().numpy()
    rows = prefill_rows(L)
    idx_o, sc = oracle.select(op, as_u16(x.q), kc_o, rows=rows, want_scores=True)
    compare_selection(idx_g[:, :, rows], idx_o, sc, np.tile(rows, (B, 1)), p)


def test_select_prefill_long_sequence():
    # 200,000 tokens at G = 16: 3125 blocks of keys per query row, which the tensor-core
    # kernel holds by running its Kc ring with two slots instead of three
    B, L, Hq, Hkv, topk = 1, 200000, 16, 1, 96
    x = inputs(B, L, Hq, Hkv, seed=210)
    p = ops.Params(B, Hq, Hkv, topk=topk)
    op = oparams(p)
    kc_o = oracle.compress(op, as_u16(x.k))
    kc_t = torch.from_numpy(kc_o.view(np.int16)).view(torch.bfloat16).cuda()
    idx_g = ops.select_blocks_prefill(p, x.q.cuda(), kc_t).cpu().numpy()
    rows = np.unique(np.concatenate([np.arange(0, L, 997), np.arange(L - 64, L)]))
    idx_o, sc = oracle.select(op, as_u16(x.q), kc_o, rows=rows, want_scores=True)
    compare_selection(idx_g[:, :, rows], idx_o, sc, np.tile(rows, (B, 1)), p)


# score / pool variants: (score_mode, pool_mode); (0, 0) is the default reading above
VARIANTS = [(1, 0), (0, 1), (1, 1)]


@pytest.mark.parametrize("score_mode,pool_mode", VARIANTS)
@pytest.mark.parametrize("B,L,Hq,Hkv,topk", [(1, 3000, 32, 2, 16), (2, 1000, 8, 1, 6)])
def test_select_prefill_variants_match_oracle(B, L, Hq, Hkv, topk, score_mode, pool_mode):
    # G = 16 (tcgen05 kernel) and G = 8 (m16n8k16 kernel), rows across the sequence
    x = inputs(B, L, Hq, Hkv, seed=250 + L + 7 * score_mode + pool_mode)
    p = ops.Params(B, Hq, Hkv, topk=topk, score_mode=score_mode, pool_mode=pool_mode)
    op = oparams(p)
    kc_o = oracle.compress(op, as_u16(x.k))
    kc_t = torch.from_numpy(kc_o.view(np.int16)).view(torch.bfloat16).cuda()
    idx_g = ops.select_blocks_prefill(p, x.q.cuda(), kc_t).cpu().numpy()
    rows = prefill_rows(L)
    idx_o, sc = oracle.select(op, as_u16(x.q), kc_o, rows=rows, want_scores=True)
    _, n_tie = compare_selection(idx_g[:, :, rows], idx_o, sc, np.tile(rows, (B, 1)), p)
    report_ties(f"prefill variant s{score_mode} p{pool_mode} G={Hq // Hkv}", n_tie, B * Hkv * len(rows))


@pytest.mark.parametrize("score_mode,pool_mode", VARIANTS)
def test_select_decode_variants_match_oracle(score_mode, pool_mode):
    lens, Lmax, Hq, Hkv, topk = [9000, 1, 31, 1500, 2049, 64, 65], 9000, 32, 2, 16
    B = len(lens)
    x = inputs(B, Lmax, Hq, Hkv, seed=350 + 7 * score_mode + pool_mode, mode="decode", lens=lens)
    p = ops.Params(B, Hq, Hkv, topk=topk, score_mode=score_mode, pool_mode=pool_mode)
    op = oparams(p)
    lens_np = np.array(lens, np.int32)
    kc_o = oracle.compress(op, as_u16(x.k), lens=lens_np)
    kc_t = torch.from_numpy(kc_o.view(np.int16)).view(torch.bfloat16).cuda()
    idx_g = ops.select_blocks_decode(p, x.q.cuda(), kc_t, x.lens.cuda(), Lmax).cpu().numpy()
    idx_o, sc = oracle.select(op, as_u16(x.q)[:, None], kc_o, lens=lens_np, Lmax=Lmax, want_scores=True)
    compare_selection(idx_g, idx_o, sc, (lens_np - 1)[:, None], p)


@pytest.mark.parametrize("mode", ["prefill", "decode"])
def test_logit_sum_with_negative_scores(mode):
    # keys shifted by -2 in every component and queries made positive: nearly every logit,
    # and so every block's logit sum, is negative; the top-k order must still follow the
    # values (order-preserving keys over all 32 bits)
    B, L, Hq, Hkv, topk = 1, 3000, 32, 2, 16
    x = inputs(B, L, Hq, Hkv, seed=450)
    q = x.q.float().abs().to(torch.bfloat16)
    k = (x.k.float() - 2.0).to(torch.bfloat16)
    p = ops.Params(B, Hq, Hkv, topk=topk, score_mode=1)
    op = oparams(p)
    kc_o = oracle.compress(op, as_u16(k))
    kc_t = torch.from_numpy(kc_o.view(np.int16)).view(torch.bfloat16).cuda()
    rows = prefill_rows(L)
    idx_o, sc = oracle.select(op, as_u16(q), kc_o, rows=rows, want_scores=True)
    fin = sc[np.isfinite(sc)]
    assert (fin < 0).mean() > 0.99
    if mode == "prefill":
        idx_g = ops.select_blocks_prefill(p, q.cuda(), kc_t).cpu().numpy()[:, :, rows]
        compare_selection(idx_g, idx_o, sc, np.tile(rows, (B, 1)), p)
    else:  # each sampled row as a decode query over the cache up to it
        lens_np = (rows[-40:] + 1).astype(np.int32)
        pd = ops.Params(len(lens_np), Hq, Hkv, topk=topk, score_mode=1)
        kd = k.expand(len(lens_np), -1, -1, -1).contiguous().cuda()
        lens_t = torch.from_numpy(lens_np).cuda()
        kc_d = ops.compress_keys(pd, kd, lens=lens_t)
        idx_g = ops.select_blocks_decode(pd, q[0, rows[-40:]].contiguous().cuda(), kc_d, lens_t, L).cpu().numpy()
        for r in range(len(lens_np)):
            for g in range(Hkv):
                res = check_row_selection(idx_g[r, g, 0], idx_o[0, g, len(rows) - 40 + r],
                                          sc[0, g, len(rows) - 40 + r], int(lens_np[r] - 1), topk, 1, 2)
                assert res in ("exact", "tie"), res


@pytest.mark.parametrize("lens,Lmax,Hq,Hkv,topk", [([3000, 1, 31, 1500, 2049], 3000, 32, 2, 16),
                                                  ([70, 64, 65, 128], 128, 8, 1, 3),
                                                  ([9000, 8193], 9000, 4, 4, 100)])
def test_select_decode_matches_oracle(lens, Lmax, Hq, Hkv, topk):
    B = len(lens)
    x = inputs(B, Lmax, Hq, Hkv, seed=300 + Lmax, mode="decode", lens=lens)
    p = ops.Params(B, Hq, Hkv, topk=topk)
    op = oparams(p)
    lens_np = np.array(lens, np.int32)
    kc_o = oracle.compress(op, as_u16(x.k), lens=lens_np)
    kc_t = torch.from_numpy(kc_o.view(np.int16)).view(torch.bfloat16).cuda()
    idx_g = ops.select_blocks_decode(p, x.q.cuda(), kc_t, x.lens.cuda(), Lmax).cpu().numpy()
    idx_o, sc = oracle.select(op, as_u16(x.q)[:, None], kc_o, lens=lens_np, Lmax=Lmax, want_scores=True)
    compare_selection(idx_g, idx_o, sc, (lens_np - 1)[:, None], p)


# -------------------------------------------------------------------- attention

ATTN_CASES = [(1, 4500, 32, 2, 16), (2, 1000, 8, 1, 6), (1, 777, 2, 2, 5), (1, 700, 16, 1, 16), (1, 64, 16, 1, 4),
              (1, 900, 8, 2, 6), (1, 500, 4, 2, 4)]


@pytest.mark.parametrize("B,L,Hq,Hkv,topk", ATTN_CASES)
def test_attn_prefill_matches_oracle(B, L, Hq, Hkv, topk):
    x = inputs(B, L, Hq, Hkv, seed=400 + L)
    p = ops.Params(B, Hq, Hkv, topk=topk)
    op = oparams(p)
    kc_o = oracle.compress(op, as_u16(x.k))
    idx_all = oracle.select(op, as_u16(x.q), kc_o)  # every row, so the GPU sees the oracle's lists
    o_g, lse_g = ops.sparse_attn_prefill(p, x.q.cuda(), x.k.cuda(), x.v.cuda(),
                                         torch.from_numpy(idx_all).cuda())
    rows = prefill_rows(L)[::3]
    o_o, lse_o = oracle.attn(op, as_u16(x.q), as_u16(x.k), as_u16(x.v), idx_all[:, :, rows], rows=rows)
    o_g = o_g.float().cpu().numpy()[:, rows]
    lse_g = lse_g.cpu().numpy()[:, :, rows]
    compare_attention(o_g, o_o, lse_g, lse_o)


@pytest.mark.parametrize("lens,Lmax,Hq,Hkv,topk", [([3000, 1, 31, 1500, 2049], 3000, 32, 2, 16),
                                                  ([3000, 1, 31, 1500, 2049], 3000, 8, 2, 16),
                                                  ([9000, 8193, 64], 9000, 16, 1, 96)])
def test_attn_decode_matches_oracle(lens, Lmax, Hq, Hkv, topk):
    # 10 (sequence, kv-head) items take the cluster path (G = 16 and G = 4); 3 items the
    # workspace split path
    B = len(lens)
    x = inputs(B, Lmax, Hq, Hkv, seed=500 + Lmax, mode="decode", lens=lens)
    p = ops.Params(B, Hq, Hkv, topk=topk)
    op = oparams(p)
    lens_np = np.array(lens, np.int32)
    kc_o = oracle.compress(op, as_u16(x.k), lens=lens_np)
    idx_o = oracle.select(op, as_u16(x.q)[:, None], kc_o, lens=lens_np, Lmax=Lmax)
    o_g, lse_g = ops.sparse_attn_decode(p, x.q.cuda(), x.k.cuda(), x.v.cuda(), x.lens.cuda(),
                                        torch.from_numpy(idx_o).cuda())
    o_o, lse_o = oracle.attn(op, as_u16(x.q)[:, None], as_u16(x.k), as_u16(x.v), idx_o, lens=lens_np)
    compare_attention(o_g.float().cpu().numpy(), o_o[:, 0], lse_g.cpu().numpy(), lse_o[:, :, 0])


def test_decode_at_the_maximum_length():
    # caches of INFLLMV2_MAX_SEQ_LEN tokens: 16383 kernels per sequence, so the selection's
    # clusters run at their 2048-kernel-per-CTA limit (20 items: clusters of 8), next to
    # sequences of 1, 33, 64 and 65 tokens in the same batch
    Lmax = 262144
    lens = [262144, 262143, 131072, 65, 64, 1, 200000, 5000, 262100, 33]
    B, Hq, Hkv, topk = len(lens), 32, 2, 96
    x = inputs(B, Lmax, Hq, Hkv, seed=800, mode="decode", lens=lens)
    p = ops.Params(B, Hq, Hkv, topk=topk)
    op = oparams(p)
    lens_np = np.array(lens, np.int32)
    kc_o = oracle.compress(op, as_u16(x.k), lens=lens_np)
    k, v, q, ln = x.k.cuda(), x.v.cuda(), x.q.cuda(), x.lens.cuda()
    kc_g = ops.compress_keys(p, k, lens=ln)
    for b, n in enumerate(lens):
        nk = oracle.num_kernels(op, n)
        assert np.array_equal(u16(kc_g)[b, :, :nk], kc_o[b, :, :nk])
    kc_t = torch.from_numpy(kc_o.view(np.int16)).view(torch.bfloat16).cuda()
    idx_g = ops.select_blocks_decode(p, q, kc_t, ln, Lmax).cpu().numpy()
    idx_o, sc = oracle.select(op, as_u16(x.q)[:, None], kc_o, lens=lens_np, Lmax=Lmax, want_scores=True)
    compare_selection(idx_g, idx_o, sc, (lens_np - 1)[:, None], p)
    o_g, lse_g = ops.sparse_attn_decode(p, q, k, v, ln, torch.from_numpy(idx_o).cuda())
    o_o, lse_o = oracle.attn(op, as_u16(x.q)[:, None], as_u16(x.k), as_u16(x.v), idx_o, lens=lens_np)
    compare_attention(o_g.float().cpu().numpy(), o_o[:, 0], lse_g.cpu().numpy(), lse_o[:, :, 0])
    # the fused step at the same lengths: the separate selection's lists, the exact
    # attention over them
    o_f, lse_f, idx_f = ops.decode_step(p, q, k, v, kc_t, ln)
    assert np.array_equal(idx_f.cpu().numpy(), idx_g)
    o_o2, lse_o2 = oracle.attn(op, as_u16(x.q)[:, None], as_u16(x.k), as_u16(x.v), idx_g, lens=lens_np)
    compare_attention(o_f.float().cpu().numpy(), o_o2[:, 0], lse_f.cpu().numpy(), lse_o2[:, :, 0])


def test_attn_decode_many_items_per_cta_is_deterministic():
    # more work items than CTAs, ragged lengths: repeated runs must agree bit for bit
    # and match the oracle
    rng = np.random.default_rng(7)
    B, Lmax, Hq, Hkv, topk = 24, 20000, 32, 2, 96
    lens = rng.integers(1, Lmax + 1, size=B).tolist()
    x = inputs(B, Lmax, Hq, Hkv, seed=700, mode="decode", lens=lens)
    p = ops.Params(B, Hq, Hkv, topk=topk)
    op = oparams(p)
    lens_np = np.array(lens, np.int32)
    kc_o = oracle.compress(op, as_u16(x.k), lens=lens_np)
    idx_o = oracle.select(op, as_u16(x.q)[:, None], kc_o, lens=lens_np, Lmax=Lmax)
    q, k, v, ln, idx = x.q.cuda(), x.k.cuda(), x.v.cuda(), x.lens.cuda(), torch.from_numpy(idx_o).cuda()
    o_ref, lse_ref = ops.sparse_attn_decode(p, q, k, v, ln, idx)
    for _ in range(5):
        o_g, lse_g = ops.sparse_attn_decode(p, q, k, v, ln, idx)
        assert torch.equal(o_g, o_ref) and torch.equal(lse_g, lse_ref)
    o_o, lse_o = oracle.attn(op, as_u16(x.q)[:, None], as_u16(x.k), as_u16(x.v), idx_o, lens=lens_np)
    compare_attention(o_ref.float().cpu().numpy(), o_o[:, 0], lse_ref.cpu().numpy(), lse_o[:, :, 0])


def test_attn_prefill_is_deterministic():
    B, L, Hq, Hkv, topk = 1, 6000, 32, 2, 24
    x = inputs(B, L, Hq, Hkv, seed=701)
    p = ops.Params(B, Hq, Hkv, topk=topk)
    q, k, v = x.q.cuda(), x.k.cuda(), x.v.cuda()
    kc = ops.compress_keys(p, k)
    idx = ops.select_blocks_prefill(p, q, kc)
    o_ref, lse_ref = ops.sparse_attn_prefill(p, q, k, v, idx)
    idx_ref = idx.clone()
    for _ in range(3):
        assert torch.equal(ops.select_blocks_prefill(p, q, kc), idx_ref)
        o_g, lse_g = ops.sparse_attn_prefill(p, q, k, v, idx)
        assert torch.equal(o_g, o_ref) and torch.equal(lse_g, lse_ref)


def test_attn_decode_ignores_garbage_past_the_length():
    # cache rows at or past lens[b] hold NaN: they must not reach the output
    lens, Lmax = [100, 64, 65], 192
    B, Hq, Hkv = 3, 16, 1
    x = inputs(B, Lmax, Hq, Hkv, seed=600, mode="decode", lens=lens)
    p = ops.Params(B, Hq, Hkv, topk=4)
    op = oparams(p)
    lens_np = np.array(lens, np.int32)
    kc_o = oracle.compress(op, as_u16(x.k), lens=lens_np)
    idx_o = oracle.select(op, as_u16(x.q)[:, None], kc_o, lens=lens_np, Lmax=Lmax)
    k, v = x.k.clone(), x.v.clone()
    for b, n in enumerate(lens):
        k[b, :, n:] = float("nan")
        v[b, :, n:] = float("nan")
    o_g, _ = ops.sparse_attn_decode(p, x.q.cuda(), k.cuda(), v.cuda(), x.lens.cuda(), torch.from_numpy(idx_o).cuda())
    o_o, _ = oracle.attn(op, as_u16(x.q)[:, None], as_u16(x.k), as_u16(x.v), idx_o, lens=lens_np)
    assert torch.isfinite(o_g).all()
    compare_attention(o_g.float().cpu().numpy(), o_o[:, 0])


# ------------------------------------------------------------- fused decode step

def run_decode_step_case(lens, Lmax, Hq, Hkv, topk, seed, score_mode=0, pool_mode=0, nan_tail=False):
    """The fused decode step (selection and attention in one launch) on the oracle's
    kernels: its block lists are the separate selection's, bit for bit, and checked
    against the oracle's; its outputs against the exact attention over those lists and
    against the separate attention call.  With nan_tail the cache rows at or past lens[b]
    hold NaN, which must not reach the outputs."""
    B = len(lens)
    x = inputs(B, Lmax, Hq, Hkv, seed=seed, mode="decode", lens=lens)
    p = ops.Params(B, Hq, Hkv, topk=topk, score_mode=score_mode, pool_mode=pool_mode)
    op = oparams(p)
    lens_np = np.array(lens, np.int32)
    kc_o = oracle.compress(op, as_u16(x.k), lens=lens_np)
    kc_t = torch.from_numpy(kc_o.view(np.int16)).view(torch.bfloat16).cuda()
    k, v = x.k.clone(), x.v.clone()
    if nan_tail:
        for b, n in enumerate(lens):
            k[b, :, n:] = float("nan")
            v[b, :, n:] = float("nan")
    q, kd, vd, ln = x.q.cuda(), k.cuda(), v.cuda(), x.lens.cuda()
    o_g, lse_g, idx_g = ops.decode_step(p, q, kd, vd, kc_t, ln)
    idx_s = ops.select_blocks_decode(p, q, kc_t, ln, Lmax)
    o_s, lse_s = ops.sparse_attn_decode(p, q, kd, vd, ln, idx_s)
    torch.cuda.synchronize()
    assert torch.equal(idx_g, idx_s)
    assert torch.isfinite(o_g).all()
    idx_gn = idx_g.cpu().numpy()
    idx_o, sc = oracle.select(op, as_u16(x.q)[:, None], kc_o, lens=lens_np, Lmax=Lmax, want_scores=True)
    _, n_tie = compare_selection(idx_gn, idx_o, sc, (lens_np - 1)[:, None], p)
    o_o, lse_o = oracle.attn(op, as_u16(x.q)[:, None], as_u16(x.k), as_u16(x.v), idx_gn, lens=lens_np)
    compare_attention(o_g.float().cpu().numpy(), o_o[:, 0], lse_g.cpu().numpy(), lse_o[:, :, 0])
    # the separate attention may split the list over CTAs differently: last bits only
    assert (o_g.float() - o_s.float()).abs().max().item() <= 1e-2
    assert (lse_g - lse_s).abs().max().item() <= 1e-4
    return n_tie


@pytest.mark.parametrize("lens,Lmax,Hq,Hkv,topk", [([3000, 1, 31, 1500, 2049], 3000, 32, 2, 16),
                                                  ([70, 64, 65, 128], 128, 8, 1, 3),
                                                  ([9000, 8193, 64], 9000, 16, 1, 96),
                                                  ([9000, 8193], 9000, 4, 4, 100),
                                                  ([20000, 4097, 12345, 600, 19999, 33], 20000, 32, 2, 96)])
def test_decode_step_matches_oracle(lens, Lmax, Hq, Hkv, topk):
    # 3 to 12 items: clusters of 16 CTAs
    run_decode_step_case(lens, Lmax, Hq, Hkv, topk, seed=900 + Lmax)


@pytest.mark.parametrize("B", [40, 80])
def test_decode_step_small_clusters(B):
    # 80 and 160 (sequence, kv-head) items: clusters of 2 CTAs and of 1
    lens = np.random.default_rng(B).integers(1, 4001, size=B).tolist()
    run_decode_step_case(lens, 4000, 32, 2, 16, seed=980 + B)


@pytest.mark.parametrize("score_mode,pool_mode", VARIANTS)
def test_decode_step_variants_match_oracle(score_mode, pool_mode):
    run_decode_step_case([5000, 4999, 64, 1000], 5000, 32, 2, 24, seed=950, score_mode=score_mode,
                         pool_mode=pool_mode)


def test_decode_step_ignores_garbage_past_the_length():
    run_decode_step_case([100, 64, 65, 3001], 3072, 16, 1, 8, seed=960, nan_tail=True)


def test_decode_step_empty_sequence_and_determinism():
    # lens[b] = 0: no query, the list is all -1, o is 0 and lse is -inf; the other rows
    # are unaffected, and repeated steps agree bit for bit
    lens, Lmax, Hq, Hkv, topk = [0, 3000, 5, 2500], 3000, 32, 2, 16
    B = len(lens)
    x = inputs(B, Lmax, Hq, Hkv, seed=970, mode="decode", lens=lens)
    p = ops.Params(B, Hq, Hkv, topk=topk)
    q, k, v, ln = x.q.cuda(), x.k.cuda(), x.v.cuda(), x.lens.cuda()
    kc = ops.compress_keys(p, k, lens=ln)
    o_ref, lse_ref, idx_ref = ops.decode_step(p, q, k, v, kc, ln)
    assert torch.all(idx_ref[0] == -1)
    assert torch.all(o_ref[0] == 0) and torch.all(torch.isneginf(lse_ref[0]))
    for _ in range(3):
        o_g, lse_g, idx_g = ops.decode_step(p, q, k, v, kc, ln)
        assert torch.equal(idx_g, idx_ref) and torch.equal(o_g, o_ref) and torch.equal(lse_g, lse_ref)
    # rows 1..3 against the oracle
    op = oparams(ops.Params(B - 1, Hq, Hkv, topk=topk))
    lens_np = np.array(lens[1:], np.int32)
    kc_o = oracle.compress(op, as_u16(x.k[1:]), lens=lens_np)
    idx_o, sc = oracle.select(op, as_u16(x.q[1:])[:, None], kc_o, lens=lens_np, Lmax=Lmax, want_scores=True)
    idx_gn = idx_ref[1:].cpu().numpy()
    compare_selection(idx_gn, idx_o, sc, (lens_np - 1)[:, None], ops.Params(B - 1, Hq, Hkv, topk=topk))
    o_o, lse_o = oracle.attn(op, as_u16(x.q[1:])[:, None], as_u16(x.k[1:]), as_u16(x.v[1:]), idx_gn, lens=lens_np)
    compare_attention(o_ref[1:].float().cpu().numpy(), o_o[:, 0], lse_ref[1:].cpu().numpy(), lse_o[:, :, 0])


def test_decode_step_with_append_equals_append_then_step():
    # the step that appends the new token itself must leave the caches, kc and the lengths
    # as infllmv2_append_kv does, and give the outputs of a step on the appended cache;
    # lengths cover a completed kernel (n = 32 + 16 i), a block boundary, an empty cache
    # and a full one (left untouched, flagged)
    Lmax, Hq, Hkv, topk = 3000, 32, 2, 16
    lens0 = [2015, 2047, 63, 0, 31, 2999, 1000, 3000]  # cached tokens before the step
    B = len(lens0)
    x = inputs(B, Lmax, Hq, Hkv, seed=990, mode="decode", lens=[max(n, 1) for n in lens0])
    p = ops.Params(B, Hq, Hkv, topk=topk)
    g = torch.Generator().manual_seed(991)
    k_new = torch.randn((B, Hkv, 128), generator=g).to(torch.bfloat16).cuda()
    v_new = torch.randn((B, Hkv, 128), generator=g).to(torch.bfloat16).cuda()
    q, k0, v0 = x.q.cuda(), x.k.cuda(), x.v.cuda()
    l0 = torch.tensor(lens0, dtype=torch.int32).cuda()
    kc0 = ops.compress_keys(p, k0, lens=l0)
    # reference: the append kernel, then the step without append
    k_a, v_a, kc_a, l_a = k0.clone(), v0.clone(), kc0.clone(), l0.clone()
    ops.append_kv(p, k_new, v_new, k_a, v_a, l_a, kc_a)
    o_a, lse_a, idx_a = ops.decode_step(p, q, k_a, v_a, kc_a, l_a)
    assert ops.device_error(clear=True) != 0  # the full cache (lens 3000) was flagged
    # the fused step with append
    k_f, v_f, kc_f = k0.clone(), v0.clone(), kc0.clone()
    l_out = torch.full_like(l0, -5)
    o_f, lse_f, idx_f, l_f = ops.decode_step(p, q, k_f, v_f, kc_f, l0, k_new=k_new, v_new=v_new, lens_out=l_out)
    torch.cuda.synchronize()
    assert ops.device_error(clear=True) != 0
    assert torch.equal(l_f, l_a) and torch.equal(l0.cpu(), torch.tensor(lens0, dtype=torch.int32))
    bits = lambda t: t.view(torch.int16)  # bitwise: kc rows past a sequence's kernels are never written
    assert torch.equal(bits(k_f), bits(k_a)) and torch.equal(bits(v_f), bits(v_a))
    assert torch.equal(bits(kc_f), bits(kc_a))
    assert torch.equal(idx_f, idx_a) and torch.equal(o_f, o_a) and torch.equal(lse_f, lse_a)


# ---------------------------------------------------------- whole path, workloads

def report_ties(what, n_tie, n_rows):
    """Makes the number of excused near-tie rows visible in the test log (warnings summary)."""
    warnings.warn(f"{what}: {n_tie} of {n_rows} (sequence, kv-head, row) selections differ from the oracle's "
                  f"only through an excused near-tie", UserWarning)


def sample_rows(L):
    if L <= 4096:
        return np.arange(L)
    stride = max(1, L // 1024)
    return np.unique(np.concatenate([np.arange(128), np.arange(128, L - 128, stride), np.arange(L - 128, L)]))


@pytest.mark.parametrize("name", ["prefill_2k", "prefill_32k", "prefill_128k"])
def test_prefill_workload_end_to_end(name):
    wl = WORKLOADS[name]
    x = make_inputs(wl, seed=0)
    p = ops.Params.from_workload(wl)
    op = oparams(p)
    q, k, v = x.q.cuda(), x.k.cuda(), x.v.cuda()
    o_g, lse_g, idx_g, kc_g = ops.prefill(p, q, k, v)
    torch.cuda.synchronize()
    kc_o = oracle.compress(op, as_u16(x.k))
    assert np.array_equal(u16(kc_g), kc_o)
    rows = sample_rows(wl.seq_len)
    rows_t = torch.from_numpy(rows).cuda()
    idx_o, sc = oracle.select(op, as_u16(x.q), kc_o, rows=rows, want_scores=True)
    idx_gr = idx_g[:, :, rows_t].cpu().numpy()
    same, n_tie = compare_selection(idx_gr, idx_o, sc, np.tile(rows, (wl.batch, 1)), p)
    report_ties(name, n_tie, same.size)
    # every sampled row's output against the exact attention over the GPU's own block
    # lists: rows whose list differs from the oracle's through an excused near-tie are
    # checked too, on the list the GPU actually used
    o_o, lse_o = oracle.attn(op, as_u16(x.q), as_u16(x.k), as_u16(x.v), idx_gr, rows=rows)
    o_gr = o_g[:, rows_t].float().cpu().numpy()  # [B, R, Hq, d]
    lse_gr = lse_g[:, :, rows_t].cpu().numpy()   # [B, Hq, R]
    compare_attention(o_gr, o_o, lse_gr, lse_o)


@pytest.mark.parametrize("name", ["decode_32k", "decode_ragged_128k"])
def test_decode_workload_end_to_end(name):
    wl = WORKLOADS[name]
    x = make_inputs(wl, seed=0)
    p = ops.Params.from_workload(wl)
    op = oparams(p)
    lens_np = x.lens.numpy()
    k, v, lens = x.k.cuda(), x.v.cuda(), x.lens.cuda()
    kc_g = ops.compress_keys(p, k, lens=lens)
    o_g, lse_g, idx_g = ops.decode(p, x.q.cuda(), k, v, kc_g, lens, wl.seq_len)
    torch.cuda.synchronize()
    kc_o = oracle.compress(op, as_u16(x.k), lens=lens_np)
    kcg = u16(kc_g)
    for b in range(wl.batch):
        nk = oracle.num_kernels(op, int(lens_np[b]))
        assert np.array_equal(kcg[b, :, :nk], kc_o[b, :, :nk]), b
    idx_o, sc = oracle.select(op, as_u16(x.q)[:, None], kc_o, lens=lens_np, Lmax=wl.seq_len, want_scores=True)
    idx_gn = idx_g.cpu().numpy()
    same, n_tie = compare_selection(idx_gn, idx_o, sc, (lens_np - 1)[:, None], p)
    report_ties(name, n_tie, same.size)
    # all rows, each on the block list the GPU used (near-tie rows included)
    o_o, lse_o = oracle.attn(op, as_u16(x.q)[:, None], as_u16(x.k), as_u16(x.v), idx_gn, lens=lens_np)
    compare_attention(o_g.float().cpu().numpy(), o_o[:, 0], lse_g.cpu().numpy(), lse_o[:, :, 0])


# ------------------------------------------------------- chunked / ragged prefill

def run_chunk_case(B, Lmax, Hq, Hkv, topk, kv_lens, q_lens, Lq, seed):
    """Whole chunk path on the GPU (compress the caches, select, attend) against the oracle,
    sequence by sequence.  Cache rows past kv_lens[b] and query rows past q_lens[b] hold
    NaN: nothing of them may reach the outputs, and padding rows must stay unwritten."""
    x = inputs(B, Lmax, Hq, Hkv, seed=seed)  # prefill-shaped: q [B, Lmax, Hq, d]
    q = x.q[:, :Lq].clone()
    k, v = x.k.clone(), x.v.clone()
    for b in range(B):
        k[b, :, kv_lens[b]:] = float("nan")
        v[b, :, kv_lens[b]:] = float("nan")
        q[b, q_lens[b]:] = float("nan")
    p = ops.Params(B, Hq, Hkv, topk=topk)
    ql = torch.tensor(q_lens, dtype=torch.int32).cuda()
    kl = torch.tensor(kv_lens, dtype=torch.int32).cuda()
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kc = ops.compress_keys(p, kd, lens=kl)
    idx = torch.full((B, Hkv, Lq, topk), -7, dtype=torch.int32, device="cuda")
    ops.select_blocks_chunk(p, qd, kc, Lmax, q_lens=ql, kv_lens=kl, out=idx)
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((B, Hq, Lq), 7.0, dtype=torch.float32, device="cuda")
    ops.sparse_attn_chunk(p, qd, kd, vd, idx, q_lens=ql, kv_lens=kl, out=o, lse=lse)
    torch.cuda.synchronize()
    idx, o, lse = idx.cpu().numpy(), o.float().cpu().numpy(), lse.cpu().numpy()
    op1 = oparams(ops.Params(1, Hq, Hkv, topk=topk))
    n_tie = 0
    for b in range(B):
        n, m = kv_lens[b], q_lens[b]
        assert np.all(idx[b, :, m:] == -7), "padding rows of block_idx written"
        assert np.all(np.isnan(o[b, m:])) and np.all(lse[b, :, m:] == 7.0), "padding rows of o / lse written"
        if m == 0:
            continue
        kb = as_u16(x.k[b:b + 1])  # the oracle reads only the first n rows
        kc_o = oracle.compress(op1, kb, lens=np.array([n], np.int32))
        idx_o, sc = oracle.select(op1, as_u16(x.q[b:b + 1, :m]), kc_o, lens=np.array([n], np.int32), Lmax=Lmax,
                                  want_scores=True)
        pos = np.arange(n - m, n)[None]
        _, nt = compare_selection(idx[b:b + 1, :, :m], idx_o, sc, pos, p)
        n_tie += nt
        o_o, lse_o = oracle.attn(op1, as_u16(x.q[b:b + 1, :m]), kb, as_u16(x.v[b:b + 1]), idx[b:b + 1, :, :m],
                                 lens=np.array([n], np.int32))
        compare_attention(o[b:b + 1, :m], o_o, lse[b:b + 1, :, :m], lse_o)
    report_ties(f"chunk B={B} G={Hq // Hkv}", n_tie, int(sum(q_lens)) * Hkv)


@pytest.mark.parametrize("Hq,Hkv", [(32, 2), (8, 1)])
def test_chunk_against_a_longer_cache(Hq, Hkv):
    # one sequence: a 700-query chunk at the end of a 5000-token cache (query row r at
    # position 4300 + r), cache length not a multiple of 64
    run_chunk_case(1, 5000, Hq, Hkv, 16, [5000], [700], 700, seed=1000 + Hq)


@pytest.mark.parametrize("Hq,Hkv", [(32, 2), (8, 1)])
def test_chunk_ragged_batch(Hq, Hkv):
    # ragged batch: chunk and cache lengths differ per sequence (a whole fresh prefill, a
    # chunk ending mid-block, a short chunk, an empty chunk), padded to Lq = 1200
    run_chunk_case(4, 3000, Hq, Hkv, 16, [3000, 1200, 100, 700], [500, 1200, 17, 0], 1200, seed=1100 + Hq)


def test_chunk_rows_equal_the_same_rows_of_a_full_prefill():
    # the last 300 queries as a chunk give bit-identical block lists, and the same outputs
    # up to the fp32 summation order, as the same rows of a full prefill of the sequence
    # (a persistent CTA splits an item's block pairs between its two softmax warpgroups by
    # the parity of its running pair count, which depends on the items it ran before)
    B, L, Hq, Hkv, topk, m = 1, 4100, 32, 2, 16, 300
    x = inputs(B, L, Hq, Hkv, seed=1200)
    p = ops.Params(B, Hq, Hkv, topk=topk)
    q, k, v = x.q.cuda(), x.k.cuda(), x.v.cuda()
    o_f, lse_f, idx_f, kc = ops.prefill(p, q, k, v)
    o_c, lse_c, idx_c = ops.prefill_chunk(p, q[:, L - m:].contiguous(), k, v, kc)
    assert torch.equal(idx_c, idx_f[:, :, L - m:])
    assert float((o_c.float() - o_f[:, L - m:].float()).abs().max()) <= 1e-2
    assert float((lse_c - lse_f[:, :, L - m:]).abs().max()) <= 1e-5


# ------------------------------------------------------------------ backward

BWD_CASES = [
    # B, L, Hq, Hkv, topk
    (1, 1300, 32, 2, 16),  # G = 16, ragged tail (1300 % 64 = 20)
    (2, 1000, 8, 1, 6),    # G = 8, two sequences
    (1, 700, 4, 2, 5),     # G = 2
    (1, 330, 16, 1, 8),    # every visible block selected: dense causal attention
]


@pytest.mark.parametrize("B,L,Hq,Hkv,topk", BWD_CASES)
def test_attn_backward_matches_oracle(B, L, Hq, Hkv, topk):
    # the backward in isolation, on the oracle's inputs: block lists, forward output (as
    # bf16, the form the backward takes it in) and log-sum-exp (as fp32) from the oracle;
    # the oracle forms sum_u P_u dP_u from that same output
    x = inputs(B, L, Hq, Hkv, seed=1300 + L)
    p = ops.Params(B, Hq, Hkv, topk=topk)
    op = oparams(p)
    idx = oracle.select(op, as_u16(x.q), oracle.compress(op, as_u16(x.k)))  # fixed lists, every row
    o_ex, lse_ex = oracle.attn(op, as_u16(x.q), as_u16(x.k), as_u16(x.v), idx)
    o_b = oracle.bf16_round(o_ex)
    g = torch.Generator().manual_seed(1400 + L)
    d_o = torch.randn(x.q.shape, generator=g).to(torch.bfloat16)
    q, k, v, idx_t = x.q.cuda(), x.k.cuda(), x.v.cuda(), torch.from_numpy(idx).cuda()
    o = torch.from_numpy(o_b.view(np.int16)).view(torch.bfloat16).cuda()
    lse = torch.from_numpy(lse_ex.astype(np.float32)).cuda()
    dq, dk, dv = ops.sparse_attn_backward(p, q, k, v, o, lse, d_o.cuda(), idx_t)
    torch.cuda.synchronize()
    rq, rk, rv = oracle.attn_backward(op, as_u16(x.q), as_u16(x.k), as_u16(x.v), idx, as_u16(d_o),
                                      o=bf16_to_f64(o_b))
    errs = [compare_grad(dq, rq, "dq"), compare_grad(dk, rk, "dk"), compare_grad(dv, rv, "dv")]
    warnings.warn(f"backward B={B} L={L} G={Hq // Hkv}: (max, mean) error / row RMS for dq, dk, dv: "
                  + ", ".join(f"({a:.2e}, {b:.2e})" for a, b in errs), UserWarning)
    # dq is computed per query row without atomics: repeated runs agree bit for bit
    dq2, dk2, dv2 = ops.sparse_attn_backward(p, q, k, v, o, lse, d_o.cuda(), idx_t)
    assert torch.equal(dq2, dq)
    assert float((dk2.float() - dk.float()).abs().max()) <= 1e-2 * float(dk.float().abs().max())


# ------------------------------------------------------------ decode cache append

def test_append_kv_matches_a_full_compression():
    # one appended token per sequence: lengths chosen so that the new token completes
    # kernel 0 (n = 32), kernel 1 (n = 48), kernel 2 (n = 64), the last kernel of the
    # cache (n = Lmax), or no kernel (n = 1, 40)
    Lmax = 4096
    lens0 = [0, 31, 47, 63, 4095, 39]
    B, Hq, Hkv = len(lens0), 32, 2
    x = inputs(B, Lmax, Hq, Hkv, seed=900, mode="decode", lens=lens0)
    new = inputs(B, 1, Hq, Hkv, seed=901, mode="prefill")  # k, v [B, Hkv, 1, d]: the appended rows
    p = ops.Params(B, Hq, Hkv, topk=16)
    op = oparams(p)
    k, v, ln = x.k.clone().cuda(), x.v.clone().cuda(), x.lens.cuda()
    kc = ops.compress_keys(p, k, lens=ln)
    ops.append_kv(p, new.k[:, :, 0].contiguous().cuda(), new.v[:, :, 0].contiguous().cuda(), k, v, ln, kc)
    lens1 = [n + 1 for n in lens0]
    assert ln.cpu().tolist() == lens1
    k_ref, v_ref = x.k.clone(), x.v.clone()
    for b, n in enumerate(lens0):
        k_ref[b, :, n] = new.k[b, :, 0]
        v_ref[b, :, n] = new.v[b, :, 0]
    assert torch.equal(k.cpu(), k_ref) and torch.equal(v.cpu(), v_ref)
    kc_o = oracle.compress(op, as_u16(k_ref), lens=np.array(lens1, np.int32))
    for b, n in enumerate(lens1):
        nk = oracle.num_kernels(op, n)
        assert np.array_equal(u16(kc)[b, :, :nk], kc_o[b, :, :nk]), b
    assert ops.device_error(clear=True) == 0


def test_append_kv_over_many_steps_then_decode():
    # 40 decode steps on a 20-token sequence (kernels complete at 32, 48) and a longer one;
    # after the appends the caches, kernels and one decode step match the oracle
    Lmax = 256
    lens0 = [20, 150]
    B, Hq, Hkv, steps = len(lens0), 16, 1, 40
    x = inputs(B, Lmax, Hq, Hkv, seed=910, mode="decode", lens=lens0)
    new = inputs(B, steps, Hq, Hkv, seed=911, mode="prefill")  # row s of k/v: the token of step s
    p = ops.Params(B, Hq, Hkv, topk=4)
    op = oparams(p)
    k, v, ln = x.k.clone().cuda(), x.v.clone().cuda(), x.lens.cuda()
    kc = ops.compress_keys(p, k, lens=ln)
    nk_, nv_ = new.k.cuda(), new.v.cuda()
    for s in range(steps):
        ops.append_kv(p, nk_[:, :, s].contiguous(), nv_[:, :, s].contiguous(), k, v, ln, kc)
    lens1 = [n + steps for n in lens0]
    assert ln.cpu().tolist() == lens1
    k_ref, v_ref = x.k.clone(), x.v.clone()
    for b, n in enumerate(lens0):
        k_ref[b, :, n:n + steps] = new.k[b, :, :steps]
        v_ref[b, :, n:n + steps] = new.v[b, :, :steps]
    assert torch.equal(k.cpu(), k_ref) and torch.equal(v.cpu(), v_ref)
    lens_np = np.array(lens1, np.int32)
    kc_o = oracle.compress(op, as_u16(k_ref), lens=lens_np)
    for b, n in enumerate(lens1):
        nk = oracle.num_kernels(op, n)
        assert np.array_equal(u16(kc)[b, :, :nk], kc_o[b, :, :nk]), b
    o_g, lse_g, idx_g = ops.decode(p, x.q.cuda(), k, v, kc, ln, Lmax)
    idx_o, sc = oracle.select(op, as_u16(x.q)[:, None], kc_o, lens=lens_np, Lmax=Lmax, want_scores=True)
    compare_selection(idx_g.cpu().numpy(), idx_o, sc, (lens_np - 1)[:, None], p)
    o_o, lse_o = oracle.attn(op, as_u16(x.q)[:, None], as_u16(k_ref), as_u16(v_ref), idx_g.cpu().numpy(),
                             lens=lens_np)
    compare_attention(o_g.float().cpu().numpy(), o_o[:, 0], lse_g.cpu().numpy(), lse_o[:, :, 0])
    assert ops.device_error(clear=True) == 0


def test_append_kv_into_a_full_cache_is_refused_on_the_gpu():
    Lmax = 128
    B, Hq, Hkv = 2, 16, 1
    x = inputs(B, Lmax, Hq, Hkv, seed=920, mode="decode", lens=[128, 5])
    p = ops.Params(B, Hq, Hkv, topk=4)
    k, v, ln = x.k.clone().cuda(), x.v.clone().cuda(), x.lens.cuda()
    kc = ops.compress_keys(p, k, lens=ln)
    kc0 = kc.clone()
    kn = torch.zeros((B, Hkv, 128), dtype=torch.bfloat16, device="cuda")
    assert ops.device_error(clear=True) == 0
    ops.append_kv(p, kn, kn, k, v, ln, kc)
    err = ops.device_error(clear=True)
    assert err == 2, err  # INFLLMV2_DEVERR_CACHE_FULL, set by the full sequence only
    assert ln.cpu().tolist() == [128, 6]  # the full one untouched, the other appended
    assert torch.equal(k[0].cpu(), x.k[0]) and torch.equal(kc[0], kc0[0])
    assert torch.equal(k[1, :, 5].cpu(), torch.zeros((Hkv, 128), dtype=torch.bfloat16))
