"""Host-side multi-process path of the benchmark (one process per GPU), run as two gloo
ranks on CPU: per-rank inputs differ, the job time is the slowest rank's, the rate
counts every rank's units, and the barrier really waits for the late rank.  A second
test runs the method itself on every rank's shard (the CPU oracle stands in for the
GPU path here) and checks that the shards are independent: each rank's results equal a
single-process run on that rank's inputs."""
import os
import socket
import time

import pytest
import torch
import torch.multiprocessing as mp

from trainable_block_sparse_compress_b200 import dist
from trainable_block_sparse_compress_b200.synthetic import Workload, make_inputs


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        ri = dist.rank_info()
        assert (ri.rank, ri.world, ri.local) == (rank, world, rank)
        wl = Workload("tiny", "decode", 2, 256, 4, 1, 4, ragged=(100, 256))
        x = make_inputs(wl, seed=dist.rank_seed(7, ri.rank))
        # the timed-region protocol: barrier, "work" of a rank-dependent length, barrier
        dist.barrier(world)
        t0 = time.perf_counter()
        time.sleep(0.05 + 0.15 * rank)
        own = time.perf_counter() - t0
        dist.barrier(world)
        after = time.perf_counter() - t0  # the barrier held every rank until the slowest finished
        slowest = dist.max_over_ranks(own, world)
        rate = dist.weak_scaling_rate(world, 1000.0, 3, slowest)
        out[rank] = (float(x.q.float().sum()), int(x.lens.sum()), own, after, slowest, rate)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_shard_and_time_like_the_benchmark():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    (q0, l0, own0, after0, slow0, rate0), (q1, l1, own1, after1, slow1, rate1) = res[0], res[1]
    assert q0 != q1 and l0 != l1  # each rank draws its own sequences
    assert own1 > own0
    assert slow0 == slow1 == pytest.approx(max(own0, own1))  # every rank reports the slowest time
    assert after0 >= own1 - 0.02  # rank 0 waited at the barrier for rank 1
    assert rate0 == rate1 == pytest.approx(world * 1000.0 * 3 / max(own0, own1))


def test_single_process_needs_no_process_group():
    assert not torch.distributed.is_initialized()
    assert dist.max_over_ranks(1.5, 1) == 1.5
    dist.barrier(1)
    assert dist.weak_scaling_rate(1, 10.0, 2, 4.0) == 5.0
    assert dist.rank_seed(3, 0) != dist.rank_seed(3, 1)


def _method_digest(rank_seed):
    """compress -> select -> attend of one rank's decode shard with the oracle: a digest
    of the block lists, outputs and log-sum-exps."""
    import hashlib

    import numpy as np

    import oracle
    from trainable_block_sparse_compress_b200.synthetic import as_u16
    wl = Workload("tiny", "decode", 3, 512, 16, 2, 6, ragged=(70, 512))
    x = make_inputs(wl, seed=rank_seed)
    op = oracle.Params(wl.batch, wl.num_q_heads, wl.num_kv_heads, 128, 64, 32, 16, wl.topk, 1, 2, 0.0, 0, 0)
    lens = x.lens.numpy().astype(np.int32)
    kc = oracle.compress(op, as_u16(x.k), lens=lens)
    idx = oracle.select(op, as_u16(x.q)[:, None], kc, lens=lens, Lmax=wl.seq_len)
    o, lse = oracle.attn(op, as_u16(x.q)[:, None], as_u16(x.k), as_u16(x.v), idx, lens=lens)
    return hashlib.sha256(idx.tobytes()).hexdigest(), float(np.asarray(o).sum()), float(np.asarray(lse).sum()), \
        int(lens.sum())


def _method_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    try:
        ri = dist.rank_info()
        dist.barrier(world)
        t0 = time.perf_counter()
        digest = _method_digest(dist.rank_seed(11, ri.rank))
        own = time.perf_counter() - t0
        dist.barrier(world)
        slowest = dist.max_over_ranks(own, world)
        gathered = [None] * world
        torch.distributed.all_gather_object(gathered, digest)
        out[rank] = (gathered, own, slowest)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_run_independent_shards_of_the_method():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_method_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    g0, own0, slow0 = res[0]
    g1, own1, slow1 = res[1]
    assert g0 == g1  # every rank holds every rank's digest
    assert g0[0] != g0[1]  # the shards differ
    for r in range(world):  # and each equals a single-process run of that rank's inputs
        assert tuple(g0[r]) == _method_digest(dist.rank_seed(11, r))
    assert slow0 == slow1 == pytest.approx(max(own0, own1))
