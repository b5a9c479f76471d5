"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): each rank
takes its own slice of the global batch (weak scaling, no data exchange), and
the timing reduction is the max over ranks."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, _ = bench.dist_init()
    assert (r, w) == (rank, world)
    base, gw, lens = bench.rank_workload(rank, world)
    t = bench.max_over_ranks(10.0 + rank, world, "cpu")
    bench.barrier(world)
    np.save(os.path.join(out_dir, f"r{rank}.npy"), np.concatenate([lens, [t]]))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_ranks_shard_batch_and_reduce_max(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r0, r1 = (np.load(tmp_path / f"r{r}.npy") for r in range(world))
    import duo_workloads as W
    base = W.WORKLOADS["gqa128k"]
    full = W.context_lengths(W.scaled(base, batch=base.batch * world))
    # rank r holds sequences 8r .. 8r+7 of the global batch; per-GPU work is fixed
    assert np.array_equal(r0[:-1], full[:8]) and np.array_equal(r1[:-1], full[8:])
    # the single-GPU workload is rank 0's slice
    assert np.array_equal(r0[:-1], W.context_lengths(base))
    assert r0[-1] == r1[-1] == 11.0


def _split_rank_main(rank, world, port, out_dir):
    """One rank of a sequence split: attention (oracle, CPU) over its slice
    of the history, partials all-gathered with the library's helper."""
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo")
    from head_wise_kv_b200 import seqsplit
    from oracle import duo_oracle as O
    rng = np.random.default_rng(9)
    T, d, cap = 300, 16, 160
    k = rng.standard_normal((T, d))
    v = rng.standard_normal((T, d))
    q = rng.standard_normal(d)
    lo, hi = seqsplit.slice_bounds(cap, rank)
    rows = int(seqsplit.local_rows(torch.tensor([T], dtype=torch.int32), cap, rank)[0])
    assert (lo, rows) == ((0, 160) if rank == 0 else (160, 140))
    o, l = O.attend(q, k[lo:lo + rows], v[lo:lo + rows], 0.3)
    outs, lses = seqsplit.gather_partials(torch.tensor(o, dtype=torch.float32),
                                          torch.tensor([l], dtype=torch.float32))
    np.save(os.path.join(out_dir, f"s{rank}.npy"),
            np.concatenate([outs.numpy().ravel(), lses.numpy().ravel()]))
    dist.destroy_process_group()


def test_sequence_split_partials_gather_to_every_rank(tmp_path):
    world = 2
    mp.start_processes(_split_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    a, b = (np.load(tmp_path / f"s{r}.npy") for r in range(world))
    assert np.array_equal(a, b)                       # every rank holds every partial
    d = 16
    outs, lses = a[:2 * d].reshape(2, d), a[2 * d:]
    from oracle import duo_oracle as O
    rng = np.random.default_rng(9)
    k, v, q = rng.standard_normal((300, d)), rng.standard_normal((300, d)), rng.standard_normal(d)
    full, _ = O.attend(q, k, v, 0.3)
    wts = np.exp(lses - np.logaddexp(lses[0], lses[1]))
    np.testing.assert_allclose(wts @ outs, full, rtol=1e-5, atol=1e-6)


def test_slices_partition_every_sequence_exactly():
    """R slices of `cap` rows: each sequence's first L positions are covered
    once, slice r holding [r cap, r cap + rows_r) with 0 <= rows_r <= cap."""
    import torch
    from head_wise_kv_b200 import seqsplit
    rng = np.random.default_rng(5)
    for R, cap in [(2, 160), (3, 1100), (4, 1)]:
        L = torch.tensor(rng.integers(0, R * cap + 1, size=7), dtype=torch.int32)
        held = [seqsplit.local_rows(L, cap, r) for r in range(R)]
        assert torch.equal(sum(h.to(torch.int64) for h in held), L.to(torch.int64))
        for r, h in enumerate(held):
            lo, hi = seqsplit.slice_bounds(cap, r)
            assert (lo, hi) == (r * cap, (r + 1) * cap)
            assert bool(((h >= 0) & (h <= cap)).all())
            # a slice holds rows only once every earlier slice is full
            assert bool(((h == 0) | (L >= lo)).all())
