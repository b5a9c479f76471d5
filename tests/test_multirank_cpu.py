"""Multi-rank host logic on CPU (gloo, world size 2): in bench.py each rank
takes its own slice of the global batch (weak scaling, no data exchange) and
the timing reduction is the max over ranks; in a sequence split each rank
decodes its slice and the partials are exchanged and merged."""
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


class _OracleSlice:
    """CPU stand-in for one rank's cache in a sequence split: decode_rows
    over the rank's slice of the retrieval history (positions lo .. lo+rows)
    and over ring slots [0, s_len) of the streaming head, computed by the
    oracle.  One sequence; query head 0 reads retrieval KV head 0, query head
    1 streaming KV head 1."""

    def __init__(self, k, v, lo, sink, window):
        self.k, self.v, self.lo, self.sink, self.window = k, v, lo, sink, window
        self.calls = []

    def decode_rows(self, layer, q, rows, scale, s_len=None):
        import torch
        from oracle import duo_oracle as O
        n, ns = int(rows[0]), int(s_len[0])
        self.calls.append((n, ns))
        d = self.k.shape[-1]
        out = np.zeros((1, 2, d))
        lse = np.full((1, 2), -np.inf)
        if n > 0:
            keys = np.arange(self.lo, self.lo + n)
            out[0, 0], lse[0, 0] = O.attend(q[0, 0].numpy(), self.k[0][keys], self.v[0][keys], scale)
        if ns > 0:                              # a full ring holds the key set of position ns - 1
            keys = O.keep_set(ns - 1, self.sink, self.window)
            out[0, 1], lse[0, 1] = O.attend(q[0, 1].numpy(), self.k[1][keys], self.v[1][keys], scale)
        return torch.tensor(out, dtype=torch.float32), torch.tensor(lse, dtype=torch.float32)


def _cpu_lse_merge(parts_out, parts_lse):
    """Log-sum-exp merge of partial attentions (stand-in for the library's
    GPU merge): out = sum_i exp(l_i - L) o_i, L = log sum_i exp(l_i)."""
    import torch
    L = torch.logsumexp(parts_lse.double(), dim=0)
    w = torch.exp(parts_lse.double() - L)
    w = torch.nan_to_num(w, nan=0.0)
    return (w.unsqueeze(-1) * parts_out.double()).sum(0).float(), L.float()


def _split_rank_main(rank, world, port, out_dir):
    """One rank of a sequence split: seqsplit.split_decode_step on the rank's
    slice (oracle stand-in for the cache), partials exchanged over gloo."""
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo")
    from head_wise_kv_b200 import seqsplit
    seqsplit.lse_merge = _cpu_lse_merge
    rng = np.random.default_rng(9)
    T, d, cap, S, Wn = 300, 16, 160, 4, 32
    k = rng.standard_normal((2, T, d))
    v = rng.standard_normal((2, T, d))
    q = torch.tensor(rng.standard_normal((1, 2, d)), dtype=torch.float32)
    lo, _ = seqsplit.slice_bounds(cap, rank)
    cache = _OracleSlice(k, v, lo, S, Wn)
    out, lse = seqsplit.split_decode_step(cache, 0, q, torch.tensor([T], dtype=torch.int32), 0.3, cap, rank,
                                          world)
    # rank 0 reads its 160 rows and no ring slots; the last rank its 140 rows and the ring
    assert cache.calls == ([(160, 0)] if rank == 0 else [(140, T)]), cache.calls
    np.save(os.path.join(out_dir, f"s{rank}.npy"), np.concatenate([out.numpy().ravel(), lse.numpy().ravel()]))
    dist.destroy_process_group()


def test_split_decode_step_over_two_ranks(tmp_path):
    """Both ranks end with the oracle's single-device decode (out and lse)."""
    world = 2
    mp.start_processes(_split_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    a, b = (np.load(tmp_path / f"s{r}.npy") for r in range(world))
    assert np.array_equal(a, b)                       # every rank holds the same merged result
    d = 16
    from oracle import duo_oracle as O
    rng = np.random.default_rng(9)
    k, v = rng.standard_normal((2, 300, d)), rng.standard_normal((2, 300, d))
    q = np.asarray(torch_tensor_f32(rng.standard_normal((1, 2, d))), dtype=np.float64)
    ref, ref_lse = O.decode_attention(q, lambda b_, g: k[g], lambda b_, g: v[g], np.array([300]),
                                      np.array([1, 0], np.uint8), 4, 32, 0.3)
    np.testing.assert_allclose(a[:2 * d].reshape(1, 2, d), ref, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(a[2 * d:].reshape(1, 2), ref_lse, rtol=1e-5, atol=1e-5)


def torch_tensor_f32(x):
    import torch
    return torch.tensor(x, dtype=torch.float32).numpy()


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
