"""The multi-GPU host logic of bench.py on two gloo ranks (CPU, no GPU).

The ranks hold parts of one problem: batch rows (weak scaling) or heads (strong scaling).  No data
crosses between ranks; the only collective is the max of the per-rank step times.  Each rank
computes its part with the oracle under the shard's Philox offsets, the parts are gathered here
(test-only), and the whole must equal the oracle run of the whole problem: sharding changes no
decision and no output.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


# the whole problems: tiny fp32 Thinformer with 2 batch rows x 2 heads, and a short Express one
_WHOLE = {
    "thin": W.WORKLOADS["tiny"].with_(B=2, H=2),
    "express": W.Workload("xs", 1, 2, 700, 700, 32, 32, "fp32", True, 1, 7, 5, "rope", n_exact=64, batch=128),
}


def _oracle_part(w, shard):
    from oracle import express, thinformer
    q, k, v = shard.inputs(w)
    kw = dict(heads=(shard.H_total, shard.heads), b0=shard.b0)
    if w.causal:
        return express(q, k, v, w.n_exact, w.batch, w.g, w.seed, **kw)
    return thinformer(q, k, v, w.g, w.seed, **kw)


def _rank(rank, world, port, q, name, mode):
    import datetime
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        whole = _WHOLE[name]
        whole = whole.with_(B=whole.B // world) if mode == "batch" else whole
        sh = bench.Shard(whole, world, rank, mode)
        part = _oracle_part(sh.local, sh)
        out = torch.from_numpy(np.ascontiguousarray(part.out))
        parts = [torch.empty_like(out) for _ in range(world)]
        dist.all_gather(parts, out)                      # test-only: compare the whole on rank 0
        ms = bench.max_over_ranks([2.0, 3.5][rank], dist, torch.device("cpu"))
        q.put((rank, sh.b0, sh.h0, sh.local.B, sh.local.H, sh.scaling, sh.whole_tokens, ms,
               [p.numpy() for p in parts] if rank == 0 else None))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(name, mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q, name, mode)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(2)), key=lambda r: r[0])
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs)
    return res


@pytest.mark.parametrize("name,mode", [("thin", "batch"), ("thin", "heads"), ("express", "heads")])
def test_two_rank_shards_reproduce_the_whole_problem(name, mode):
    from oracle import express, thinformer
    res = _run(name, mode)
    whole = _WHOLE[name]
    assert all(r[7] == 3.5 for r in res)                 # the slowest rank bounds the job
    if mode == "batch":
        assert [(r[1], r[2], r[3], r[4]) for r in res] == [(0, 0, 1, 2), (1, 0, 1, 2)]
        assert {r[5] for r in res} == {"weak"}
        assert all(r[6] == whole.B * whole.H * whole.T for r in res)
    else:
        assert [(r[1], r[2], r[3], r[4]) for r in res] == [(0, 0, whole.B, 1), (0, 1, whole.B, 1)]
        assert {r[5] for r in res} == {"strong"}
    q, k, v = W.make_qkv(whole)
    ref = (express(q, k, v, whole.n_exact, whole.batch, whole.g, whole.seed) if whole.causal
           else thinformer(q, k, v, whole.g, whole.seed))
    got = np.concatenate(res[0][8], axis=0 if mode == "batch" else 2)
    np.testing.assert_array_equal(got, ref.out)


def test_philox_offsets_matter():
    """A shard that forgot its offset draws another stream: some decision differs."""
    from oracle import thinformer
    w = _WHOLE["thin"]
    q, k, v = W.make_qkv(w)
    whole = thinformer(q, k, v, w.g, w.seed)
    q1, k1, v1 = q[1:], k[1:], v[1:]
    right = thinformer(q1, k1, v1, w.g, w.seed, heads=(w.H, [0, 1]), b0=1)
    wrong = thinformer(q1, k1, v1, w.g, w.seed)
    np.testing.assert_array_equal(right.coreset, whole.coreset[1:])
    assert not np.array_equal(wrong.coreset, whole.coreset[1:])


def test_single_process_needs_no_collective():
    import bench
    assert bench.max_over_ranks(4.25, None, torch.device("cpu")) == 4.25
    sh = bench.Shard(W.WORKLOADS["express32k"], 1, 0)
    assert sh.abi == (0, 0, 32) and sh.local == W.WORKLOADS["express32k"] and sh.scaling == "weak"
    with pytest.raises(ValueError):
        bench.Shard(W.WORKLOADS["express32k"], 3, 0, "heads")


def _rank_seq(rank, world, port, q, name):
    import datetime
    import bench
    from oracle import express, thinformer
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = _WHOLE[name]
        sh = bench.Shard(w, world, rank, "seq")
        q0, q1 = sh.q_range
        qq, kk, vv = sh.inputs(sh.local)
        rows = list(range(q0, q1))
        part = (express(qq, kk, vv, w.n_exact, w.batch, w.g, w.seed, rows=rows) if w.causal
                else thinformer(qq, kk, vv, w.g, w.seed, rows=rows))
        ms = bench.max_over_ranks([2.0, 3.5][rank], dist, torch.device("cpu"))
        q.put((rank, sh.q_range, sh.abi, sh.local.H, sh.scaling, sh.parallelism, sh.whole_tokens, ms, part.out))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", ["thin", "express"])
def test_two_rank_sequence_shards_reproduce_the_whole_problem(name):
    """--shard seq: each rank holds every head and attends a 128-aligned slice of the query rows
    (the last ending at T); the slices partition [0, T) and the stacked rows equal the whole run's
    (the oracle evaluates a subset of rows with other BLAS blocking: equal to 1e-12)."""
    from oracle import express, thinformer
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_seq, args=(r, 2, port, qu, name)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((qu.get(timeout=300) for _ in range(2)), key=lambda r: r[0])
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs)
    whole = _WHOLE[name]
    ranges = [r[1] for r in res]
    assert ranges[0][0] == 0 and ranges[0][1] == ranges[1][0] and ranges[1][1] == whole.T
    assert ranges[0][1] % 128 == 0
    assert all(r[2] == (0, 0, whole.H) and r[3] == whole.H for r in res)
    assert {r[4] for r in res} == {"strong"} and {r[5] for r in res} == {"sp2"}
    assert all(r[6] == whole.B * whole.H * whole.T and r[7] == 3.5 for r in res)
    q, k, v = W.make_qkv(whole)
    ref = (express(q, k, v, whole.n_exact, whole.batch, whole.g, whole.seed) if whole.causal
           else thinformer(q, k, v, whole.g, whole.seed))
    np.testing.assert_allclose(np.concatenate([r[8] for r in res], axis=1), ref.out, rtol=0, atol=1e-12)


def test_sequence_shard_needs_rows_for_every_rank():
    import bench
    with pytest.raises(ValueError):
        bench.Shard(W.WORKLOADS["tiny"], 3, 0, "seq")        # T = 256 < 3 x 128
    sh = bench.Shard(W.WORKLOADS["express32k"], 8, 7, "seq")
    assert sh.q_range == (28672, 32768) and sh.rows == (28672, 32768)


class _FakeNodes:
    """A stand-in for a thin_split handle's batch coresets on the CPU: n_b blocks of bpb bytes, the
    owned ones filled by 'phase 1' with a pattern of (batch, byte), the others zero until imported."""

    def __init__(self, k0, k1, n_b, bpb):
        self.k0, self.k1, self.n_b, self.bpb = k0, k1, n_b, bpb
        self.device = torch.device("cpu")
        self.blocks = torch.zeros(n_b, bpb, dtype=torch.uint8)
        for kk in range(k0, k1):
            self.blocks[kk] = (torch.arange(bpb) * 7 + kk * 13) % 251

    def nodes_layout(self, g=2):
        return self.k0, self.k1, self.n_b, self.bpb

    def nodes_export(self, dst, g=2):
        dst[:(self.k1 - self.k0) * self.bpb] = self.blocks[self.k0:self.k1].reshape(-1)

    def nodes_import(self, src, a, b, g=2):
        self.blocks[a:b] = src[:(b - a) * self.bpb].reshape(b - a, self.bpb)


def _rank_exchange(rank, world, port, q, owned):
    import datetime
    import thinned_softmax_attention_b200 as TA
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        k0, k1 = owned[rank]
        h = _FakeNodes(k0, k1, owned[-1][1], 96)
        TA.exchange_batch_coresets(h, 2, dist)
        q.put((rank, h.blocks.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("owned", [[(0, 3), (3, 7)], [(0, 0), (0, 4), (4, 5)]])
def test_batch_coreset_exchange_over_ranks(owned):
    """exchange_batch_coresets on gloo ranks (the thin_split handles replaced by CPU stand-ins with the
    same three calls): after the all-gather every rank holds every batch's block, each from the rank
    that owns it -- unequal ownership (padding) and a rank owning no batch included."""
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    world = len(owned)
    procs = [ctx.Process(target=_rank_exchange, args=(r, world, port, qu, owned)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qu.get(timeout=300) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs)
    n_b, bpb = owned[-1][1], 96
    want = np.stack([((np.arange(bpb) * 7 + kk * 13) % 251).astype(np.uint8) for kk in range(n_b)])
    for _, blocks in res:
        np.testing.assert_array_equal(blocks, want)
