"""Multi-rank host logic of the bench on CPU (gloo, world size 2).

The op shards with no data-path exchange: each rank runs its own batch
(weak scaling). What needs ranks is the plumbing: distinct per-rank inputs,
the max-over-ranks timing reduction and the whole-job aggregate.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import workloads
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = workloads.WORKLOADS["tiny"]
        seed = bench.rank_seed(w, rank)
        inp = workloads.make_inputs(w, seed=seed)
        mine = [1.0 + rank, 10.0 - rank, 5.0]
        got = bench.max_over_ranks(mine, world, torch.device("cpu"))
        gathered = [None] * world
        dist.all_gather_object(gathered, (seed, float(inp.q.sum())))
        out[rank] = (got, gathered)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    for rank in range(world):
        got, gathered = out[rank]
        assert got == [2.0, 10.0, 5.0]          # element-wise max over ranks
        seeds = [g[0] for g in gathered]
        assert len(set(seeds)) == world          # every rank draws its own batch
        assert gathered[0][1] != gathered[1][1]


def test_aggregate_is_whole_job():
    import bench
    assert bench.aggregate_tokens_per_s(4, 1000, 2.0) == pytest.approx(2_000_000.0)
    assert bench.max_over_ranks([1.5, 2.5], 1, torch.device("cpu")) == [1.5, 2.5]


def _lw_worker(rank, world, port, out):
    """One rank of a layerwise (all-heads) QK-norm under tensor parallelism:
    it holds a slice of the heads, sums squares over its slice, and the
    binding's exchange sums the per-token partials over the group."""
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import numpy as np
    import workloads
    import qk_rmsnorm_rope_norm_b200 as qknr
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp = workloads.make_inputs("tiny", seed=21, Hq=4, Hkv=2)
        w = inp.w
        hq, hk = w.Hq // world, w.Hkv // world
        q = inp.q[:, :, rank * hq:(rank + 1) * hq].double().numpy()
        k = inp.k[:, :, rank * hk:(rank + 1) * hk].double().numpy()
        sq = torch.from_numpy((q ** 2).sum(axis=(2, 3)).reshape(-1).astype(np.float32))
        sk = torch.from_numpy((k ** 2).sum(axis=(2, 3)).reshape(-1).astype(np.float32))
        qknr.all_reduce_stats([sq, sk], dist.group.WORLD)
        totals = qknr._totals(hq, hk, None, None, dist.group.WORLD)
        out[rank] = (sq.numpy().tolist(), sk.numpy().tolist(), totals)
    finally:
        dist.destroy_process_group()


def test_layerwise_stats_exchange_two_gloo_ranks():
    import numpy as np
    import oracle
    import workloads
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_lw_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    inp = workloads.make_inputs("tiny", seed=21, Hq=4, Hkv=2)
    w = inp.w
    T = w.B * w.S
    m = oracle.positions(None, w.B, w.S)
    for rank in range(world):
        sq, sk, totals = out[rank]
        assert totals == (w.Hq, w.Hkv)
        # the exchanged statistic gives the oracle's full-hidden inverse RMS
        for s, x, H in ((sq, inp.q, w.Hq), (sk, inp.k, w.Hkv)):
            _, r = oracle.get().lw_fwd(x.reshape(T, H, w.D), np.ones(H * w.D), m, 0, w.theta,
                                       w.eps)
            got = 1.0 / np.sqrt(np.asarray(s, np.float64) / (H * w.D) + w.eps)
            assert np.abs(got / r - 1).max() <= H * w.D * 2.0 ** -24
    assert out[0][0] == out[1][0] and out[0][1] == out[1][1]


def test_layerwise_exchange_without_group_is_identity():
    import qk_rmsnorm_rope_norm_b200 as qknr
    a, b = torch.arange(4.0), torch.ones(3)
    ra, rb = qknr.all_reduce_stats([a, b], None)
    assert ra is a and rb is b and torch.equal(a, torch.arange(4.0))
    assert qknr._totals(4, 2, None, None, None) == (4, 2)
    assert qknr._totals(4, 2, 16, 8, None) == (16, 8)


def _lw_chunk_worker(rank, world, port, out):
    """One tensor-parallel rank running the binding's chunked exchange
    schedule (``run_chunked``): per chunk, the partial sums of squares over
    its heads, an asynchronous gloo all-reduce of them, and the element-wise
    pass once the sum is in, here restated with the oracle's rotation. The
    schedule's call log is returned with the outputs."""
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import numpy as np
    import oracle
    import workloads
    import qk_rmsnorm_rope_norm_b200 as qknr
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp = workloads.make_inputs("tiny", seed=22, B=2, S=19, Hq=4, Hkv=2)
        w = inp.w
        T = w.B * w.S
        gq, gk = workloads.layerwise_gamma(w, 22)
        hq, hk = w.Hq // world, w.Hkv // world
        x = {"q": inp.q.double().numpy().reshape(T, w.Hq, w.D)[:, rank * hq:(rank + 1) * hq],
             "k": inp.k.double().numpy().reshape(T, w.Hkv, w.D)[:, rank * hk:(rank + 1) * hk]}
        g = {"q": gq.double().numpy()[rank * hq * w.D:(rank + 1) * hq * w.D].reshape(hq, w.D),
             "k": gk.double().numpy()[rank * hk * w.D:(rank + 1) * hk * w.D].reshape(hk, w.D)}
        tot = {"q": w.Hq * w.D, "k": w.Hkv * w.D}
        m = oracle.positions(None, w.B, w.S)
        spans = qknr.token_chunks(T, 4)
        sums, works, log = {}, {}, []
        y = {"q": np.zeros_like(x["q"]), "k": np.zeros_like(x["k"])}

        def partial(i):
            t0, t1 = spans[i]
            sums[i] = torch.from_numpy(np.stack([(x[n][t0:t1] ** 2).sum(axis=(1, 2))
                                                 for n in ("q", "k")]))
            log.append(("partial", i))

        def exchange(i):
            works[i] = dist.all_reduce(sums[i], op=dist.ReduceOp.SUM, async_op=True)
            log.append(("exchange", i))

        def finish(i):
            works[i].wait()
            t0, t1 = spans[i]
            for j, n in enumerate(("q", "k")):
                r = 1.0 / np.sqrt(sums[i][j].numpy() / tot[n] + w.eps)
                nrm = x[n][t0:t1] * r[:, None, None] * g[n][None]
                H = nrm.shape[1]
                rows = nrm.reshape(-1, w.D)
                mm = np.repeat(m[t0:t1], H)
                y[n][t0:t1] = oracle.get().rope_rows(rows, mm, w.rotary_dim,
                                                     w.theta).reshape(nrm.shape)
            log.append(("finish", i))

        qknr.run_chunked(len(spans), partial, exchange, finish)
        out[rank] = (y["q"].tolist(), y["k"].tolist(), log)
    finally:
        dist.destroy_process_group()


def test_layerwise_chunked_exchange_two_gloo_ranks():
    """The chunked exchange schedule over two gloo ranks gives the oracle's
    layerwise forward on the full hidden vector, and each chunk's exchange is
    in flight while the next chunk's partial sums are taken."""
    import numpy as np
    import oracle
    import workloads
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_lw_chunk_worker, args=(world, port, out), nprocs=world,
                       start_method="spawn", join=True)
    inp = workloads.make_inputs("tiny", seed=22, B=2, S=19, Hq=4, Hkv=2)
    w = inp.w
    T = w.B * w.S
    gq, gk = workloads.layerwise_gamma(w, 22)
    m = oracle.positions(None, w.B, w.S)
    ref_q, _ = oracle.get().lw_fwd(inp.q.reshape(T, w.Hq, w.D), gq, m, w.rotary_dim, w.theta,
                                   w.eps)
    ref_k, _ = oracle.get().lw_fwd(inp.k.reshape(T, w.Hkv, w.D), gk, m, w.rotary_dim, w.theta,
                                   w.eps)
    got_q = np.concatenate([np.asarray(out[r][0]) for r in range(world)], axis=1)
    got_k = np.concatenate([np.asarray(out[r][1]) for r in range(world)], axis=1)
    assert np.abs(got_q - ref_q).max() <= 1e-12
    assert np.abs(got_k - ref_k).max() <= 1e-12
    for rank in range(world):
        log = out[rank][2]
        at = {e: n for n, e in enumerate(log)}
        C = len([e for e in log if e[0] == "partial"])
        assert C == 4 and len(log) == 3 * C
        for i in range(C):
            assert at[("partial", i)] < at[("exchange", i)] < at[("finish", i)]
            if i + 1 < C:  # chunk i finishes only after chunk i + 1's partial sums
                assert at[("partial", i + 1)] < at[("finish", i)]


def test_token_chunks_cover_every_token():
    import qk_rmsnorm_rope_norm_b200 as qknr
    for T in (0, 1, 3, 4, 5, 97, 65536):
        for n in (1, 2, 4, 7):
            spans = qknr.token_chunks(T, n)
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert all(t1 > t0 for t0, t1 in spans) or T == 0


def test_chunk_count_rule():
    """A sharded layerwise call is cut into at most `chunks` token runs, each
    of at least MIN_CHUNK_TOKENS tokens and MIN_CHUNK_BYTES of the rank's
    rows, and always at least one."""
    import qk_rmsnorm_rope_norm_b200 as qknr
    row = lambda T, H, D=128, e=2: T * H * D * e
    # every head of the Llama-3-8B and 64k partial-RoPE shapes: byte floor
    # 96 MiB -> 3 and 4 (the cap) chunks
    assert qknr.chunk_count(32768, row(32768, 40), 4) == 3
    assert qknr.chunk_count(65536, row(65536, 40), 4) == 4
    # one TP-8 rank of the Llama-3-8B shape (4 + 1 heads, 42 MB of rows):
    # a single run, the plain stats -> exchange -> normalise sequence
    assert qknr.chunk_count(32768, row(32768, 5), 4) == 1
    # the token floor binds on short calls; both floors off: the cap
    assert qknr.chunk_count(8191, row(8191, 400), 4) == 1
    assert qknr.chunk_count(100, row(100, 5), 7, min_chunk=1, min_chunk_bytes=0) == 7
    assert qknr.chunk_count(3, row(3, 5), 7, min_chunk=1, min_chunk_bytes=0) == 3
    assert qknr.chunk_count(0, 0, 4) == 1
