"""The N > 1 host path of bench.py on CPU: two `gloo` ranks on 127.0.0.1.

With N GPUs every rank quantizes its own independent layer of the same shape
(the path partitions: no data-path collective); the only cross-rank step is
the reduction of the device-timed region to the slowest rank, and the job's
rate counts the units of all ranks.  These tests run that host logic -- the
per-rank data, the max-over-ranks time, the whole-job rate, and the oracle
step on each rank's own layer -- in two processes, without a GPU."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from post_weight_quantization_philox_b200 import synth
        cfg = synth.small_config(16, 256, 32, 0, number=91)
        w_seed, x_seed, philox_seed = bench.layer_seeds(cfg, rank)
        W = synth.make_weight(cfg, seed=w_seed)
        X = synth.make_calib(cfg, seed=x_seed)
        # each rank's own layer, stepped by the oracle on this rank alone
        st = oracle.init(cfg.grid, W, seed=philox_seed)
        Y = oracle.reference_output(W, X)
        loss = oracle.step(st, X, Y, 0.5, 1e-3)
        # a rank-dependent "device time": the job's time is the slowest rank's
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, device="cpu")
        digests = [None] * world
        dist.all_gather_object(digests, (float(W.sum()), float(X.sum()), philox_seed, loss))
        out[rank] = {"ms": ms, "digests": digests,
                     "rate": bench.whole_job_rate(world, cfg.N * cfg.K * 3, ms)}
    finally:
        dist.destroy_process_group()


def _run(world):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return dict(out)


def test_two_ranks_independent_layers_and_max_time(oracle_mod):
    out = _run(2)
    assert sorted(out) == [0, 1]
    # the slowest rank's time on every rank
    assert out[0]["ms"] == out[1]["ms"] == 15.0
    # both ranks saw the same gathered view
    assert out[0]["digests"] == out[1]["digests"]
    (w0, x0, s0, l0), (w1, x1, s1, l1) = out[0]["digests"]
    # each rank has its own data and Philox stream, hence its own loss
    assert w0 != w1 and x0 != x1 and s0 != s1 and l0 != l1
    # whole-job rate: the units of both ranks over the slowest rank's time
    assert out[0]["rate"] == pytest.approx(2 * 16 * 256 * 3 / 0.015)


def _shard_worker(rank, world, port, out):
    """One layer split by rows over the ranks (bench.py --split rows): each
    rank steps its band with the band's global row offset, then the states
    and losses are gathered on rank 0."""
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from post_weight_quantization_philox_b200 import synth
        mode = int(os.environ.get("SHARD_MODE", "0"))
        cfg = synth.small_config(24, 256, 32, mode, number=93)
        W = synth.make_weight(cfg)          # the same layer on every rank
        X = synth.make_calib(cfg)
        r0, n = bench.row_shard(cfg.N, rank, world, align=8)
        st = oracle.init(cfg.grid, W[r0:r0 + n], seed=5, row0=r0)
        Y = oracle.reference_output(W[r0:r0 + n], X)
        losses = [oracle.step(st, X, Y, tau, 1e-3) for tau in (1.0, 0.4, 0.1)]
        got = [None] * world
        dist.all_gather_object(got, (r0, n, st.logits, st.mom, st.s, st.ms, losses))
        out[rank] = got
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_row_shards_reproduce_the_whole_layer(oracle_mod, mode):
    """Two ranks holding rows [0, 8) and [8, 24) of one layer, each keyed by
    its global row offset, end in exactly the whole layer's state for those
    rows, and their losses add up to the layer's loss, step by step."""
    import torch.multiprocessing as mp
    os.environ["SHARD_MODE"] = str(mode)
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    shards = out[0]
    assert [(r0, n) for r0, n, *_ in shards] == [(0, 8), (8, 16)]
    sys.path.insert(0, ROOT)
    import oracle
    from post_weight_quantization_philox_b200 import synth
    cfg = synth.small_config(24, 256, 32, mode, number=93)
    W, X = synth.make_weight(cfg), synth.make_calib(cfg)
    full = oracle.init(cfg.grid, W, seed=5)
    Y = oracle.reference_output(W, X)
    full_losses = [oracle.step(full, X, Y, tau, 1e-3) for tau in (1.0, 0.4, 0.1)]
    for r0, n, logits, mom, s, ms, _ in shards:
        assert np.array_equal(logits, full.logits[:, r0:r0 + n])
        assert np.array_equal(mom, full.mom[:, r0:r0 + n])
        assert np.array_equal(s, full.s[r0:r0 + n])
        assert np.array_equal(ms, full.ms[r0:r0 + n])
    summed = np.sum([sh[6] for sh in shards], axis=0)
    assert np.allclose(summed, full_losses, rtol=1e-12, atol=0)
    # a shard keyed with the wrong offset draws other noise
    wrong = oracle.init(cfg.grid, W[8:24], seed=5, row0=0)
    oracle.step(wrong, X, oracle.reference_output(W[8:24], X), 1.0, 1e-3)
    assert not np.array_equal(wrong.logits, shards[1][2])


def test_row_shard_bounds():
    sys.path.insert(0, ROOT)
    import bench
    for N, world in [(4096, 8), (14336, 8), (8192, 3), (24, 2), (100, 4)]:
        bands = [bench.row_shard(N, r, world) for r in range(world)]
        assert bands[0][0] == 0
        assert sum(n for _, n in bands) == N
        assert all(bands[r][0] + bands[r][1] == bands[r + 1][0] for r in range(world - 1))
    assert [bench.row_shard(4096, r, 8) for r in range(8)] == [(512 * r, 512) for r in range(8)]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(1, 1000, 2.0) == pytest.approx(5e5)
    from post_weight_quantization_philox_b200 import synth
    cfg = synth.CONFIGS["c2_qproj_4096x4096"]
    seeds = {bench.layer_seeds(cfg, r) for r in range(8)}
    assert len(seeds) == 8
    # rank 0's layer is the configuration's own seeded layer
    assert bench.layer_seeds(cfg, 0)[:2] == (1000 + cfg.number, 2000 + cfg.number)
    W0 = synth.make_weight(synth.small_config(8, 128, 8, 0, number=2),
                           seed=bench.layer_seeds(cfg, 0)[0])
    W1 = synth.make_weight(synth.small_config(8, 128, 8, 0, number=2),
                           seed=bench.layer_seeds(cfg, 1)[0])
    assert not np.array_equal(W0, W1)
