"""Multi-rank host logic on CPU (gloo, world size 2): each rank builds its own
independent cache shard, the step time is the max over ranks, and the
whole-job throughput counts every rank's keys.  No data-path collective exists."""
import hashlib
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
import synth
from tests import harness as H


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        base = synth.WORKLOADS["single_layer_4k"].with_(seq_len=(300, 300), n_calib=8)
        wl = bench.rank_workload(base, rank, 64)
        cache = synth.make_contig(wl, "cpu")
        digest = hashlib.sha256(H.bits16(cache.K).tobytes()).hexdigest()
        # stand-in for the rank's step: the oracle on its own rows (no GPU here)
        cs, ms = H.oracle_calibration(cache.qcal)
        Kf = H.to_f64(cache.K)
        r = 0
        a, b = cache.row_off_np[r], cache.row_off_np[r + 1]
        s = oracle.row_scores(wl.theta, cs[0], ms[0], 0, wl.group, Kf[a:b],
                              cache.pos[a:b].numpy().astype(np.int64), True, 300, wl.offsets)
        kept = oracle.select(s, 64, wl.window)
        my_ms = 10.0 + 5.0 * rank
        slow = bench.max_over_ranks(my_ms, world, "cpu")
        digests = [None] * world
        dist.all_gather_object(digests, digest)
        out[rank] = (slow, bench.throughput(cache.total, world, slow), digests, len(kept), cache.total)
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_time_max():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        ctx = mp.get_context("spawn")
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
            assert p.exitcode == 0
        res = dict(out)
    assert set(res) == {0, 1}
    for r in range(world):
        slow, value, digests, nkept, total = res[r]
        assert slow == 15.0  # the slower rank's time on every rank
        assert value == total * world / 0.015
        assert digests[0] != digests[1]  # independent shards
        assert nkept == 64
