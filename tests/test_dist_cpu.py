"""Multi-process host logic of the replica benchmark, on CPU with gloo.

Two ranks join a process group the way ``bench.py --gpus 2`` does, check that
they draw different batches, that the timing reduction takes the slowest
rank, and that the whole-job rate counts every rank's units.  A rank that
never joins makes the other rank's join fail within its timeout instead of
hanging.
"""
import os
import socket
import time

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.timeout(120)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, ws: int, port: int):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(ws), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))


def _replica_rank(rank, ws, port, out):
    _env(rank, ws, port)
    from mlra_latent_kv_b200 import dist as mdist, synth
    r, w, local = mdist.world()
    assert (r, w, local) == (rank, ws, rank)
    assert mdist.init("gloo", timeout_s=30)
    wl = synth.workload("dsv2_contiguous").with_(B=2, seq_len=70)
    inp = synth.make_inputs(wl.with_(seed=mdist.rank_seed(wl.seed, r)))
    mdist.barrier()
    slowest = mdist.max_over_ranks(1.0 + r)
    rate = mdist.throughput(100.0, w, slowest)
    out[r] = (float(inp["q_nope"].float().sum()), slowest, rate)
    mdist.shutdown()


def test_two_replicas_gloo():
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as m:
        out = m.dict()
        ps = [ctx.Process(target=_replica_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in ps:
            p.start()
        for p in ps:
            p.join(90)
        assert all(p.exitcode == 0 for p in ps), [p.exitcode for p in ps]
        res = dict(out)
    (s0, t0, v0), (s1, t1, v1) = res[0], res[1]
    assert s0 != s1  # each replica decodes its own sequences
    assert t0 == t1 == 2.0  # the slowest rank's time, on every rank
    assert v0 == v1 == pytest.approx(100.0 * 2 / 2.0)


def _lonely_rank(port, out):
    _env(0, 2, port)
    from mlra_latent_kv_b200 import dist as mdist
    t = time.monotonic()
    try:
        mdist.init("gloo", timeout_s=3)
        out["raised"] = False
    except Exception as e:  # noqa: BLE001 - the join must fail, whatever the exception type
        out["raised"] = True
        out["msg"] = type(e).__name__
    out["secs"] = time.monotonic() - t


def test_missing_rank_times_out():
    """Rank 1 never starts: rank 0's join ends with an error, not a hang."""
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        p = ctx.Process(target=_lonely_rank, args=(_free_port(), out))
        p.start()
        p.join(100)
        if p.is_alive():
            p.kill()
            pytest.fail("rank 0 hung waiting for the missing rank")
        res = dict(out)
    assert res.get("raised") is True, res
    assert res["secs"] < 90
