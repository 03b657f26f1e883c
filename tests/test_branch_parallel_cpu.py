"""Branch-parallel MLRA-4 decode (one branch per rank, one sum all-reduce),
host side on CPU: four gloo ranks each decode their branch slice with the
fp64 oracle (n_branch = 1, the branch weight), and the all-reduced sum must
equal the oracle's one-process MLRA-4 decode of the whole cache
(wispaper.ai, "MLRA：突破 MLA 并行瓶颈…", section "2.1 架构拆解": the output
is the weighted sum of independent branch attentions)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.timeout(180)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload():
    from mlra_latent_kv_b200 import synth
    return synth.workload("mlra4").with_(B=3, H=4, d_h=8, d_v=6, d_c=32, d_r=8, seq_len=None,
                                         seq_len_range=(1, 150), dtype="f32", weight_std=0.35, seed=31)


def _as_tensor(res, B, H, d_v):
    out = torch.zeros((B, H, d_v), dtype=torch.float64)
    for (b, h), v in res.items():
        out[b, h] = torch.from_numpy(v)
    return out


def _rank(rank, ws, port, result):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(ws), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), ".."))
    import oracle
    from oracle.inputs import oracle_inputs
    from mlra_latent_kv_b200 import dist as mdist, synth
    from mlra_latent_kv_b200.branch_parallel import all_reduce_sum, branch_slice
    assert mdist.init("gloo", timeout_s=60)
    w = _workload()
    inp = synth.make_inputs(w)                     # every rank draws the same step (replicated inputs)
    w_r, inp_r = branch_slice(w, inp, rank)
    assert w_r.n_branch == 1 and w_r.d_c == w.d_c // 4 and w_r.branch_scale == w.branch_scale
    part = _as_tensor(oracle.decode(oracle_inputs(w_r, inp_r)), w.B, w.H, w.d_v)
    total = all_reduce_sum(part.clone())
    if rank == 0:
        ref = _as_tensor(oracle.decode(oracle_inputs(w, inp)), w.B, w.H, w.d_v)
        result["err"] = float((total - ref).abs().max())
        result["scale"] = float(ref.abs().max())
        result["single_branch_err"] = float((part - ref).abs().max())
    mdist.shutdown()


def test_four_branch_ranks_sum_to_the_mlra4_decode():
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        result = mgr.dict()
        procs = [ctx.Process(target=_rank, args=(r, 4, port, result)) for r in range(4)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(150)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        assert result["err"] <= 1e-12 * max(1.0, result["scale"])
        assert result["single_branch_err"] > 1e-3      # one branch alone is not the output


def test_branch_slices_partition_the_latent_and_the_weights():
    from mlra_latent_kv_b200 import synth
    from mlra_latent_kv_b200.branch_parallel import branch_slice
    w = _workload()
    inp = synth.make_inputs(w)
    parts = [branch_slice(w, inp, r)[1] for r in range(4)]
    assert torch.equal(torch.cat([p["c_kv"] for p in parts], dim=1), inp["c_kv"])
    assert torch.equal(torch.cat([p["W_UK"] for p in parts], dim=2), inp["W_UK"])
    assert torch.equal(torch.cat([p["W_UV"] for p in parts], dim=1), inp["W_UV"])
    for p in parts:   # the rope key, queries and page table are replicated
        for k in ("k_rope", "q_nope", "q_rope", "q_pos", "page_table", "attn_lens"):
            assert torch.equal(p[k], inp[k])
    # each rank reads (d_cb + d_r) / (d_c + d_r) of the cache bytes: 1/3 at the MLRA-4 workload's sizes
    big = synth.workload("mlra4")
    assert (big.d_c // 4 + big.d_r) / (big.d_c + big.d_r) == pytest.approx(1 / 3)
    with pytest.raises(ValueError):
        branch_slice(w, inp, 4)
    wa = synth.workload("longctx_append").with_(B=1, seq_len=70, n_branch=4)
    with pytest.raises(ValueError):
        branch_slice(wa, synth.make_inputs(wa), 0)
