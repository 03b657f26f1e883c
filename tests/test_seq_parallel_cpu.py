"""Sequence-sharded decode across GPUs, host side on CPU: the page-aligned
token shards partition every sequence's cache, and three gloo ranks that
each attend their own token range (fp64, absolute positions), all-gather
their partials and merge them by log-sum-exp reproduce the oracle's decode of
the whole cache."""
import math
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
    return synth.workload("longctx_append").with_(B=5, H=3, d_h=8, d_v=6, d_c=16, d_r=8, seq_len=None,
                                                  seq_len_range=(1, 400), append_d_model=0, dtype="f32",
                                                  weight_std=0.3, seed=51)


def _inputs(w):
    from mlra_latent_kv_b200 import synth
    inp = synth.make_inputs(w)
    # one empty sequence, one shorter than a page per rank, one exactly on a page boundary
    L = inp["attn_lens"].clone()
    L[0], L[1], L[2] = 0, 70, 128
    keep = torch.from_numpy(inp["tok_pos"].numpy() < L.numpy()[inp["tok_seq"].numpy()])
    for k in ("c_kv", "k_rope", "tok_seq", "tok_pos"):
        inp[k] = inp[k][keep]
    inp["attn_lens"] = L
    inp["seq_lens"] = L.clone()
    inp["q_pos"] = L.clone()
    return inp


def _partial_fp64(w, inp, sh):
    """Test-local fp64 partial of one rank: per (b, h) the output over the rank's
    tokens (value space) and the log-sum-exp of their scores in base 2."""
    import oracle
    scale = 1.0 / math.sqrt(w.d_h + w.d_r)
    o = torch.zeros((w.B, w.H, w.d_v), dtype=torch.float64)
    lse = torch.full((w.B, w.H), -math.inf, dtype=torch.float64)
    tseq, tpos = sh["tok_seq"].numpy(), sh["tok_pos"].numpy()
    C, K = sh["c_kv"].double().numpy(), sh["k_rope"].double().numpy()
    for b in range(w.B):
        rows = np.where(tseq == b)[0]
        if len(rows) == 0:
            continue
        kr = oracle.rope(K[rows], tpos[rows].astype(np.float64))
        for h in range(w.H):
            Wk = inp["W_UK"][h].double().numpy()
            Wv = inp["W_UV"][h].double().numpy()
            qr = oracle.rope(inp["q_rope"][b, h].double().numpy(), float(inp["q_pos"][b]))
            s = scale * ((C[rows] @ Wk.T) @ inp["q_nope"][b, h].double().numpy() + kr @ qr)
            mx = s.max()
            p = np.exp(s - mx)
            lse[b, h] = (mx + math.log(p.sum())) / math.log(2.0)
            o[b, h] = torch.from_numpy((p / p.sum()) @ (C[rows] @ Wv))
    return o, lse


def _rank(rank, ws, port, result):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(ws), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), ".."))
    import torch.distributed as dist
    import oracle
    from oracle.inputs import oracle_inputs
    from mlra_latent_kv_b200 import dist as mdist
    from mlra_latent_kv_b200.seq_parallel import merge_host, token_shard
    assert mdist.init("gloo", timeout_s=60)
    w = _workload()
    inp = _inputs(w)
    o, lse = _partial_fp64(w, inp, token_shard(w, inp, rank, ws))
    o_all = [torch.empty_like(o) for _ in range(ws)]
    l_all = [torch.empty_like(lse) for _ in range(ws)]
    dist.all_gather(o_all, o)
    dist.all_gather(l_all, lse)
    out = merge_host(torch.stack(o_all), torch.stack(l_all))
    if rank == 0:
        ref = oracle.decode(oracle_inputs(w, inp))
        R = torch.stack([torch.stack([torch.from_numpy(ref[(b, h)]) for h in range(w.H)]) for b in range(w.B)])
        result["err"] = float((out - R).abs().max())
        result["scale"] = float(R.abs().max())
        result["empty_row_zero"] = bool(torch.all(out[0] == 0))
    mdist.shutdown()


def test_three_ranks_merge_to_the_oracle_decode():
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        result = mgr.dict()
        procs = [ctx.Process(target=_rank, args=(r, 3, port, result)) for r in range(3)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(150)
        for p in procs:
            if p.is_alive():
                p.kill()
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        assert result["err"] <= 1e-12 * max(1.0, result["scale"])
        assert result["empty_row_zero"]


@pytest.mark.parametrize("R", [1, 2, 3, 5])
def test_token_shards_partition_every_sequence(R):
    from mlra_latent_kv_b200.seq_parallel import token_shard
    w = _workload()
    inp = _inputs(w)
    L = inp["attn_lens"].numpy()
    seen = set()
    total = 0
    for r in range(R):
        sh = token_shard(w, inp, r, R)
        pairs = set(zip(sh["tok_seq"].tolist(), sh["tok_pos"].tolist()))
        assert not pairs & seen
        seen |= pairs
        total += int(sh["lens_loc"].sum())
        ta, tl = sh["table_abs"].numpy(), sh["table_loc"].numpy()
        for b in range(w.B):
            nb = int(sh["lens_loc"][b])
            own = np.where(ta[b] >= 0)[0]
            assert len(own) == (nb + 63) // 64 or (nb == 0 and len(own) == 0)
            if len(own):
                assert np.array_equal(own, np.arange(own[0], own[0] + len(own)))
                assert np.array_equal(tl[b, :len(own)], ta[b, own])       # the local table is the shifted row
                # the rank's tokens start on a page boundary and sit at absolute positions
                pos = sh["tok_pos"].numpy()[sh["tok_seq"].numpy() == b]
                assert pos.min() == 64 * own[0] and pos.max() < 64 * (own[0] + len(own))
    assert seen == set(zip(inp["tok_seq"].tolist(), inp["tok_pos"].tolist()))
    assert total == int(L.sum())
