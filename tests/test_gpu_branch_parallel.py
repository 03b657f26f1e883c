"""Branch-parallel MLRA-4 on the library's kernels, with the four ranks' shares
run one after another on one GPU (the ranks never wait on one another: each
decodes its own branch slice, and the sum stands in for the all-reduce).
The summed partials must match the fp64 oracle's one-process MLRA-4 decode at
the parity tolerance, at reduced size over every (b, h) and with NaN in the
unused cache slots."""
import pytest
import torch

import oracle
from mlra_latent_kv_b200 import synth
from mlra_latent_kv_b200.branch_parallel import BranchParallelDecode

from _support import compare, oracle_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H", [128, 64])
def test_branch_parallel_shares_sum_to_the_mlra4_decode(H):
    w = synth.workload("mlra4").with_(B=3, H=H, seq_len=None, seq_len_range=(1, 700))
    inp = synth.make_inputs(w)
    total = None
    for r in range(w.n_branch):
        bp = BranchParallelDecode(w, inp, r)
        plan = bp.sess.plan()
        assert plan["family"] == "tcgen05" and "128-dim latent" in plan["attention"], plan
        part = bp.partial().float()
        torch.cuda.synchronize()
        bp.sess.check()
        total = part if total is None else total + part
    err, tol = compare(total, oracle.decode(oracle_inputs(w, inp)))
    assert err <= tol, f"H={H}: {err:.3e} > {tol:.3e}"
