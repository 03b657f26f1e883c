"""Sequence-sharded decode on the library's kernels, with the R ranks run one
after another on one GPU (each attends its own token range; the ranks never
wait on one another, and stacking the partials stands in for the
all-gather): mlra_attend_partial per rank, then mlra_merge_upproj, must match
the fp64 oracle's decode of the whole cache at the parity tolerance, for every
attention kernel family, with empty and short sequences and NaN in the unused
cache slots."""
import pytest
import torch

import oracle
from mlra_latent_kv_b200 import synth
from mlra_latent_kv_b200.seq_parallel import SeqParallelRank

from _support import compare, oracle_inputs

pytestmark = pytest.mark.gpu


def _ragged(w):
    inp = synth.make_inputs(w)
    L = inp["attn_lens"].clone()
    L[0], L[1] = 0, 70
    keep = torch.from_numpy(inp["tok_pos"].numpy() < L.numpy()[inp["tok_seq"].numpy()])
    for k in ("c_kv", "k_rope", "tok_seq", "tok_pos"):
        inp[k] = inp[k][keep]
    inp["attn_lens"] = L
    inp["seq_lens"] = L.clone()
    inp["q_pos"] = L.clone()
    return inp


@pytest.mark.parametrize("R", [2, 3])
@pytest.mark.parametrize("name,over", [("longctx_append", dict(B=4, H=128, append_d_model=0)),
                                       ("paged_varlen_h32", dict(B=4)),
                                       ("mlra4", dict(B=4))])
def test_sharded_partials_merge_to_the_decode(name, over, R):
    w = synth.workload(name).with_(seq_len=None, seq_len_range=(500, 1500), **over)
    inp = _ragged(w)
    ranks = [SeqParallelRank(w, inp, r, R) for r in range(R)]
    parts = [rk.partial() for rk in ranks]
    o = torch.stack([p[0].clone() for p in parts])
    lse = torch.stack([p[1].clone() for p in parts])
    out = ranks[0].merge(o, lse).clone()
    torch.cuda.synchronize()
    from mlra_latent_kv_b200 import abi
    for rk in ranks:
        abi.check_status(rk.workspace)
    err, tol = compare(out, oracle.decode(oracle_inputs(w, inp)))
    assert err <= tol, f"{name}/R={R}: {err:.3e} > {tol:.3e}"
    assert torch.all(out[0] == 0)
