"""MLRA-n decode with its branches spread over n GPUs: one process per GPU,
one branch per rank, one all-reduce per step.

wispaper.ai, "MLRA：突破 MLA 并行瓶颈…", section "2.1 架构拆解": the KV latent
is cut into n independent blocks, every block (branch) runs its own
attention, and the step's output is the weighted sum of the branch outputs;
sections "1. 痛点" and "3.2 解码效率的飞跃": that independence is what lets
each GPU of a tensor-parallel group hold only its own branch, so no GPU
reads the whole cache.

Partition (rank r of n = n_branch ranks):
  * latent cache: columns [r d_cb, (r + 1) d_cb) of every cached row
    (d_cb = d_c / n), in the rank's own paged pool;
  * rope cache: replicated (the rope score is shared by every branch);
  * W_UK[:, :, r-th column block] and W_UV[:, r-th row block, :];
  * queries, positions, lengths and the page table: replicated.
Each rank runs the library's decode on its slice with n_branch = 1 and
branch_scale = the workload's branch weight, which gives that branch's term
of the output; a sum all-reduce of out [B, H, d_v] completes the step.  A
rank reads (d_cb + d_r) / (d_c + d_r) of the bytes a one-GPU MLRA decode
reads (1/3 at d_c = 512, d_r = 64, n = 4).

The collective goes through torch.distributed (NCCL between GPUs, gloo on
the host); no tensor map or load here reaches another GPU's memory.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from .synth import Workload


def branch_slice(w: Workload, inp: dict, r: int) -> tuple[Workload, dict]:
    """Workload and generator tensors of rank r's branch (host-side slicing only)."""
    n = w.n_branch
    if not 0 <= r < n:
        raise ValueError(f"rank {r} has no branch (n_branch = {n})")
    d_cb = w.d_c // n
    cols = slice(r * d_cb, (r + 1) * d_cb)
    out = dict(inp)
    out["c_kv"] = inp["c_kv"][:, cols].contiguous()
    out["W_UK"] = inp["W_UK"][:, :, cols].contiguous()
    out["W_UV"] = inp["W_UV"][:, cols, :].contiguous()
    for k in ("h", "W_DKV", "W_KR", "pos"):  # an appending step would compress into the branch block only
        if k in inp:
            raise ValueError("branch-parallel decode takes a cache that is already filled (no append)")
    return w.with_(d_c=d_cb, n_branch=1), out


def all_reduce_sum(t: torch.Tensor) -> torch.Tensor:
    """Sums the ranks' partial outputs in place (the step's one collective)."""
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t


class BranchParallelDecode:
    """Rank r's share of a branch-parallel MLRA decode step on its GPU."""

    def __init__(self, w: Workload, inp: dict, rank: int, device="cuda", kernel: str = "auto"):
        from .session import DecodeSession
        self.w = w
        self.rank = rank
        self.w_r, inp_r = branch_slice(w, inp, rank)
        self.sess = DecodeSession(self.w_r, inp_r, device=device, kernel=kernel)

    def partial(self) -> torch.Tensor:
        """This rank's branch term of the output (branch_scale folded in)."""
        return self.sess.step()

    def step(self) -> torch.Tensor:
        """The whole step's output on every rank: the partial, summed over ranks."""
        return all_reduce_sum(self.partial())
