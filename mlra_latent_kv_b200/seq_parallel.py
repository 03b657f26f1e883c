"""Sequence-sharded decode across GPUs for long contexts: one process per
GPU, each holding a page-aligned range of every sequence's cached tokens.

wispaper.ai, "MLRA：突破 MLA 并行瓶颈…", section "1. 痛点": long-context
decode is bound by reading the cache, so its bytes are what gets spread.
Rank r of R holds pages [r P_b / R, (r + 1) P_b / R) of sequence b (P_b =
its page count), attends them with ``mlra_attend_partial`` (a latent output
normalised over its tokens, and their log-sum-exp in base 2), the ranks
all-gather the partials in rank order, and every rank merges them with
``mlra_merge_upproj``, which weighs part r by 2^(lse_r - lse) -- the softmax
over all the sequence's tokens -- and applies W_UV.

Positions: a rank's pool and page table address its own tokens from 0, but
every cached rope key must carry the rotation of its absolute position, so
the cache is written (``latent_store``) through a table indexed by absolute
page and attended through that table's rows shifted to the rank's first
page.  The query position is absolute on every rank.

The collective is torch.distributed's (NCCL between GPUs, gloo on the host);
no tensor map or load here reaches another GPU's memory.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import abi
from .synth import PAGE_SIZE, Workload, nan_bits


def page_range(n_pages: int, r: int, R: int) -> tuple[int, int]:
    """Pages [p0, p1) of a sequence with n_pages pages that rank r of R holds."""
    return (r * n_pages) // R, ((r + 1) * n_pages) // R


def token_shard(w: Workload, inp: dict, r: int, R: int) -> dict:
    """Rank r's share of one decode step's cache (host-side bookkeeping only).

    Returns the rank's cached rows (absolute positions), its pool size, the
    absolute-page table its cache is written through, and the local table and
    lengths its decode reads through."""
    if w.append_d_model:
        raise ValueError("the sequence-sharded decode takes a cache that is already filled (no append)")
    if not 0 <= r < R:
        raise ValueError(f"rank {r} of {R}")
    L = inp["attn_lens"].numpy().astype(np.int64)
    tok_seq = inp["tok_seq"].numpy().astype(np.int64)
    tok_pos = inp["tok_pos"].numpy().astype(np.int64)
    B = w.B
    n_pages = (L + PAGE_SIZE - 1) // PAGE_SIZE
    rng = [page_range(int(n), r, R) for n in n_pages]
    own = np.array([p1 - p0 for p0, p1 in rng], dtype=np.int64)
    num_pages = int(max(1, own.sum()))
    maxp_abs = int(max(1, n_pages.max()))
    maxp_loc = int(max(1, own.max()))
    table_abs = np.full((B, maxp_abs), -1, dtype=np.int64)
    table_loc = np.full((B, maxp_loc), -1, dtype=np.int64)
    nxt = 0
    lens_loc = np.zeros(B, dtype=np.int64)
    for b, (p0, p1) in enumerate(rng):
        ids = np.arange(nxt, nxt + (p1 - p0))
        nxt += p1 - p0
        table_abs[b, p0:p1] = ids
        table_loc[b, : p1 - p0] = ids
        lens_loc[b] = max(0, min(int(L[b]), PAGE_SIZE * p1) - PAGE_SIZE * p0)
    lo = np.array([PAGE_SIZE * p0 for p0, _ in rng])[tok_seq]
    hi = np.array([PAGE_SIZE * p1 for _, p1 in rng])[tok_seq]
    keep = (tok_pos >= lo) & (tok_pos < hi)
    kt = torch.from_numpy(keep)
    return dict(
        c_kv=inp["c_kv"][kt], k_rope=inp["k_rope"][kt],
        tok_seq=torch.from_numpy(tok_seq[keep].astype(np.int32)),
        tok_pos=torch.from_numpy(tok_pos[keep].astype(np.int32)),
        num_pages=num_pages, maxp_abs=maxp_abs, maxp_loc=maxp_loc,
        table_abs=torch.from_numpy(table_abs.astype(np.int32)),
        table_loc=torch.from_numpy(table_loc.astype(np.int32)),
        lens_loc=torch.from_numpy(lens_loc.astype(np.int32)),
    )


def merge_host(o_parts: torch.Tensor, lse_parts: torch.Tensor, branch_scale: float = 1.0) -> torch.Tensor:
    """The merge of R partials on the host, one branch: o_parts [R, ..., d],
    lse_parts [R, ...] (base 2) -> branch_scale * sum_r 2^(lse_r - lse) o_r."""
    M = lse_parts.max(dim=0).values
    finite = torch.isfinite(M)
    Mz = torch.where(finite, M, torch.zeros_like(M))
    w = torch.exp2(lse_parts - Mz)
    w = torch.where(finite, w, torch.zeros_like(w))
    S = w.sum(dim=0)
    out = (w.unsqueeze(-1) * o_parts).sum(dim=0) / torch.where(S > 0, S, torch.ones_like(S)).unsqueeze(-1)
    return branch_scale * out


class SeqParallelRank:
    """Rank r's cache and partial of a sequence-sharded decode step on its GPU."""

    def __init__(self, w: Workload, inp: dict, r: int, R: int, device="cuda", kernel: str = "auto"):
        dev = torch.device(device)
        self.w, self.r, self.R = w, r, R
        sh = token_shard(w, inp, r, R)
        tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        common = dict(B=w.B, H=w.H, d_h=w.d_h, d_v=w.d_v, d_c=w.d_c, d_r=w.d_r, num_pages=sh["num_pages"],
                      n_branch=w.n_branch, branch_scale=w.branch_scale, rope_base=w.rope_base, dtype=w.dtype,
                      kernel=kernel)
        self.dims_store = abi.make_dims(max_pages_per_seq=sh["maxp_abs"], **common)
        self.dims = abi.make_dims(max_pages_per_seq=sh["maxp_loc"], **common)
        itype = torch.int16 if w.dtype == "bf16" else torch.int32
        bits = nan_bits(w.dtype)
        if w.dtype == "bf16" and bits >= (1 << 15):
            bits -= 1 << 16
        self.latent_cache = torch.empty((sh["num_pages"], PAGE_SIZE, w.d_c), dtype=tdt, device=dev)
        self.rope_cache = torch.empty((sh["num_pages"], PAGE_SIZE, w.d_r), dtype=tdt, device=dev)
        self.latent_cache.view(itype).fill_(bits)   # unwritten slots read as NaN
        self.rope_cache.view(itype).fill_(bits)
        self.workspace = torch.zeros(abi.workspace_bytes(self.dims), dtype=torch.uint8, device=dev)
        n = int(sh["c_kv"].shape[0])
        if n:
            abi.latent_store(self.dims_store, n, sh["c_kv"].to(dev), sh["k_rope"].to(dev), sh["tok_seq"].to(dev),
                             sh["tok_pos"].to(dev), sh["table_abs"].to(dev), self.latent_cache, self.rope_cache,
                             self.workspace)
        self.page_table = sh["table_loc"].to(dev)
        self.seq_lens = sh["lens_loc"].to(dev)
        self.q_nope, self.q_rope = inp["q_nope"].to(dev), inp["q_rope"].to(dev)
        self.q_pos = inp["q_pos"].to(dev)
        self.W_UK, self.W_UV = inp["W_UK"].to(dev), inp["W_UV"].to(dev)
        self.o = torch.empty((w.B, w.H, w.d_c), dtype=torch.float32, device=dev)
        self.lse = torch.empty((w.B, w.n_branch, w.H), dtype=torch.float32, device=dev)
        self.out = torch.empty((w.B, w.H, w.d_v), dtype=tdt, device=dev)
        self.merge_ws = torch.zeros(abi.merge_workspace_bytes(self.dims), dtype=torch.uint8, device=dev)
        torch.cuda.synchronize(dev)
        abi.check_status(self.workspace)

    def partial(self) -> tuple[torch.Tensor, torch.Tensor]:
        """This rank's (o [B,H,d_c] fp32, lse [B,n_branch,H] fp32)."""
        abi.attend_partial(self.dims, self.q_nope, self.q_rope, self.q_pos, self.W_UK, self.latent_cache,
                           self.rope_cache, self.page_table, self.seq_lens, self.o, self.lse, self.workspace)
        return self.o, self.lse

    def merge(self, o_parts: torch.Tensor, lse_parts: torch.Tensor) -> torch.Tensor:
        """out [B,H,d_v] from the gathered partials of all ranks (rank order)."""
        abi.merge_upproj(self.dims, o_parts, lse_parts, self.W_UV, self.out, self.merge_ws)
        return self.out

    def step(self) -> torch.Tensor:
        """One decode step: this rank's partial, the all-gather, the merge."""
        o, lse = self.partial()
        if dist.is_initialized() and dist.get_world_size() > 1:
            o_all = torch.empty((self.R,) + tuple(o.shape), dtype=o.dtype, device=o.device)
            l_all = torch.empty((self.R,) + tuple(lse.shape), dtype=lse.dtype, device=lse.device)
            dist.all_gather_into_tensor(o_all, o)
            dist.all_gather_into_tensor(l_all, lse)
        else:
            o_all, l_all = o.unsqueeze(0), lse.unsqueeze(0)
        return self.merge(o_all, l_all)
