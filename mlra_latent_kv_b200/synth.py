"""Seeded synthetic inputs for latent-KV decode workloads.

This module holds random draws, shapes and the paged-cache bookkeeping
(which page holds which token) and nothing else: no step of the attention
method is computed here.  Both the CUDA path and the CPU oracle consume
what it returns.

Draw order for a workload with seed s (numpy PCG64, ``default_rng(s)``,
float32 standard normals, stored as bf16 by round-to-nearest-even when the
workload is bf16):

  1. seq_lens, when drawn: integers uniform in [lo, hi] inclusive
  2. q_nope [B, H, d_h]            N(0, 1)
  3. q_rope [B, H, d_r]            N(0, 1)   (un-rotated)
  4. W_UK   [H, d_h, d_c]          N(0, 1) * weight_std
  5. W_UV   [H, d_c, d_v]          N(0, 1) * weight_std
  6. c_kv   rows [T, d_c]          N(0, 1)   (tokens packed sequence-major)
  7. k_rope rows [T, d_r]          N(0, 1)   (un-rotated)
  8. page permutation, when paged: ``rng.permutation(num_pages)``
  9. append inputs, when the step appends: h [B, d_model] N(0, 1);
     W_DKV [d_model, d_c] and W_KR [d_model, d_r] N(0, 1) / sqrt(d_model)
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch

PAGE_SIZE = 64
_CHUNK_ROWS = 1 << 16


@dataclass(frozen=True)
class Workload:
    """One synthetic decode workload (sizes, distributions, cache layout)."""
    name: str
    B: int
    H: int
    d_h: int
    d_v: int
    d_c: int
    d_r: int
    seq_len: int | None = None
    seq_len_range: tuple[int, int] | None = None
    n_branch: int = 1
    branch_scale: float = 1.0
    dtype: str = "bf16"
    weight_std: float = 1.0
    paged: bool = False
    nan_tails: bool = False
    append_d_model: int = 0
    seed: int = 0
    rope_base: float = 10000.0

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads of the decode study (tiny fp32 check, DeepSeek-V2-shaped
# contiguous batch, paged variable-length batch, MLRA-4, long context with a
# fused append).  Seed = position in this list.
WORKLOADS: list[Workload] = [
    Workload("tiny_mla_fp32", B=1, H=8, d_h=32, d_v=32, d_c=64, d_r=16, seq_len=256,
             dtype="f32", weight_std=1.0 / math.sqrt(64), seed=0),
    Workload("dsv2_contiguous", B=32, H=128, d_h=128, d_v=128, d_c=512, d_r=64, seq_len=4096,
             weight_std=1.0 / math.sqrt(512), seed=1),
    Workload("paged_varlen_h32", B=64, H=32, d_h=128, d_v=128, d_c=512, d_r=64,
             seq_len_range=(1024, 32768), weight_std=1.0 / math.sqrt(512), paged=True,
             nan_tails=True, seed=2),
    Workload("mlra4", B=32, H=128, d_h=128, d_v=128, d_c=512, d_r=64, seq_len=16384,
             n_branch=4, branch_scale=0.5, weight_std=1.0 / math.sqrt(128), paged=True, seed=3),
    Workload("longctx_append", B=4, H=128, d_h=128, d_v=128, d_c=512, d_r=64, seq_len=131072,
             weight_std=1.0 / math.sqrt(512), paged=True, append_d_model=5120, seed=4),
]


def workload(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        return WORKLOADS[name_or_index]
    for w in WORKLOADS:
        if w.name == name_or_index:
            return w
    raise KeyError(name_or_index)


def _normal(rng, shape, dtype: str, std: float = 1.0) -> torch.Tensor:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    t = torch.from_numpy(a)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _normal_rows(rng, n: int, d: int, dtype: str) -> torch.Tensor:
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.empty((n, d), dtype=tdt)
    for r0 in range(0, n, _CHUNK_ROWS):
        r1 = min(n, r0 + _CHUNK_ROWS)
        out[r0:r1] = torch.from_numpy(rng.standard_normal(size=(r1 - r0, d), dtype=np.float32)).to(tdt)
    return out


def make_inputs(w: Workload) -> dict:
    """Draw every input of one decode step of workload ``w`` (CPU tensors).

    Returned keys:
      seq_lens [B] int32     tokens already cached per sequence
      attn_lens [B] int32    tokens the step attends (seq_lens + 1 when it appends)
      q_nope, q_rope, q_pos, W_UK, W_UV
      c_kv [T, d_c], k_rope [T, d_r], tok_seq [T], tok_pos [T]   cached rows, packed
      page_table [B, maxp] int32 (-1 = unused), num_pages
      h, W_DKV, W_KR, pos   (only when the step appends)
    """
    rng = np.random.default_rng(w.seed)
    if w.seq_len_range is not None:
        lo, hi = w.seq_len_range
        seq_lens = rng.integers(lo, hi, size=w.B, endpoint=True).astype(np.int64)
    else:
        seq_lens = np.full(w.B, int(w.seq_len), dtype=np.int64)
    app = 1 if w.append_d_model else 0
    cap = seq_lens + app
    npages = (cap + PAGE_SIZE - 1) // PAGE_SIZE
    maxp = int(max(1, npages.max()))
    num_pages = int(max(1, npages.sum()))

    q_nope = _normal(rng, (w.B, w.H, w.d_h), w.dtype)
    q_rope = _normal(rng, (w.B, w.H, w.d_r), w.dtype)
    W_UK = _normal(rng, (w.H, w.d_h, w.d_c), w.dtype, w.weight_std)
    W_UV = _normal(rng, (w.H, w.d_c, w.d_v), w.dtype, w.weight_std)
    T = int(seq_lens.sum())
    c_kv = _normal_rows(rng, T, w.d_c, w.dtype)
    k_rope = _normal_rows(rng, T, w.d_r, w.dtype)
    tok_seq = np.repeat(np.arange(w.B, dtype=np.int64), seq_lens)
    starts = np.concatenate([[0], np.cumsum(seq_lens)[:-1]])
    tok_pos = np.arange(T, dtype=np.int64) - np.repeat(starts, seq_lens)

    base = np.concatenate([[0], np.cumsum(npages)[:-1]])
    if w.paged:
        order = rng.permutation(num_pages)
    else:
        order = np.arange(num_pages)
    page_table = np.full((w.B, maxp), -1, dtype=np.int64)
    for b in range(w.B):
        page_table[b, : npages[b]] = order[base[b]: base[b] + npages[b]]

    out = dict(
        seq_lens=torch.from_numpy(seq_lens.astype(np.int32)),
        attn_lens=torch.from_numpy((seq_lens + app).astype(np.int32)),
        q_nope=q_nope, q_rope=q_rope,
        q_pos=torch.from_numpy((seq_lens).astype(np.int32)),
        W_UK=W_UK, W_UV=W_UV,
        c_kv=c_kv, k_rope=k_rope,
        tok_seq=torch.from_numpy(tok_seq.astype(np.int32)),
        tok_pos=torch.from_numpy(tok_pos.astype(np.int32)),
        page_table=torch.from_numpy(page_table.astype(np.int32)),
        num_pages=num_pages,
    )
    if app:
        d = w.append_d_model
        out["h"] = _normal(rng, (w.B, d), w.dtype)
        out["W_DKV"] = _normal(rng, (d, w.d_c), w.dtype, 1.0 / math.sqrt(d))
        out["W_KR"] = _normal(rng, (d, w.d_r), w.dtype, 1.0 / math.sqrt(d))
        out["pos"] = torch.from_numpy(seq_lens.astype(np.int32))
    return out


def cache_bytes_per_token(w: Workload) -> int:
    """Bytes one cached token occupies: the latent plus the positional key."""
    return (w.d_c + w.d_r) * (2 if w.dtype == "bf16" else 4)


def nan_bits(dtype: str) -> int:
    """Bit pattern used to poison unused cache slots (a quiet NaN)."""
    return 0x7FC0 if dtype == "bf16" else 0x7FC00000
