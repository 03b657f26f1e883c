"""fp64 CPU oracle for latent-KV single-token decode attention (MLA and MLRA-n).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The product path
(the CUDA library and its Python binding) never calls it, and this module
imports nothing from the product package.

What it computes, and where each step comes from (pages are cited by site,
title and section):

* Joint KV compression -- yololab.net, "超越 GQA 的推理革命：DeepSeek 如何用
  MLA 重新定義 LLM 的記憶體極限？", section "1. 鍵值聯合低秩壓縮": every token
  keeps only a latent ``c_KV`` (width d_c); keys and values are restored from
  it by up-projection when attention reads the cache.  agentalpha.top,
  "MLA (Multi-head Latent Attention) 是什么", 核心机制 steps 1-3 (compress,
  store, restore-then-attend) say the same.
* Decoupled RoPE key -- same yololab.net page, section "2. 解耦旋轉位置編碼":
  a small positional key ``k_rope`` (width d_r) is kept beside the latent,
  is not compressed, and adds its own term to the attention score.
* RoPE itself -- the pages cite RoFormer without printing the formula; the
  reading used here is RoFormer's interleaved pairs (x[2i], x[2i+1]) rotated
  by the angle pos * base**(-2i/d_r).
* Scaled softmax attention -- yunthe.com, "多头潜在注意力机制：内存优化与推理
  加速的革新方案", section "二、MLA技术原理" (softmax of scaled QK^T times V;
  the printed formula is garbled, its plain reading is used).
* MLRA branches -- wispaper.ai, "MLRA：突破 MLA 并行瓶颈，长文本解码提速 280%",
  section "2.1 架构拆解": the KV projection is cut into blocks, each branch
  runs its own attention, and the output is the weighted sum of the branch
  outputs.  Section "2.2 方差校准" names a scaling whose formula is missing
  from the page, so the branch weight is a plain input (``branch_scale``).
  Parity of that calibration formula is unpinned (there is no formula).

This oracle deliberately computes the UNABSORBED form: per head it
materialises K = c_KV W_UK^T and V = c_KV W_UV and then runs softmax
attention.  The CUDA path computes the absorbed form (the yololab.net
section "矩陣吸收：推理加速的最後一哩路"); the two agree by associativity.

Readings of points the pages leave open:
  * softmax scale defaults to 1/sqrt(d_h + d_r);
  * cached token t sits at position t; the query sits at ``q_pos[b]``;
  * the cache holds the raw (un-rotated) ``k_rope`` in this oracle's own
    index pool, and RoPE is applied on read (the CUDA cache stores it rotated);
  * MLRA branch ``br`` owns latent columns [br*d_cb, (br+1)*d_cb) of c_KV and
    of W_UK, and the same rows of W_UV; one query per head, one shared rope
    score added to every branch;
  * an empty sequence gives a zero output.

All arithmetic is numpy float64; the inputs are the exact values the GPU
sees (bf16 or fp32 widened to fp64 by the caller).
"""
from __future__ import annotations

import numpy as np

DEFAULT_ROPE_BASE = 10000.0


def default_softmax_scale(d_h: int, d_r: int) -> float:
    """1/sqrt(d_h + d_r): the query-key dot spans d_h content + d_r rope dims."""
    return 1.0 / np.sqrt(float(d_h + d_r))


# ----------------------------------------------------------------------------
# RoPE (decoupled positional key; RoFormer rotation)
# ----------------------------------------------------------------------------

def rope_angles(pos, d_r: int, base: float = DEFAULT_ROPE_BASE) -> np.ndarray:
    """Angles pos * base**(-2i/d_r) for i < d_r/2; shape pos.shape + (d_r/2,)."""
    i = np.arange(d_r // 2, dtype=np.float64)
    theta = np.power(float(base), -2.0 * i / float(d_r))
    return np.multiply.outer(np.asarray(pos, dtype=np.float64), theta)


def rope(x, pos, base: float = DEFAULT_ROPE_BASE) -> np.ndarray:
    """Rotate each interleaved pair (x[2i], x[2i+1]) by pos * theta_i.

    ``x`` has shape (..., d_r); ``pos`` broadcasts against x.shape[:-1].
    """
    x = np.asarray(x, dtype=np.float64)
    ang = rope_angles(pos, x.shape[-1], base)
    c, s = np.cos(ang), np.sin(ang)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (x.shape[-1],)))
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


# ----------------------------------------------------------------------------
# Paged cache addressing (integer bookkeeping only)
# ----------------------------------------------------------------------------

def build_slot_index(tok_seq, tok_pos, page_table, num_pages: int, page_size: int) -> np.ndarray:
    """Index pool: slot (page, offset) -> row of the packed token arrays, -1 if empty.

    Writing token (b, t) goes to page page_table[b, t // page_size], offset
    t % page_size -- the same addressing the CUDA cache uses.
    """
    tok_seq = np.asarray(tok_seq, dtype=np.int64)
    tok_pos = np.asarray(tok_pos, dtype=np.int64)
    pt = np.asarray(page_table, dtype=np.int64)
    pool = np.full((num_pages, page_size), -1, dtype=np.int64)
    pages = pt[tok_seq, tok_pos // page_size]
    if np.any(pages < 0) or np.any(pages >= num_pages):
        raise ValueError("page table entry out of range for a written token")
    pool[pages, tok_pos % page_size] = np.arange(tok_seq.shape[0], dtype=np.int64)
    return pool


def gather_rows(slot_index, page_table_row, L: int, page_size: int) -> np.ndarray:
    """Packed-row indices of tokens 0..L-1 of one sequence, read through its page table."""
    t = np.arange(L, dtype=np.int64)
    row = np.asarray(page_table_row, dtype=np.int64)
    if L > row.shape[0] * page_size:
        raise ValueError("sequence longer than its page table row")
    pages = row[t // page_size]
    if np.any(pages < 0) or np.any(pages >= slot_index.shape[0]):
        raise ValueError("page table entry out of range")
    rows = slot_index[pages, t % page_size]
    if np.any(rows < 0):
        raise ValueError("sequence reads an unwritten cache slot")
    return rows


# ----------------------------------------------------------------------------
# Attention, unabsorbed
# ----------------------------------------------------------------------------

def attend_sequence(q_nope, q_rope, q_pos, W_UK, W_UV, C, K_raw, heads, *,
                    n_branch: int = 1, branch_scale: float = 1.0,
                    softmax_scale: float | None = None,
                    rope_base: float = DEFAULT_ROPE_BASE) -> np.ndarray:
    """Decode output of one sequence for the listed heads, shape (len(heads), d_v).

    q_nope [H, d_h], q_rope [H, d_r] (un-rotated), q_pos scalar;
    W_UK [H, d_h, d_c], W_UV [H, d_c, d_v]; C [L, d_c] latent rows,
    K_raw [L, d_r] un-rotated positional keys of tokens 0..L-1.
    """
    C = np.asarray(C, dtype=np.float64)
    K_raw = np.asarray(K_raw, dtype=np.float64)
    L, d_c = C.shape
    d_h = W_UK.shape[1]
    d_r = K_raw.shape[1]
    d_v = W_UV.shape[2]
    scale = default_softmax_scale(d_h, d_r) if softmax_scale is None else float(softmax_scale)
    out = np.zeros((len(heads), d_v), dtype=np.float64)
    if L == 0:
        return out
    if d_c % n_branch:
        raise ValueError("d_c must split evenly into branches")
    d_cb = d_c // n_branch
    k_rot = rope(K_raw, np.arange(L), rope_base)              # [L, d_r], token t at position t
    for oi, h in enumerate(heads):
        q_rot = rope(np.asarray(q_rope[h], dtype=np.float64), q_pos, rope_base)   # [d_r]
        rope_score = k_rot @ q_rot                              # [L], shared by all branches
        qn = np.asarray(q_nope[h], dtype=np.float64)            # [d_h]
        Wk = np.asarray(W_UK[h], dtype=np.float64)              # [d_h, d_c]
        Wv = np.asarray(W_UV[h], dtype=np.float64)              # [d_c, d_v]
        for br in range(n_branch):
            cols = slice(br * d_cb, (br + 1) * d_cb)
            K = C[:, cols] @ Wk[:, cols].T                      # [L, d_h] restored keys
            V = C[:, cols] @ Wv[cols, :]                        # [L, d_v] restored values
            s = scale * (K @ qn + rope_score)                   # [L]
            p = np.exp(s - s.max())
            p /= p.sum()
            out[oi] += branch_scale * (p @ V)
    return out


def decode(inp: dict, pairs=None, *, page_size: int = 64) -> dict:
    """Oracle decode over a batch given as numpy fp64 arrays.

    ``inp`` keys: q_nope [B,H,d_h], q_rope [B,H,d_r], q_pos [B], W_UK, W_UV,
    c_kv [T,d_c], k_rope [T,d_r] (packed rows, raw), tok_seq [T], tok_pos [T],
    page_table [B,maxp], num_pages, seq_lens [B] (tokens attended),
    n_branch, branch_scale, softmax_scale (None = default), rope_base.

    ``pairs`` is None (every (b, h)) or an iterable of (b, h).  Returns
    {(b, h): out[d_v]}.
    """
    B, H = inp["q_nope"].shape[:2]
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(H)]
    by_b: dict[int, list[int]] = {}
    for b, h in pairs:
        by_b.setdefault(int(b), []).append(int(h))
    slot_index = build_slot_index(inp["tok_seq"], inp["tok_pos"], inp["page_table"],
                                  int(inp["num_pages"]), page_size)
    res = {}
    for b, heads in by_b.items():
        L = int(inp["seq_lens"][b])
        rows = gather_rows(slot_index, inp["page_table"][b], L, page_size)
        o = attend_sequence(inp["q_nope"][b], inp["q_rope"][b], float(inp["q_pos"][b]),
                            inp["W_UK"], inp["W_UV"], inp["c_kv"][rows], inp["k_rope"][rows], heads,
                            n_branch=int(inp.get("n_branch", 1)),
                            branch_scale=float(inp.get("branch_scale", 1.0)),
                            softmax_scale=inp.get("softmax_scale"),
                            rope_base=float(inp.get("rope_base", DEFAULT_ROPE_BASE)))
        for oi, h in enumerate(heads):
            res[(b, h)] = o[oi]
    return res


# ----------------------------------------------------------------------------
# Token compression (latent_append) and the cache write of given rows
# ----------------------------------------------------------------------------

def latent_append(h, W_DKV, W_KR, pos, rope_base: float = DEFAULT_ROPE_BASE):
    """Compress new tokens: c_KV = h W_DKV and k_rope = RoPE(h W_KR, pos).

    yololab.net page, sections "1. 鍵值聯合低秩壓縮" (c_KV) and "2. 解耦旋轉位置
    編碼" (k_rope kept beside the latent, RoPE'd, not compressed).
    Returns (c [B, d_c], k_rot [B, d_r], k_raw [B, d_r]) in fp64.
    """
    h = np.asarray(h, dtype=np.float64)
    c = h @ np.asarray(W_DKV, dtype=np.float64)
    k_raw = h @ np.asarray(W_KR, dtype=np.float64)
    k_rot = rope(k_raw, np.asarray(pos, dtype=np.float64), rope_base)
    return c, k_rot, k_raw


def cache_rows_rotated(k_rope_raw, tok_pos, rope_base: float = DEFAULT_ROPE_BASE) -> np.ndarray:
    """The positional keys as a cache that stores them rotated holds them: RoPE(k, t)."""
    return rope(np.asarray(k_rope_raw, dtype=np.float64), np.asarray(tok_pos, dtype=np.float64), rope_base)
