"""Oracle view of generator tensors (test infrastructure only).

Widens the generator's bf16/fp32 tensors to numpy fp64 exactly and, for a step
that appends a token, compresses that token with the oracle's own
``latent_append`` and adds it to the cached rows.
"""
from __future__ import annotations

import numpy as np

from .mla_oracle import latent_append


def f64(t) -> np.ndarray:
    """Exact widening of a tensor (torch or numpy) to a numpy array (fp64 for floats)."""
    if hasattr(t, "is_floating_point"):
        return t.double().numpy() if t.is_floating_point() else t.numpy()
    return np.asarray(t)


def oracle_inputs(w, inp: dict) -> dict:
    """``w``: workload description (attributes n_branch, branch_scale, rope_base,
    append_d_model, B); ``inp``: the generator's tensors for one step."""
    d = dict(
        q_nope=f64(inp["q_nope"]), q_rope=f64(inp["q_rope"]), q_pos=f64(inp["q_pos"]),
        W_UK=f64(inp["W_UK"]), W_UV=f64(inp["W_UV"]),
        c_kv=f64(inp["c_kv"]), k_rope=f64(inp["k_rope"]),
        tok_seq=f64(inp["tok_seq"]).astype(np.int64), tok_pos=f64(inp["tok_pos"]).astype(np.int64),
        page_table=f64(inp["page_table"]).astype(np.int64), num_pages=int(inp["num_pages"]),
        seq_lens=f64(inp["attn_lens"]).astype(np.int64),
        n_branch=w.n_branch, branch_scale=w.branch_scale, softmax_scale=None, rope_base=w.rope_base,
    )
    if w.append_d_model:
        c, _, k_raw = latent_append(f64(inp["h"]), f64(inp["W_DKV"]), f64(inp["W_KR"]), f64(inp["pos"]),
                                    w.rope_base)
        d["c_kv"] = np.concatenate([d["c_kv"], c])
        d["k_rope"] = np.concatenate([d["k_rope"], k_raw])
        d["tok_seq"] = np.concatenate([d["tok_seq"], np.arange(w.B)])
        d["tok_pos"] = np.concatenate([d["tok_pos"], f64(inp["pos"]).astype(np.int64)])
    return d
