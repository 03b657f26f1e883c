"""Pins for the fp64 oracle: values it must reproduce that do not come from itself.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a wrong branch block, a wrong
softmax normalisation) fails at least one of them; ``test_planted_mistakes``
plants such slips in the oracle and checks that they are caught.
"""
import cmath
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import inputs as oracle_inputs_mod
from oracle import mla_oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _ev(x):
    return float(eval(x, {"math": math})) if isinstance(x, str) else float(x)


def _evm(a):
    return np.array([[_ev(v) for v in row] for row in a], dtype=np.float64) if isinstance(a[0], list) \
        else np.array([_ev(v) for v in a], dtype=np.float64)


# ---------------------------------------------------------------------------
# independent brute force: pure-Python loops, RoPE as complex multiplication
# ---------------------------------------------------------------------------

def brute_rope(vec, pos, base):
    d = len(vec)
    out = []
    for i in range(d // 2):
        z = complex(vec[2 * i], vec[2 * i + 1]) * cmath.exp(1j * pos * base ** (-2.0 * i / d))
        out += [z.real, z.imag]
    return out


def brute_decode_one(qn, qr, qpos, Wk, Wv, C, Kraw, n_branch, bscale, scale, base):
    L = len(C)
    d_c = len(C[0]) if L else len(Wv)
    d_h, d_v = len(qn), len(Wv[0])
    out = [0.0] * d_v
    if L == 0:
        return out
    d_cb = d_c // n_branch
    q_rot = brute_rope(qr, qpos, base)
    for br in range(n_branch):
        cols = range(br * d_cb, (br + 1) * d_cb)
        logits = []
        for t in range(L):
            kt = brute_rope(Kraw[t], t, base)
            content = 0.0
            for j in range(d_h):
                key_j = sum(C[t][c] * Wk[j][c] for c in cols)
                content += qn[j] * key_j
            rope_s = sum(q_rot[i] * kt[i] for i in range(len(kt)))
            logits.append(scale * (content + rope_s))
        mx = max(logits)
        e = [math.exp(s - mx) for s in logits]
        z = sum(e)
        for t in range(L):
            p = e[t] / z
            for v in range(d_v):
                val = sum(C[t][c] * Wv[c][v] for c in cols)
                out[v] += bscale * p * val
    return out


def _rand_case(rng, B=2, H=2, d_h=4, d_c=8, d_v=3, d_r=4, n_branch=1, lens=(3, 5), page_size=2,
               branch_scale=1.0, permute=True):
    lens = np.array(lens[:B])
    npages = (lens + page_size - 1) // page_size
    maxp = int(npages.max())
    P = int(npages.sum()) + 3
    order = rng.permutation(P) if permute else np.arange(P)
    pt = np.full((B, maxp), -1, dtype=np.int64)
    o = 0
    for b in range(B):
        pt[b, :npages[b]] = order[o:o + npages[b]]
        o += npages[b]
    T = int(lens.sum())
    tok_seq = np.repeat(np.arange(B), lens)
    tok_pos = np.concatenate([np.arange(L) for L in lens]) if T else np.zeros(0, np.int64)
    return dict(
        q_nope=rng.standard_normal((B, H, d_h)), q_rope=rng.standard_normal((B, H, d_r)),
        q_pos=lens.astype(np.float64) + rng.integers(0, 3, B),
        W_UK=rng.standard_normal((H, d_h, d_c)) / np.sqrt(d_c),
        W_UV=rng.standard_normal((H, d_c, d_v)) / np.sqrt(d_c),
        c_kv=rng.standard_normal((T, d_c)), k_rope=rng.standard_normal((T, d_r)),
        tok_seq=tok_seq, tok_pos=tok_pos, page_table=pt, num_pages=P, seq_lens=lens,
        n_branch=n_branch, branch_scale=branch_scale, softmax_scale=None, rope_base=10000.0,
    ), page_size


def _brute_all(inp, page_size):
    B, H = inp["q_nope"].shape[:2]
    d_h, d_r = inp["q_nope"].shape[2], inp["q_rope"].shape[2]
    scale = 1.0 / math.sqrt(d_h + d_r)
    res = {}
    for b in range(B):
        L = int(inp["seq_lens"][b])
        # logical token order: token t of sequence b is the packed row with tok_seq=b, tok_pos=t
        rows = [i for i in range(len(inp["tok_seq"])) if inp["tok_seq"][i] == b]
        rows.sort(key=lambda i: inp["tok_pos"][i])
        C = [list(inp["c_kv"][i]) for i in rows][:L]
        K = [list(inp["k_rope"][i]) for i in rows][:L]
        for h in range(H):
            res[(b, h)] = np.array(brute_decode_one(
                list(inp["q_nope"][b, h]), list(inp["q_rope"][b, h]), float(inp["q_pos"][b]),
                inp["W_UK"][h].tolist(), inp["W_UV"][h].tolist(), C, K,
                inp["n_branch"], inp["branch_scale"], scale, inp["rope_base"]))
    return res


def _max_err(a, b):
    return max(float(np.max(np.abs(a[k] - b[k]))) for k in a)


@pytest.mark.parametrize("n_branch,bscale", [(1, 1.0), (2, 0.7), (4, 0.5)])
def test_brute_force_tiny(n_branch, bscale):
    rng = np.random.default_rng(100 + n_branch)
    inp, ps = _rand_case(rng, n_branch=n_branch, branch_scale=bscale)
    got = oracle.decode(inp, page_size=ps)
    ref = _brute_all(inp, ps)
    assert _max_err(got, ref) <= 1e-12


def test_brute_force_empty_and_single():
    rng = np.random.default_rng(7)
    inp, ps = _rand_case(rng, lens=(0, 1))
    got = oracle.decode(inp, page_size=ps)
    ref = _brute_all(inp, ps)
    assert _max_err(got, ref) <= 1e-12
    assert np.all(got[(0, 0)] == 0.0) and np.all(got[(0, 1)] == 0.0)


# ---------------------------------------------------------------------------
# closed-form worked examples
# ---------------------------------------------------------------------------

def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("case", _golden()["cases"], ids=lambda c: c["name"])
def test_golden_worked_example(case):
    C = _evm(case["c_kv"])
    K = _evm(case["k_rope"])
    out = oracle.attend_sequence(
        _evm(case["q_nope"]), _evm(case["q_rope"]), float(case["q_pos"]),
        np.array(case["W_UK"], dtype=np.float64), np.array(case["W_UV"], dtype=np.float64),
        C, K, [0], n_branch=case["n_branch"], branch_scale=case["branch_scale"])
    exp = _evm(case["expected"])
    np.testing.assert_allclose(out, exp, rtol=0, atol=1e-13)


@pytest.mark.parametrize("case", _golden()["rope_cases"], ids=lambda c: c["name"])
def test_golden_rope(case):
    out = oracle.rope(np.array(case["x"]), float(case["pos"]), case["base"])
    np.testing.assert_allclose(out, _evm(case["expected"]), rtol=0, atol=1e-13)


# ---------------------------------------------------------------------------
# RoPE invariants
# ---------------------------------------------------------------------------

def test_rope_matches_complex_multiplication():
    rng = np.random.default_rng(3)
    for d in (2, 4, 16, 64):
        x = rng.standard_normal(d)
        for pos in (0, 1, 17, 4096, 131072):
            np.testing.assert_allclose(oracle.rope(x, pos), brute_rope(list(x), pos, 10000.0),
                                       rtol=0, atol=1e-11)


def test_rope_preserves_norm_and_is_relative():
    rng = np.random.default_rng(4)
    q, k = rng.standard_normal(64), rng.standard_normal(64)
    for pos in (0, 5, 1000, 131072):
        assert abs(np.linalg.norm(oracle.rope(q, pos)) - np.linalg.norm(q)) < 1e-12
    # the score depends only on the position difference
    s1 = oracle.rope(q, 40) @ oracle.rope(k, 13)
    s2 = oracle.rope(q, 40 + 777) @ oracle.rope(k, 13 + 777)
    assert abs(s1 - s2) < 1e-11
    # and it does depend on it (catches a rotation that ignores positions)
    assert abs(s1 - oracle.rope(q, 41) @ oracle.rope(k, 13)) > 1e-6
    np.testing.assert_array_equal(oracle.rope(q, 0), q)


# ---------------------------------------------------------------------------
# softmax / attention invariants
# ---------------------------------------------------------------------------

def test_absorbed_form_equals_unabsorbed():
    """Matrix absorption (yololab.net section '矩陣吸收') is associativity."""
    rng = np.random.default_rng(5)
    inp, ps = _rand_case(rng, B=1, H=3, d_h=6, d_c=12, d_v=5, d_r=4, n_branch=3, lens=(9,),
                         branch_scale=0.6)
    got = oracle.decode(inp, page_size=ps)
    L = 9
    rows = np.argsort(inp["tok_pos"])
    C, K = inp["c_kv"][rows], inp["k_rope"][rows]
    kr = oracle.rope(K, np.arange(L))
    scale = 1 / math.sqrt(6 + 4)
    for h in range(3):
        q_lat = inp["q_nope"][0, h] @ inp["W_UK"][h]                    # [d_c]
        qr = oracle.rope(inp["q_rope"][0, h], inp["q_pos"][0])
        o_lat = np.zeros(12)
        for br in range(3):
            cols = slice(4 * br, 4 * br + 4)
            s = scale * (C[:, cols] @ q_lat[cols] + kr @ qr)
            p = np.exp(s - s.max())
            o_lat[cols] = 0.6 * (p / p.sum()) @ C[:, cols]
        out = o_lat @ inp["W_UV"][h]
        np.testing.assert_allclose(got[(0, h)], out, rtol=1e-10, atol=1e-12)


def test_softmax_weights_sum_to_one():
    """Equal cached rows: every token has the same value, so out = V(c) iff weights sum to 1."""
    rng = np.random.default_rng(6)
    inp, ps = _rand_case(rng, B=1, H=2, lens=(7,))
    c = rng.standard_normal(8)
    inp["c_kv"][:] = c
    got = oracle.decode(inp, page_size=ps)
    for h in range(2):
        np.testing.assert_allclose(got[(0, h)], c @ inp["W_UV"][h], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("n_branch,bscale", [(1, 1.0), (4, 0.5)])
def test_single_token_closed_form(n_branch, bscale):
    """L = 1: each branch puts weight 1 on the only token, whatever the query and its position."""
    rng = np.random.default_rng(14)
    inp, ps = _rand_case(rng, B=1, H=3, d_h=4, d_c=8, d_v=3, n_branch=n_branch, lens=(1,), branch_scale=bscale)
    inp["q_nope"] *= 50.0          # large logits change nothing with one token
    got = oracle.decode(inp, page_size=ps)
    c = inp["c_kv"][0]
    d_cb = 8 // n_branch
    for h in range(3):
        exp = sum(bscale * c[br * d_cb:(br + 1) * d_cb] @ inp["W_UV"][h][br * d_cb:(br + 1) * d_cb]
                  for br in range(n_branch))
        np.testing.assert_allclose(got[(0, h)], exp, rtol=1e-14, atol=1e-15)


def test_planted_dominant_key():
    rng = np.random.default_rng(8)
    inp, ps = _rand_case(rng, B=1, H=1, d_h=4, d_c=8, lens=(6,))
    inp["q_rope"][:] = 0.0
    # token 3 gets a logit 40 above the others: q_nope . K_3 * scale = 40 + others ~ 0
    inp["c_kv"][:] = 0.0
    qn = inp["q_nope"][0, 0]
    Wk = inp["W_UK"][0]
    target = np.linalg.lstsq(Wk, qn / (qn @ qn), rcond=None)[0]  # c with K = W_UK c ~ q direction
    row3 = int(np.where(inp["tok_pos"] == 3)[0][0])
    scale = 1 / math.sqrt(4 + 4)
    K3 = Wk @ target
    inp["c_kv"][row3] = target * (40.0 / (scale * (qn @ K3)))
    got = oracle.decode(inp, page_size=ps)[(0, 0)]
    v3 = inp["c_kv"][row3] @ inp["W_UV"][0]
    np.testing.assert_allclose(got, v3, rtol=1e-15 + 1e-16, atol=6 * math.exp(-40) * np.abs(v3).max() + 1e-15)


def test_mlra_identical_branches_equal_mla():
    """Four identical branches with weight 1/4 reduce to MLA on one block (wispaper.ai section 2.1)."""
    rng = np.random.default_rng(9)
    inp1, ps = _rand_case(rng, B=1, H=2, d_h=4, d_c=4, d_v=3, lens=(5,))
    inp4 = dict(inp1)
    inp4["c_kv"] = np.tile(inp1["c_kv"], (1, 4))
    inp4["W_UK"] = np.tile(inp1["W_UK"], (1, 1, 4))
    inp4["W_UV"] = np.tile(inp1["W_UV"], (1, 4, 1))
    inp4["n_branch"], inp4["branch_scale"] = 4, 0.25
    a = oracle.decode(inp1, page_size=ps)
    b = oracle.decode(inp4, page_size=ps)
    assert _max_err(a, b) <= 1e-12


def test_mlra_one_branch_is_mla_and_branches_matter():
    rng = np.random.default_rng(10)
    inp, ps = _rand_case(rng, n_branch=1)
    a = oracle.decode(inp, page_size=ps)
    b = oracle.decode(dict(inp, n_branch=2, branch_scale=1.0), page_size=ps)
    assert _max_err(a, b) > 1e-3      # separate softmaxes are a different function


def test_page_table_permutation_invariance():
    rng = np.random.default_rng(11)
    inp, ps = _rand_case(rng, lens=(9, 4))
    a = oracle.decode(inp, page_size=ps)
    perm = rng.permutation(inp["num_pages"])
    pt = inp["page_table"].copy()
    pt[pt >= 0] = perm[pt[pt >= 0]]
    b = oracle.decode(dict(inp, page_table=pt), page_size=ps)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])


def test_gather_rejects_unwritten_slot():
    rng = np.random.default_rng(12)
    inp, ps = _rand_case(rng, lens=(4, 4))
    with pytest.raises(ValueError):
        oracle.decode(dict(inp, seq_lens=np.array([5, 4])), page_size=ps)


# ---------------------------------------------------------------------------
# token compression
# ---------------------------------------------------------------------------

def test_latent_append_brute_force():
    rng = np.random.default_rng(13)
    B, D, d_c, d_r = 2, 5, 4, 4
    h = rng.standard_normal((B, D))
    Wd = rng.standard_normal((D, d_c))
    Wr = rng.standard_normal((D, d_r))
    pos = np.array([3, 250])
    c, k_rot, k_raw = oracle.latent_append(h, Wd, Wr, pos)
    for b in range(B):
        cb = [sum(h[b, k] * Wd[k, j] for k in range(D)) for j in range(d_c)]
        kb = [sum(h[b, k] * Wr[k, j] for k in range(D)) for j in range(d_r)]
        np.testing.assert_allclose(c[b], cb, rtol=0, atol=1e-12)
        np.testing.assert_allclose(k_raw[b], kb, rtol=0, atol=1e-12)
        np.testing.assert_allclose(k_rot[b], brute_rope(kb, pos[b], 10000.0), rtol=0, atol=1e-12)


def _tiny_append_case():
    """A step that appends: lengths 63 and 64 put the new token in the last slot
    of a page and in the first slot of a new page (64-token pages)."""
    from mlra_latent_kv_b200 import synth
    w = synth.workload("longctx_append").with_(B=4, H=2, d_h=4, d_v=3, d_c=8, d_r=4, seq_len=None,
                                               seq_len_range=(62, 64), append_d_model=5, dtype="f32",
                                               weight_std=0.3, seed=41)
    inp = synth.make_inputs(w)
    assert {63, 64} <= set(inp["seq_lens"].tolist())
    return w, inp


def test_oracle_inputs_appends_token_at_its_position():
    """The oracle's view of an appending step holds each sequence's new token,
    compressed by brute force, at (sequence b, position pos[b]) with its RAW
    positional key, and decoding it equals a brute-force decode over L + 1
    tokens whose last token sits at position pos (yololab.net, sections
    "1. 鍵值聯合低秩壓縮" and "2. 解耦旋轉位置編碼")."""
    w, inp = _tiny_append_case()
    oi = oracle_inputs_mod.oracle_inputs(w, inp)
    T = inp["c_kv"].shape[0]
    h, Wd, Wr = (inp[k].double().numpy() for k in ("h", "W_DKV", "W_KR"))
    pos = inp["pos"].numpy()
    L = inp["seq_lens"].numpy()
    np.testing.assert_array_equal(pos, L)                       # the new token follows the cached ones
    np.testing.assert_array_equal(inp["q_pos"].numpy(), pos)    # and the query sits at its position
    np.testing.assert_array_equal(oi["seq_lens"], L + 1)
    np.testing.assert_array_equal(oi["c_kv"][:T], inp["c_kv"].double().numpy())
    np.testing.assert_array_equal(oi["tok_pos"][:T], inp["tok_pos"].numpy())
    appended = {}
    for b in range(w.B):
        rows = np.where((oi["tok_seq"] == b) & (oi["tok_pos"] == pos[b]))[0]
        assert len(rows) == 1 and rows[0] >= T
        c_b = [sum(h[b, k] * Wd[k, j] for k in range(h.shape[1])) for j in range(w.d_c)]
        k_b = [sum(h[b, k] * Wr[k, j] for k in range(h.shape[1])) for j in range(w.d_r)]
        np.testing.assert_allclose(oi["c_kv"][rows[0]], c_b, rtol=0, atol=1e-12)
        np.testing.assert_allclose(oi["k_rope"][rows[0]], k_b, rtol=0, atol=1e-12)
        appended[b] = (c_b, k_b)
    got = oracle.decode(oi)
    scale = 1.0 / math.sqrt(w.d_h + w.d_r)
    for b in range(w.B):
        rows = sorted(np.where(inp["tok_seq"].numpy() == b)[0], key=lambda i: int(inp["tok_pos"][i]))
        C = [list(inp["c_kv"][i].double().numpy()) for i in rows] + [appended[b][0]]
        K = [list(inp["k_rope"][i].double().numpy()) for i in rows] + [appended[b][1]]
        assert len(C) == L[b] + 1
        for hh in range(w.H):
            ref = brute_decode_one(list(inp["q_nope"][b, hh].double().numpy()),
                                   list(inp["q_rope"][b, hh].double().numpy()), float(inp["q_pos"][b]),
                                   inp["W_UK"][hh].double().numpy().tolist(),
                                   inp["W_UV"][hh].double().numpy().tolist(), C, K, 1, 1.0, scale, w.rope_base)
            np.testing.assert_allclose(got[(b, hh)], ref, rtol=0, atol=1e-12)


def test_bytes_per_cached_token():
    """576 stored dims (512 latent + 64 rope) in bf16 = 1152 B per token."""
    from mlra_latent_kv_b200 import synth
    w = synth.workload("dsv2_contiguous")
    assert synth.cache_bytes_per_token(w) == 1152
    # MHA with 32 heads of 128 keeps 2*4096 values per token; the latent keeps 576
    assert 2 * 32 * 128 / (w.d_c + w.d_r) > 14


# ---------------------------------------------------------------------------
# plant mistakes in the oracle (on the CPU) and check the pins catch them
# ---------------------------------------------------------------------------

def _pins_pass():
    """True if every pin holds; a planted slip that makes the oracle raise also counts as caught."""
    try:
        test_brute_force_tiny(2, 0.7)
        test_brute_force_tiny(4, 0.5)
        for c in _golden()["cases"]:
            test_golden_worked_example(c)
        for c in _golden()["rope_cases"]:
            test_golden_rope(c)
        test_rope_matches_complex_multiplication()
        test_mlra_identical_branches_equal_mla()
        test_softmax_weights_sum_to_one()
        test_latent_append_brute_force()
        test_oracle_inputs_appends_token_at_its_position()
    except (AssertionError, ValueError, IndexError):
        return False
    return True


def test_planted_mistakes(monkeypatch):
    assert _pins_pass()
    orig_rope = mla_oracle.rope

    def rope_wrong_sign(x, pos, base=10000.0):
        return orig_rope(x, -np.asarray(pos, dtype=np.float64), base)

    def rope_half_index(x, pos, base=10000.0):
        return orig_rope(x, np.asarray(pos, dtype=np.float64) * 2, base)

    orig_attend = mla_oracle.attend_sequence

    def attend_no_rope(q_nope, q_rope, *a, **k):
        return orig_attend(q_nope, np.zeros_like(np.asarray(q_rope, dtype=np.float64)), *a, **k)

    def attend_transposed_wuv(q_nope, q_rope, q_pos, W_UK, W_UV, C, K, heads, **k):
        Wv = np.asarray(W_UV, dtype=np.float64)
        if Wv.shape[1] == Wv.shape[2]:
            Wv = np.swapaxes(Wv, 1, 2)
        else:
            Wv = Wv[:, ::-1, :]
        return orig_attend(q_nope, q_rope, q_pos, W_UK, Wv, C, K, heads, **k)

    def attend_scale_sqrt_dh(*a, softmax_scale=None, **k):
        qn = a[0]
        return orig_attend(*a, softmax_scale=1.0 / math.sqrt(np.asarray(qn).shape[-1]), **k)

    def rope_rotate_half(x, pos, base=10000.0):
        # pairs (x[i], x[i + d/2]) instead of the interleaved (x[2i], x[2i+1])
        x = np.asarray(x, dtype=np.float64)
        d = x.shape[-1]
        idx = np.concatenate([np.arange(0, d, 2), np.arange(1, d, 2)])
        inv = np.argsort(idx)
        return orig_rope(x[..., inv], pos, base)[..., idx]

    def angles_missing_factor_two(pos, d_r, base=10000.0):
        # frequencies base**(-i/d_r) instead of base**(-2i/d_r)
        i = np.arange(d_r // 2, dtype=np.float64)
        return np.multiply.outer(np.asarray(pos, dtype=np.float64), np.power(float(base), -i / float(d_r)))

    def attend_no_branch_scale(*a, branch_scale=1.0, **k):
        return orig_attend(*a, branch_scale=1.0, **k)

    def attend_interleaved_branches(q_nope, q_rope, q_pos, W_UK, W_UV, C, K, heads, n_branch=1, **k):
        # branch br owns latent dims br, br + n, br + 2n, ... instead of one contiguous block
        d_c = np.asarray(C).shape[1] if np.asarray(C).ndim == 2 and np.asarray(C).shape[0] else W_UV.shape[1]
        perm = np.concatenate([np.arange(br, d_c, n_branch) for br in range(n_branch)])
        return orig_attend(q_nope, q_rope, q_pos, np.asarray(W_UK)[:, :, perm], np.asarray(W_UV)[:, perm, :],
                           np.asarray(C)[:, perm], K, heads, n_branch=n_branch, **k)

    def attend_keys_shifted(q_nope, q_rope, q_pos, W_UK, W_UV, C, K, heads, **k):
        # cached token t rotated as if it sat at position t + 1
        K = np.asarray(K, dtype=np.float64)
        return orig_attend(q_nope, q_rope, q_pos, W_UK, W_UV, C, orig_rope(K, np.ones(K.shape[0])), heads, **k)

    def attend_query_at_length(q_nope, q_rope, q_pos, W_UK, W_UV, C, K, heads, **k):
        # the query placed at position L (the sequence length) instead of its own q_pos
        return orig_attend(q_nope, q_rope, float(np.asarray(C).shape[0]), W_UK, W_UV, C, K, heads, **k)

    orig_gather = mla_oracle.gather_rows

    def gather_reversed(slot_index, page_table_row, L, page_size):
        return orig_gather(slot_index, page_table_row, L, page_size)[::-1]

    def gather_pages_reversed(slot_index, page_table_row, L, page_size):
        # the sequence's pages walked last to first; offsets within a page kept
        t = np.arange(L, dtype=np.int64)
        row = np.asarray(page_table_row, dtype=np.int64)
        n_pages = (L + page_size - 1) // page_size
        return slot_index[row[n_pages - 1 - t // page_size], t % page_size]

    orig_slot_index = mla_oracle.build_slot_index

    def slot_index_first_page_only(tok_seq, tok_pos, page_table, num_pages, page_size):
        pt = np.asarray(page_table).copy()
        pt[:, 1:] = pt[:, :1]
        return orig_slot_index(tok_seq, tok_pos, pt, num_pages, page_size)

    orig_append = mla_oracle.latent_append

    def append_rope_next_position(h, W_DKV, W_KR, pos, rope_base=10000.0):
        return orig_append(h, W_DKV, W_KR, np.asarray(pos) + 1, rope_base)

    def append_unrotated_key(h, W_DKV, W_KR, pos, rope_base=10000.0):
        c, _, k_raw = orig_append(h, W_DKV, W_KR, pos, rope_base)
        return c, k_raw, k_raw

    orig_inputs = oracle_inputs_mod.oracle_inputs

    def inputs_append_next_position(w, inp):
        # the appended token placed one position after the one it is written at
        d = orig_inputs(w, inp)
        d["tok_pos"] = d["tok_pos"].copy()
        d["tok_pos"][-w.B:] += 1
        return d

    def inputs_append_rotated_key(w, inp):
        # the appended token's positional key kept rotated (the oracle rotates on read)
        d = orig_inputs(w, inp)
        d["k_rope"] = d["k_rope"].copy()
        d["k_rope"][-w.B:] = mla_oracle.rope(d["k_rope"][-w.B:], d["tok_pos"][-w.B:], w.rope_base)
        return d

    for fn in (inputs_append_next_position, inputs_append_rotated_key):
        with monkeypatch.context() as m:
            m.setattr(oracle_inputs_mod, "oracle_inputs", fn)
            assert not _pins_pass(), f"planted mistake in oracle_inputs ({fn.__name__}) went unnoticed"

    for name, fn in [("rope", rope_wrong_sign), ("rope", rope_half_index), ("rope", rope_rotate_half),
                     ("rope_angles", angles_missing_factor_two),
                     ("attend_sequence", attend_no_rope),
                     ("attend_sequence", attend_transposed_wuv),
                     ("attend_sequence", attend_scale_sqrt_dh),
                     ("attend_sequence", attend_no_branch_scale),
                     ("attend_sequence", attend_interleaved_branches),
                     ("attend_sequence", attend_keys_shifted),
                     ("attend_sequence", attend_query_at_length),
                     ("gather_rows", gather_reversed),
                     ("gather_rows", gather_pages_reversed),
                     ("build_slot_index", slot_index_first_page_only),
                     ("latent_append", append_rope_next_position),
                     ("latent_append", append_unrotated_key)]:
        with monkeypatch.context() as m:
            m.setattr(mla_oracle, name, fn)
            m.setattr(oracle, name, fn)
            assert not _pins_pass(), f"planted mistake in {name} ({fn.__name__}) went unnoticed"
    assert _pins_pass()
