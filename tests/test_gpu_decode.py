"""GPU parity of the decode path against the fp64 oracle, through the C ABI.

Reduced sizes span several 64-token pages with ragged tails and compare every
(b, h); the full workload sizes compare sampled (b, h) rows in the launch
configuration the benchmark times.  Tolerance (bf16 cache, fp32 accumulate):
max|gpu - oracle| <= 1e-2 * max|oracle| + 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
from mlra_latent_kv_b200 import abi, synth
from mlra_latent_kv_b200.session import DecodeSession

from _support import compare, oracle_inputs, rel_l2

pytestmark = pytest.mark.gpu

KERNELS = ["simt", "auto"]


def run_case(w, kernel="auto", num_splits=0, pairs=None, inp=None):
    inp = inp if inp is not None else synth.make_inputs(w)
    s = DecodeSession(w, inp, kernel=kernel, num_splits=num_splits)
    out = s.step().clone()
    torch.cuda.synchronize()
    s.check()
    ref = oracle.decode(oracle_inputs(w, inp), pairs)
    err, tol = compare(out, ref)
    return err, tol, out, ref, s


REDUCED = {
    "tiny_mla_fp32": dict(),
    "dsv2_contiguous": dict(B=3, seq_len=300),
    "paged_varlen_h32": dict(B=6, seq_len_range=(1, 700)),
    "mlra4": dict(B=2, seq_len=333),
    "longctx_append": dict(B=2, seq_len=200),
}


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("name", list(REDUCED))
def test_reduced_workloads(name, kernel):
    w = synth.workload(name).with_(**REDUCED[name])
    err, tol, out, ref, _ = run_case(w, kernel)
    assert err <= tol, f"{name}/{kernel}: max err {err:.3e} > tol {tol:.3e} (rel l2 {rel_l2(out, ref):.2e})"


@pytest.mark.parametrize("G", [1, 2, 5])
@pytest.mark.parametrize("name", [n for n in REDUCED if n != "tiny_mla_fp32"])
def test_reduced_workloads_few_workers(name, G):
    """Few split workers, so every worker runs many pages and several sequences
    back to back (stage ring wrap-around, S double buffer, piece changes)."""
    w = synth.workload(name).with_(**REDUCED[name])
    err, tol, out, ref, _ = run_case(w, "auto", num_splits=G)
    assert err <= tol, f"{name}/G={G}: max err {err:.3e} > tol {tol:.3e}"


def _edge_lengths(w, kernel):
    """Empty, one-token and page-boundary lengths, with NaN in every unused cache slot."""
    lens = [0, 1, 63, 64, 65, 127, 128, 129]
    w = w.with_(B=len(lens), seq_len_range=(1, 2), paged=True, nan_tails=True)
    inp = synth.make_inputs(w.with_(seq_len_range=None, seq_len=max(lens)))
    # rebuild with explicit lengths: draw at max length, keep the first L_b tokens of each sequence
    keep = np.concatenate([np.arange(max(lens)) < L for L in lens])
    for k in ("c_kv", "k_rope", "tok_seq", "tok_pos"):
        inp[k] = inp[k][torch.from_numpy(keep)]
    inp["seq_lens"] = torch.tensor(lens, dtype=torch.int32)
    inp["attn_lens"] = inp["seq_lens"].clone()
    inp["q_pos"] = inp["seq_lens"].clone()
    err, tol, out, ref, _ = run_case(w, kernel, inp=inp)
    assert err <= tol, f"H={w.H}/n_branch={w.n_branch}/{kernel}: {err:.3e} > {tol:.3e}"
    assert torch.all(out[0] == 0), "empty sequence must give a zero row"


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("H", [128, 64, 32, 8])
def test_edge_lengths_mla(H, kernel):
    _edge_lengths(synth.workload("dsv2_contiguous").with_(H=H), kernel)


@pytest.mark.parametrize("H", [128, 64])
def test_edge_lengths_mlra4(H):
    """MLRA-4 above 32 heads runs four one-branch CTAs per worker (two 64-dim latent blocks each)."""
    _edge_lengths(synth.workload("mlra4").with_(H=H), "auto")


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("H", [128, 32])
@pytest.mark.parametrize("nbr,bscale", [(2, 0.7), (4, 0.5)])
def test_mlra_branches(nbr, bscale, H, kernel):
    w = synth.workload("mlra4").with_(B=3, H=H, seq_len_range=(60, 260), n_branch=nbr, branch_scale=bscale)
    err, tol, out, ref, _ = run_case(w, kernel)
    assert err <= tol


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("G", [1, 3, 7, 200])
def test_split_counts(G, kernel):
    """Worker counts below, near and far above the page count exercise the split plan."""
    w = synth.workload("paged_varlen_h32").with_(B=5, seq_len_range=(1, 400))
    err, tol, *_ = run_case(w, kernel, num_splits=G)
    assert err <= tol


@pytest.mark.parametrize("kernel", KERNELS)
def test_page_permutation_bitwise(kernel):
    """Moving pages around the pool (page table permuted with them) changes no output bit."""
    w = synth.workload("dsv2_contiguous").with_(B=3, seq_len=250, paged=True)
    inp = synth.make_inputs(w)
    s1 = DecodeSession(w, inp, kernel=kernel)
    o1 = s1.step().clone()
    perm = torch.randperm(inp["num_pages"], generator=torch.Generator().manual_seed(5)).to(torch.int32)
    pt = inp["page_table"].clone()
    m = pt >= 0
    pt[m] = perm[pt[m].long()]
    s2 = DecodeSession(w, dict(inp, page_table=pt), kernel=kernel)
    o2 = s2.step().clone()
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


@pytest.mark.parametrize("kernel", KERNELS)
def test_dominant_key_is_selected(kernel):
    """A planted key 120 logits above the rest (exp(120) overflows fp32): the
    output is that token's value row, so the running-max subtraction works."""
    w = synth.workload("dsv2_contiguous").with_(B=1, H=128, seq_len=200)
    inp = synth.make_inputs(w)
    inp["q_rope"].zero_()
    q_lat = inp["q_nope"][0, 0].double() @ inp["W_UK"][0].double()
    scale = 1.0 / np.sqrt(w.d_h + w.d_r)
    c77 = q_lat / (q_lat @ q_lat) * (120.0 / scale)
    inp["c_kv"][77] = c77.to(inp["c_kv"].dtype)
    ref = oracle.decode(oracle_inputs(w, inp), [(0, 0)])
    v77 = inp["c_kv"][77].double().numpy() @ inp["W_UV"][0].double().numpy()
    np.testing.assert_allclose(ref[(0, 0)], v77, rtol=1e-6, atol=1e-6)
    s = DecodeSession(w, inp, kernel=kernel)
    out = s.step()
    err, tol = compare(out, ref)
    assert err <= tol


def _scale_with_exact_log2(target=0.125):
    """A softmax scale whose fp32 product with log2(e) (the kernels' base-2
    logit scale) is exactly ``target``, so the absorbed query loses nothing."""
    c = np.float32(1.4426950408889634)
    s = np.float32(target / 1.4426950408889634)
    for _ in range(8):
        p = np.float32(s * c)
        if p == np.float32(target):
            return float(s)
        s = np.nextafter(s, np.float32(np.inf if p < target else -np.inf), dtype=np.float32)
    raise AssertionError("no fp32 scale found")


def _peaked_inputs(w, peak_log2, n_plant, seed):
    """Peaked attention with many near-ties, built so that every rounding on the
    GPU path except the scores' own arithmetic is exact: W_UK rows are one-hot
    (q_lat is q_nope placed on 128 latent dims, 64 in each half of the 512),
    q_nope entries are +-(1 + k 2^-7) (bf16-exact), latents are small
    integers, the base-2 logit scale is 1/8 exactly and there is no rope
    term.  So every QK^T partial is exact in fp32, and a score's error can
    only come from how the two halves' partials are combined.  n_plant tokens
    per sequence, spread over its pages (hence over split workers), carry
    logits near ``peak_log2`` (log2 units) within about +-0.6 of each other;
    the other tokens sit near 0.  W_UV is zero on the score dims, so the
    planted tokens' values differ (from their other 384 latent dims)."""
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(seed)
    sel = np.concatenate([np.arange(0, 256, 4), 256 + np.arange(0, 256, 4)])
    Wk = np.zeros((w.d_h, w.d_c))
    Wk[np.arange(w.d_h), sel] = 1.0
    inp["W_UK"] = torch.from_numpy(np.tile(Wk, (w.H, 1, 1))).to(torch.bfloat16)
    u = rng.choice([-1.0, 1.0], w.d_h)
    q = u * (1.0 + rng.integers(0, 128, (w.B, w.H, w.d_h)) * 2.0 ** -7)
    inp["q_nope"] = torch.from_numpy(q).to(torch.bfloat16)
    assert np.array_equal(inp["q_nope"].double().numpy(), q)
    inp["q_rope"].zero_()
    T = inp["c_kv"].shape[0]
    C = rng.integers(-2, 3, (T, w.d_c)).astype(np.float64)
    alpha = int(round(peak_log2 / (0.125 * 1.5 * w.d_h)))   # planted logit ~ alpha * sum|q| / 8
    for b in range(w.B):
        rows = np.where(inp["tok_seq"].numpy() == b)[0]
        L = len(rows)
        for t in np.linspace(3, L - 3, n_plant).astype(int) + rng.integers(-2, 3, n_plant):
            c = C[rows[t]]
            c[sel] = alpha * u
            flip = rng.choice(sel, rng.integers(0, 4), replace=False)
            c[flip] += rng.choice([-1.0, 1.0], len(flip))
    inp["c_kv"] = torch.from_numpy(C).to(torch.bfloat16)
    assert np.array_equal(inp["c_kv"].double().numpy(), C)
    Wv = inp["W_UV"].clone()
    Wv[:, sel, :] = 0
    inp["W_UV"] = Wv
    return inp


@pytest.mark.parametrize("G", [0, 3])
@pytest.mark.parametrize("peak", [120.0, 240.0])
@pytest.mark.parametrize("H", [128, 32])
def test_peaked_attention_near_ties(H, peak, G):
    """Logits of 100-300 log2 units with 8 near-tied keys per sequence, in
    different pages and split workers: the combination of the two CTAs'
    partial scores must keep each score accurate to a small fraction of a
    log2 unit, or the near-tied weights (and so the output) move."""
    w = synth.workload("dsv2_contiguous").with_(B=3, H=H, seq_len=1500, paged=True, seed=17)
    inp = _peaked_inputs(w, peak, 8, seed=170 + H)
    ss = _scale_with_exact_log2()
    s = DecodeSession(w, inp, num_splits=G)
    s.dims.softmax_scale = ss
    out = s.step().clone()
    torch.cuda.synchronize()
    s.check()
    oi = oracle_inputs(w, inp)
    oi["softmax_scale"] = ss
    ref = oracle.decode(oi)
    top = max(float(np.max(v)) for v in ref.values())
    assert top > 0.1   # the values are not all zero (W_UV keeps 384 latent dims)
    err, tol = compare(out, ref)
    assert err <= tol, f"H={H} peak={peak} G={G}: {err:.3e} > {tol:.3e} (rel l2 {rel_l2(out, ref):.2e})"


@pytest.mark.parametrize("kernel", KERNELS)
def test_device_check_bad_page_id(kernel):
    w = synth.workload("dsv2_contiguous").with_(B=2, seq_len=100)
    inp = synth.make_inputs(w)
    s = DecodeSession(w, inp, kernel=kernel)
    s.page_table[1, 1] = 10_000_000  # outside the pool
    s.decode()
    with pytest.raises(abi.MlraError) as ei:
        s.check()
    assert ei.value.status == 5
    s.check()  # cleared


# Sampled (b, h) rows at full size: sequences spread over the batch plus the longest and the shortest, heads
# spread over all four TMEM lane quarters; (sequences, heads) per workload, sized so the fp64 oracle takes seconds.
FULL_SAMPLE = {
    "tiny_mla_fp32": None,
    "dsv2_contiguous": (8, 8),
    "paged_varlen_h32": (8, 5),
    "mlra4": (6, 6),
    "longctx_append": (4, 5),
}


def full_pairs(name, w, inp):
    if FULL_SAMPLE[name] is None:
        return None
    nb, nh = FULL_SAMPLE[name]
    lens = inp["attn_lens"].numpy()
    bs = set(np.linspace(0, w.B - 1, nb).round().astype(int).tolist())
    bs |= {int(lens.argmax()), int(lens.argmin())}
    hs = sorted(set(np.linspace(0, w.H - 1, nh).round().astype(int).tolist()))
    return [(b, h) for b in sorted(bs) for h in hs]


@pytest.mark.parametrize("name", list(FULL_SAMPLE))
def test_full_size_sampled(name):
    """Full workload sizes, default launch configuration (the one the benchmark times)."""
    w = synth.workload(name)
    inp = synth.make_inputs(w)
    pairs = full_pairs(name, w, inp)
    err, tol, out, ref, _ = run_case(w, "auto", pairs=pairs, inp=inp)
    assert err <= tol, f"{name}: {err:.3e} > {tol:.3e}"
    assert torch.isfinite(out.float()).all()
    if pairs is not None:
        assert len(ref) == len(pairs) >= 12


@pytest.mark.parametrize("name", ["dsv2_contiguous", "mlra4"])
def test_staged_and_graph_launches_bitwise(name):
    """The launch with stage events between the kernels (serialised), an eager
    plain launch and a CUDA-graph replay of the plain launch (kernels chained by
    programmatic dependent launch) give the same output bits."""
    w = synth.workload(name).with_(B=4, seq_len=1000)
    s = DecodeSession(w, synth.make_inputs(w))
    o1 = s.step().clone()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    for e in ev:
        e.record()
    o2 = s.step(events=ev).clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        s.step()
    s.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    o3 = s.out.clone()
    s.check()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))
    assert ev[1].elapsed_time(ev[2]) > 0


@pytest.mark.parametrize("name", ["dsv2_contiguous", "paged_varlen_h32"])
def test_host_buffer_decode_bitwise(name):
    """mlra_decode_host (inputs and output in pinned host memory) gives the same
    bits as mlra_decode on device copies of the same inputs."""
    w = synth.workload(name).with_(B=4, seq_len=700, seq_len_range=None)
    inp = synth.make_inputs(w)
    s = DecodeSession(w, inp)
    ref = s.step().clone()
    h_out = torch.empty(s.out.shape, dtype=s.out.dtype).pin_memory()
    h_out.fill_(7)
    s.out.zero_()
    s.decode_host(inp["q_nope"].pin_memory(), inp["q_rope"].pin_memory(), inp["q_pos"].pin_memory(),
                  inp["attn_lens"].pin_memory(), h_out)
    torch.cuda.synchronize()
    s.check()
    assert torch.equal(h_out.view(torch.int16), ref.cpu().view(torch.int16))
    assert torch.count_nonzero(s.out.view(torch.int16)) == 0  # the device-buffer output was not touched


def test_bounded_wait_times_out_and_context_survives():
    """A device wait on a barrier nothing completes gives up after its limit,
    is reported as MLRA_ERR_TIMEOUT, and later work on the context runs."""
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    abi.selftest_wait_timeout(ws, 20_000_000)  # ~10 ms of SM clocks
    with pytest.raises(abi.MlraError) as ei:
        abi.check_status(ws)
    assert ei.value.status == 6 and "site 99" in str(ei.value)
    abi.check_status(ws)  # the record was cleared
    w = synth.workload("dsv2_contiguous").with_(B=2, seq_len=130)
    err, tol, *_ = run_case(w, "auto")
    assert err <= tol


@pytest.mark.parametrize("name", [w.name for w in synth.WORKLOADS])
def test_workload_kernel_family(name):
    """With the default split on the device, kernel AUTO puts every bf16
    workload on the tcgen05 kernels end to end (a fallback to the CUDA-core
    kernels would show here); the fp32 tiny workload runs on the CUDA-core
    kernels, the ones that take fp32."""
    w = synth.workload(name).with_(B=min(synth.workload(name).B, 8), seq_len=256, seq_len_range=None)
    s = DecodeSession(w, synth.make_inputs(w))
    plan = s.plan()
    assert plan["family"] == ("tcgen05" if w.dtype == "bf16" else "cuda-core"), plan
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # page ranges: a CTA pair each (tcgen05), one CTA per branch and range (128-dim branches), one CTA (CUDA cores)
    per = 1 if w.dtype != "bf16" else (w.n_branch if "branch" in plan["attention"] else 2)
    assert plan["splits"] == sms // per, plan
    s.step()
    torch.cuda.synchronize()
    s.check()


@pytest.mark.parametrize("G", [1, 2])
@pytest.mark.parametrize("logit", [30.0, 120.0])
def test_mlra4_max_jump_after_the_first_unit(logit, G):
    """MLRA-4 on the branch kernel, whose softmax exponentiates against the
    running max before a unit's maximum is known: a key planted well past the
    first two pages, ``logit`` natural-log units above head 0's others in every
    branch (30: a jump the kernel corrects by scaling; 120 = 173 log2 units:
    past its 2^64 cap, so it exponentiates that unit again).  Other heads see
    the key at random, smaller offsets, so heads with and without a jump share
    a warp."""
    w = synth.workload("mlra4").with_(B=1, H=128, seq_len=1000, seq_len_range=None)
    inp = synth.make_inputs(w)
    inp["q_rope"].zero_()
    scale = 1.0 / np.sqrt(w.d_h + w.d_r)
    t = int(np.where(inp["tok_pos"].numpy() == 700)[0][0])
    d_cb = w.d_c // w.n_branch
    c = inp["c_kv"][t].double().clone()
    for br in range(w.n_branch):
        q_lat = inp["q_nope"][0, 0].double() @ inp["W_UK"][0][:, br * d_cb:(br + 1) * d_cb].double()
        c[br * d_cb:(br + 1) * d_cb] = q_lat / (q_lat @ q_lat) * (logit / scale)
    inp["c_kv"][t] = c.to(inp["c_kv"].dtype)
    s = DecodeSession(w, inp, num_splits=G)
    assert "branch" in s.plan()["attention"], s.plan()
    out = s.step().clone()
    torch.cuda.synchronize()
    s.check()
    ref = oracle.decode(oracle_inputs(w, inp))
    err, tol = compare(out, ref)
    assert err <= tol, f"logit={logit} G={G}: {err:.3e} > {tol:.3e} (rel l2 {rel_l2(out, ref):.2e})"
