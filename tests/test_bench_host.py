"""Host-side logic of the benchmark line, on CPU: the algorithmic bytes and
flops it divides by, and the rule that a stored ncu traffic figure is reported
only while the attention kernel's sources are the ones it was captured on."""
import json
import os
import shutil

import torch

import bench
from mlra_latent_kv_b200 import synth


def test_step_bytes_dsv2_by_hand():
    """32 sequences x 4096 tokens x (512 + 64) bf16 values, W_UK and W_UV once."""
    w = synth.workload("dsv2_contiguous")
    inp = {"attn_lens": torch.full((w.B,), w.seq_len, dtype=torch.int32)}
    sb = bench.step_bytes(w, inp)
    assert sb["tokens"] == 131072
    assert sb["cache"] == 131072 * 1152 == 150_994_944
    assert sb["weights"] == 2 * 128 * 128 * 512 * 2
    assert sb["append"] == 0
    assert sb["total"] == sb["cache"] + sb["weights"]
    # QK^T over 512 + 64 dims (rope once) and PV over 512, per head and token
    assert sb["attn_flops"] == 2 * 128 * 131072 * (512 + 64 + 512)


def test_step_bytes_counts_append_weights():
    w = synth.workload("longctx_append")
    inp = {"attn_lens": torch.full((w.B,), w.seq_len + 1, dtype=torch.int32)}
    sb = bench.step_bytes(w, inp)
    assert sb["append"] == 5120 * (512 + 64) * 2
    assert sb["total"] == sb["cache"] + sb["weights"] + sb["append"]


def test_traffic_reported_only_for_matching_sources(monkeypatch):
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        stored = json.load(f)
    for name, e in stored.items():
        if e["source_digest"] == bench.source_digest():
            assert bench.captured_traffic(name) == e["dram_bytes_per_launch"]
    assert bench.captured_traffic("no_such_workload") is None
    monkeypatch.setattr(bench, "source_digest", lambda: "0" * 16)
    for name in stored:
        assert bench.captured_traffic(name) is None


def test_source_digest_follows_every_attention_source(tmp_path, monkeypatch):
    csrc = tmp_path / "mlra_latent_kv_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.ATTN_SOURCES:
        shutil.copy(os.path.join(bench.ROOT, "mlra_latent_kv_b200", "csrc", name), csrc / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.source_digest()
    assert base == bench.source_digest()
    for name in bench.ATTN_SOURCES:
        p = csrc / name
        orig = p.read_bytes()
        p.write_bytes(orig + b"\nconstexpr int kNotThere = 1;\n")
        assert bench.source_digest() != base, f"{name} is not covered by the digest"
        p.write_bytes(orig + b"\n// a comment changes no kernel\n\n")
        assert bench.source_digest() == base, f"a comment in {name} changed the digest"
        p.write_bytes(orig)
    assert bench.source_digest() == base


def _peaks():
    return {"hbm_gbs": 6545.3, "bf16_tflops": 1618.5, "bf16_tflops_sustained": 1374.0}


def test_roofline_bound_follows_the_arithmetic():
    """HBM-bound at H = 32 (60 flop/B); at H = 128 the MLRA-4 step is HBM-bound
    by a hair (92.3 us of bytes against 90.2 us of flops at these peaks); a
    hypothetical 4x-flop kernel flips to the tensor bound."""
    for name, bound in (("paged_varlen_h32", "hbm"), ("mlra4", "hbm")):
        w = synth.workload(name)
        inp = {"attn_lens": torch.full((w.B,), w.seq_len or 16000, dtype=torch.int32)}
        sb = bench.step_bytes(w, inp)
        r = bench.roofline_of(sb, 200.0, _peaks(), "measured")
        assert r["bound"] == bound and r["unit"] == "GB/s"
        assert abs(r["frac"] - sb["cache"] / 200e-6 / 1e9 / 6545.3) < 1e-12
        assert r["tensor_peak_tflops"] == 1618.5          # the burst peak, the one the bound used
        t = max(sb["cache"] / 6545.3e9, sb["attn_flops"] / 1618.5e12)
        assert abs(r["roofline_us"] - t * 1e6) < 1e-6
    sb = dict(cache=1e9, attn_flops=4 * 247 * 1e9 * 1.1)
    r = bench.roofline_of(sb, 1000.0, _peaks(), "measured")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] == 1618.5
    assert abs(r["frac"] - sb["attn_flops"] / 1e-3 / 1e12 / 1618.5) < 1e-12


def test_oracle_sampler_grows_and_scales_to_the_step():
    w = synth.workload("dsv2_contiguous").with_(B=3, H=4, seq_len=200)
    inp = synth.make_inputs(w)
    smp = bench.OracleSampler(w, inp)
    assert smp.cores == bench.host_cores() >= 1
    p = smp.pairs(5, seed=1)
    assert len(set(p)) == 5 and all(0 <= b < 3 and 0 <= h < 4 for b, h in p)
    n, t = smp.grow(0.2)
    assert 1 <= n <= 12 and t > 0
    cb = bench.cpu_baseline(w, inp, budget_s=0.2)
    assert cb["cores"] == smp.cores and cb["kind"] == "oracle" and cb["value"] > 0
