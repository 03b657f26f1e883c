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
        p.write_bytes(orig + b"\n")
        assert bench.source_digest() != base, f"{name} is not covered by the digest"
        p.write_bytes(orig)
    assert bench.source_digest() == base
