"""GPU cache writes through the C ABI: latent_store and latent_append.

Addressing is checked bit for bit (every slot the call should not touch keeps
its NaN sentinel; every written latent row is the input row bit for bit), and
rounded values are checked against the fp64 oracle to one bf16 ulp.
"""
import numpy as np
import pytest
import torch

import oracle
from mlra_latent_kv_b200 import abi, synth
from mlra_latent_kv_b200.session import DecodeSession

from oracle.inputs import f64

pytestmark = pytest.mark.gpu


def ulp_bf16(x: np.ndarray) -> np.ndarray:
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def assert_within_one_ulp(dev: torch.Tensor, ref: np.ndarray, atol: float):
    g = dev.double().cpu().numpy()
    tol = ulp_bf16(ref) if dev.dtype == torch.bfloat16 else np.abs(ref) * 2.0 ** -21
    bad = np.abs(g - ref) > tol + atol
    assert not bad.any(), f"{bad.sum()} values off by more than one ulp; worst {np.abs(g - ref).max():.3e}"


def slots_of(inp, tok_seq, tok_pos):
    pt = inp["page_table"].long()
    return pt[tok_seq.long(), tok_pos.long() // 64] * 64 + tok_pos.long() % 64


@pytest.mark.parametrize("name,over", [("dsv2_contiguous", dict(B=3, seq_len=150, paged=True)),
                                       ("paged_varlen_h32", dict(B=4, seq_len_range=(1, 300))),
                                       ("tiny_mla_fp32", dict(seq_len=77))])
def test_latent_store_addressing_and_rope(name, over):
    w = synth.workload(name).with_(**over)
    inp = synth.make_inputs(w)
    s = DecodeSession(w, inp)
    torch.cuda.synchronize()
    s.check()
    lat = s.latent_cache.view(-1, w.d_c).cpu()
    rop = s.rope_cache.view(-1, w.d_r).cpu()
    slots = slots_of(inp, inp["tok_seq"], inp["tok_pos"])
    ib = torch.int16 if w.dtype == "bf16" else torch.int32
    # latent rows: bit-exact copies
    assert torch.equal(lat[slots].view(ib), inp["c_kv"].view(ib))
    # rope rows: RoPE(k, t) within one ulp of the fp64 rotation
    ref = oracle.cache_rows_rotated(f64(inp["k_rope"]), f64(inp["tok_pos"]), w.rope_base)
    assert_within_one_ulp(rop[slots], ref, atol=1e-6)
    # every other slot keeps the NaN sentinel, bit for bit
    untouched = torch.ones(lat.shape[0], dtype=torch.bool)
    untouched[slots] = False
    sentinel = synth.nan_bits(w.dtype)
    assert torch.all(lat[untouched].view(ib) == sentinel)
    assert torch.all(rop[untouched].view(ib) == sentinel)


@pytest.mark.parametrize("name,over", [
    ("longctx_append", dict(B=3, seq_len_range=(60, 200))),                     # one launch, one batch of rows
    ("longctx_append", dict(B=9, seq_len_range=(60, 200))),                     # three batches, the last ragged
    ("longctx_append", dict(B=5, seq_len_range=(1, 130), append_d_model=1000)),  # ragged row chunks
    ("longctx_append", dict(B=3, seq_len_range=(60, 200), d_r=62)),             # two-kernel form (4-byte pairs)
    ("longctx_append", dict(B=2, seq_len_range=(60, 200), append_d_model=8 * 10240 + 8)),  # two kernels: wide h
    ("tiny_mla_fp32", dict(B=6, seq_len_range=(1, 100), append_d_model=256)),   # fp32, one launch
])
def test_latent_append_values_and_addressing(name, over):
    w = synth.workload(name).with_(**over)
    inp = synth.make_inputs(w)
    s = DecodeSession(w, inp)
    lat0 = s.latent_cache.clone()
    rop0 = s.rope_cache.clone()
    s.append()
    torch.cuda.synchronize()
    s.check()
    c, k_rot, _ = oracle.latent_append(f64(inp["h"]), f64(inp["W_DKV"]), f64(inp["W_KR"]), f64(inp["pos"]),
                                       w.rope_base)
    slots = slots_of(inp, torch.arange(w.B), inp["pos"])
    lat = s.latent_cache.view(-1, w.d_c)
    rop = s.rope_cache.view(-1, w.d_r)
    # fp32 accumulation over d_model terms of unit-variance sums: a few 1e-6 at most
    atol = 1e-5 * max(1.0, (w.append_d_model / 5120) ** 0.5)
    assert_within_one_ulp(lat[slots], c, atol=atol)
    assert_within_one_ulp(rop[slots], k_rot, atol=atol)
    mask = torch.ones(lat.shape[0], dtype=torch.bool, device=lat.device)
    mask[slots.to(lat.device)] = False
    assert torch.equal(lat[mask].view(torch.int16), lat0.view(-1, w.d_c)[mask].view(torch.int16))
    assert torch.equal(rop[mask].view(torch.int16), rop0.view(-1, w.d_r)[mask].view(torch.int16))
    # the workspace the session sized: the error record alone for the one-launch form
    one_launch = (w.d_r % (8 if w.dtype == "bf16" else 4) == 0) and w.append_d_model <= 8 * 10240
    assert (abi.append_workspace_bytes(s.dims, s.d_model) == 256) == one_launch
    assert s.append_kernels() == (1 if one_launch else 2)


def test_latent_append_rejects_position_outside_table():
    w = synth.workload("longctx_append").with_(B=2, seq_len=64)
    inp = synth.make_inputs(w)
    s = DecodeSession(w, inp)
    s.pos[1] = s.maxp * 64 + 5
    before = s.latent_cache.clone()
    s.append()
    with pytest.raises(abi.MlraError) as ei:
        s.check()
    assert ei.value.status == 5
    # sequence 0 was written, sequence 1 was not
    slot0 = slots_of(inp, torch.tensor([0]), torch.tensor([64]))
    lat = s.latent_cache.view(-1, w.d_c)
    mask = torch.ones(lat.shape[0], dtype=torch.bool, device=lat.device)
    mask[slot0.to(lat.device)] = False
    assert torch.equal(lat[mask].view(torch.int16), before.view(-1, w.d_c)[mask].view(torch.int16))
