"""FP8 (E4M3, per-page scale) latent cache on the GPU: the quantizer matches
the oracle's codec bit for bit, and a decode over the quantized cache matches
the fp64 oracle run on the dequantized rows (the quantization error itself is
pinned on the CPU, tests/test_oracle_fp8.py)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import fp8
from mlra_latent_kv_b200 import abi, synth
from mlra_latent_kv_b200.session import DecodeSession

from _support import compare, oracle_inputs, rel_l2

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_mla_fp32": dict(),
    "paged_varlen_h32": dict(B=3, seq_len_range=(1, 700)),
    "dsv2_contiguous": dict(B=2, seq_len=300),
    "mlra4": dict(B=2, seq_len=333),
}


def _quantized(name):
    w = synth.workload(name).with_(**CASES[name])
    inp = synth.make_inputs(w)
    s = DecodeSession(w, inp)
    s.quantize_fp8()
    torch.cuda.synchronize()
    return w, inp, s


@pytest.mark.parametrize("name", list(CASES))
def test_quantizer_matches_the_oracle_codec(name):
    w, inp, s = _quantized(name)
    for pool, codes, scales in ((s.latent_cache, s.lat8, s.lat_scale), (s.rope_cache, s.rop8, s.rop_scale)):
        x = pool.float().cpu().numpy()
        ref_codes, ref_scales = fp8.quantize_pages(x)
        np.testing.assert_array_equal(scales.cpu().numpy(), ref_scales)
        got = codes.cpu().numpy()
        nan = np.isnan(x)
        assert nan.any() or name == "tiny_mla_fp32"       # the unused slots are poisoned (the tiny pool is full)
        np.testing.assert_array_equal(got[~nan], ref_codes[~nan])
        assert np.all(np.isnan(fp8.e4m3_decode(got[nan])))


@pytest.mark.parametrize("name", list(CASES))
def test_decode_over_fp8_cache_matches_the_oracle(name):
    w, inp, s = _quantized(name)
    s.decode_fp8()
    out = s.out.clone()
    torch.cuda.synchronize()
    abi.check_status(s.ws_fp8)
    oi = oracle_inputs(w, inp)
    oi["c_kv"], oi["k_rope"] = fp8.dequantized_rows(s.lat8.cpu().numpy(), s.lat_scale.cpu().numpy(),
                                                    s.rop8.cpu().numpy(), s.rop_scale.cpu().numpy(),
                                                    oi["tok_seq"], oi["tok_pos"], oi["page_table"],
                                                    rope_base=w.rope_base)
    ref = oracle.decode(oi)
    err, tol = compare(out, ref)
    assert err <= tol, f"{name}: {err:.3e} > {tol:.3e} (rel l2 {rel_l2(out, ref):.2e})"
    # the same step on the bf16 cache differs from it by about the format's error, not more
    s.decode()
    torch.cuda.synchronize()
    diff = (s.out.float() - out.float()).abs().max().item()
    assert diff < 0.25 * max(1e-3, out.float().abs().max().item())


def test_fp8_decode_refuses_the_tensor_core_kernels():
    w, inp, s = _quantized("paged_varlen_h32")
    d = s.dims_fp8
    d.kernel = 2  # MLRA_KERNEL_TC
    with pytest.raises(abi.MlraError) as ei:
        abi.decode_fp8(d, s.q_nope, s.q_rope, s.q_pos, s.W_UK, s.W_UV, s.lat8, s.rop8, s.lat_scale, s.rop_scale,
                       s.page_table, s.seq_lens, s.out, s.ws_fp8)
    assert ei.value.status == 2  # MLRA_ERR_UNSUPPORTED
