"""latent_append_noalloc, the entry point for callers that cannot allocate
device memory (an engine whose cache pool owns all HBM, a decode loop that
must not risk an allocation's synchronisation, a plugin host that passes
buffers but no allocator).  It must write exactly what latent_append writes:
checked on two calls in a row (different shapes and inputs, so the second
call runs on scratch the first one left behind), and a call that would need
more than the fixed scratch must be refused without touching the cache.

This file is collected last on purpose; it also passes on its own.
"""
import numpy as np
import pytest
import torch

from mlra_latent_kv_b200 import abi, synth
from mlra_latent_kv_b200.session import DecodeSession

pytestmark = pytest.mark.gpu


def _ulp_bf16(x):
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def _within_one_ulp(a: torch.Tensor, b: torch.Tensor) -> bool:
    """The tolerance the append tests use: one bf16 ulp."""
    x, y = a.double().cpu().numpy(), b.double().cpu().numpy()
    both_nan = np.isnan(x) & np.isnan(y)   # unwritten slots keep their NaN sentinel
    close = np.abs(x - y) <= _ulp_bf16(y)
    return bool(np.all(both_nan | close))


def _session(seed, B, lens):
    w = synth.workload("longctx_append").with_(B=B, seq_len_range=lens, seed=seed)
    return DecodeSession(w, synth.make_inputs(w))


def test_noalloc_matches_latent_append_on_two_calls():
    for seed, B, lens in [(21, 4, (100, 300)), (22, 2, (64, 64))]:
        s = _session(seed, B, lens)
        lat0, rop0 = s.latent_cache.clone(), s.rope_cache.clone()
        s.append()                      # the existing entry point, with a workspace
        torch.cuda.synchronize()
        s.check()
        ref_lat, ref_rop = s.latent_cache.clone(), s.rope_cache.clone()
        s.latent_cache.copy_(lat0)
        s.rope_cache.copy_(rop0)
        abi.latent_append_noalloc(s.dims, s.d_model, s.h, s.W_DKV, s.W_KR, s.pos, s.page_table,
                                  s.latent_cache, s.rope_cache)
        torch.cuda.synchronize()
        assert _within_one_ulp(s.latent_cache, ref_lat)
        assert _within_one_ulp(s.rope_cache, ref_rop)
        # and nothing but the appended slots changed (NaN sentinels compare by bits)
        changed = (s.latent_cache.view(torch.int16) != lat0.view(torch.int16)).any(-1)
        assert int(changed.sum()) <= B


def test_noalloc_refuses_more_than_its_scratch():
    s = _session(23, 2, (64, 64))
    big = abi.make_dims(B=64, H=s.w.H, d_h=s.w.d_h, d_v=s.w.d_v, d_c=s.w.d_c, d_r=s.w.d_r,
                        max_pages_per_seq=s.maxp, num_pages=s.num_pages)
    before = s.latent_cache.clone()
    with pytest.raises(abi.MlraError) as ei:
        abi.latent_append_noalloc(big, 5120, s.h, s.W_DKV, s.W_KR, s.pos, s.page_table,
                                  s.latent_cache, s.rope_cache)
    assert ei.value.status == 2
    assert "scratch" in str(ei.value)
    torch.cuda.synchronize()
    assert torch.equal(before.view(torch.int16), s.latent_cache.view(torch.int16))
