"""latent_append_noalloc, the entry point for callers that cannot allocate
device memory (an engine whose cache pool owns all HBM, a decode loop that
must not risk an allocation's synchronisation, a plugin host that passes
buffers but no allocator).  It must write exactly the bits latent_append
writes: checked on two calls in a row (different shapes and inputs, so the
second call runs on scratch the first one left behind); a warm call must
change neither the device's free memory nor torch's reserved memory; a write
whose page id is out of range must be skipped, leaving every other cache
byte as latent_append leaves it; and a call that would need more than the
fixed scratch must be refused without touching the cache.

This file is collected last on purpose; it also passes on its own.
"""
import pytest
import torch

from mlra_latent_kv_b200 import abi, synth
from mlra_latent_kv_b200.session import DecodeSession

pytestmark = pytest.mark.gpu


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
        # same kernels, same scratch layout: the same bits as latent_append
        assert torch.equal(s.latent_cache.view(torch.int16), ref_lat.view(torch.int16))
        assert torch.equal(s.rope_cache.view(torch.int16), ref_rop.view(torch.int16))
        # and nothing but the appended slots changed (NaN sentinels compare by bits)
        changed = (s.latent_cache.view(torch.int16) != lat0.view(torch.int16)).any(-1)
        assert int(changed.sum()) <= B


def test_noalloc_refuses_more_than_its_scratch():
    s = _session(23, 2, (64, 64))
    # d_r = 62 does not split into 16-byte column groups: the two-kernel form, whose split-K sums
    # (80 chunks x 64 sequences x 574 columns of fp32) outgrow the fixed scratch
    big = abi.make_dims(B=64, H=s.w.H, d_h=s.w.d_h, d_v=s.w.d_v, d_c=s.w.d_c, d_r=62,
                        max_pages_per_seq=s.maxp, num_pages=s.num_pages)
    before = s.latent_cache.clone()
    with pytest.raises(abi.MlraError) as ei:
        abi.latent_append_noalloc(big, 5120, s.h, s.W_DKV, s.W_KR, s.pos, s.page_table,
                                  s.latent_cache, s.rope_cache)
    assert ei.value.status == 2
    assert "scratch" in str(ei.value)
    torch.cuda.synchronize()
    assert torch.equal(before.view(torch.int16), s.latent_cache.view(torch.int16))


def test_noalloc_warm_call_allocates_nothing():
    s = _session(24, 4, (100, 300))
    noalloc = lambda: abi.latent_append_noalloc(s.dims, s.d_model, s.h, s.W_DKV, s.W_KR, s.pos, s.page_table,
                                                s.latent_cache, s.rope_cache)
    noalloc()                         # warm: the first call on the device looks up the scratch address
    torch.cuda.synchronize()
    free0, reserved0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()
    for _ in range(3):
        noalloc()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_reserved() == reserved0


def test_noalloc_skips_a_write_with_a_bad_page_id():
    """Sequence 0's target page id is outside the pool: its token is not
    written anywhere (in particular not into page 0, which another sequence
    may own), and every other byte of both caches ends as latent_append
    (with a workspace) leaves it; latent_append also reports the bad id."""
    s = _session(25, 4, (100, 300))
    lat0, rop0 = s.latent_cache.clone(), s.rope_cache.clone()
    p0 = int(s.pos[0]) // 64
    s.page_table[0, p0] = 10_000_000
    s.append()
    torch.cuda.synchronize()
    with pytest.raises(abi.MlraError) as ei:
        s.check()
    assert ei.value.status == 5
    ref_lat, ref_rop = s.latent_cache.clone(), s.rope_cache.clone()
    s.latent_cache.copy_(lat0)
    s.rope_cache.copy_(rop0)
    abi.latent_append_noalloc(s.dims, s.d_model, s.h, s.W_DKV, s.W_KR, s.pos, s.page_table,
                              s.latent_cache, s.rope_cache)
    torch.cuda.synchronize()
    assert torch.equal(s.latent_cache.view(torch.int16), ref_lat.view(torch.int16))
    assert torch.equal(s.rope_cache.view(torch.int16), ref_rop.view(torch.int16))
    # exactly the three good sequences' slots changed
    changed = (s.latent_cache.view(torch.int16) != lat0.view(torch.int16)).any(-1)
    pt = s.page_table.cpu()
    good = {(int(pt[b, int(s.pos[b]) // 64]), int(s.pos[b]) % 64) for b in range(1, 4)}
    assert {tuple(x) for x in changed.nonzero().tolist()} == good
