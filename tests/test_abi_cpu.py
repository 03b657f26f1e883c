"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every symbol include/mlra.h declares, and rejects bad arguments before
enqueueing anything (fake device pointers are never dereferenced on these
paths)."""
import ctypes
import glob
import os
import re

import pytest

from mlra_latent_kv_b200 import abi, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return abi.lib()


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names += re.findall(r"MLRA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_library_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), f"libmlra.so does not export {n}"
        assert n in abi.SIGNATURES, f"binding has no signature for {n}"
    assert abi.version() == 1


def _dims(**kw):
    base = dict(B=4, H=128, d_h=128, d_v=128, d_c=512, d_r=64, max_pages_per_seq=8, num_pages=32,
                num_splits=74, dtype="bf16")
    base.update(kw)
    return abi.make_dims(**base)


FAKE = 1 << 20  # 256-byte aligned, never dereferenced on validation paths


def _decode(fn, dims, ws_bytes, **over):
    args = dict(q_nope=FAKE, q_rope=FAKE, q_pos=FAKE, W_UK=FAKE, W_UV=FAKE, latent_cache=FAKE, rope_cache=FAKE,
                page_table=FAKE, seq_lens=FAKE, out=FAKE, workspace=FAKE)
    args.update(over)
    return fn(ctypes.byref(dims), args["q_nope"], args["q_rope"], args["q_pos"], args["W_UK"], args["W_UV"],
              args["latent_cache"], args["rope_cache"], args["page_table"], args["seq_lens"], args["out"],
              args["workspace"], ws_bytes, None)


def test_workspace_layout_formula(L):
    # simt path, fp32: err 256 | q B*H*(d_c+d_r)*4 | o_part slots*H*d_c*4 | ml slots*nbr*2*H*4 | o_lat B*H*d_c*4
    d = _dims(dtype="f32", kernel="simt", num_splits=10, B=3, H=8, d_h=32, d_v=32, d_c=64, d_r=16)
    r = lambda x: (x + 255) // 256 * 256  # noqa: E731
    slots = 10 + 3 - 1
    exp = 256
    exp = r(exp + 3 * 8 * 80 * 4)
    exp = r(exp + slots * 8 * 64 * 4)
    exp = r(exp + slots * 1 * 2 * 8 * 4)
    exp = r(exp + 3 * 8 * 64 * 4)
    assert abi.workspace_bytes(d) == exp


def test_host_workspace_layout_formula(L):
    # decode workspace, then staging: q_nope | q_rope | q_pos | seq_lens | out, each rounded to 256 bytes
    d = _dims(dtype="f32", kernel="simt", num_splits=10, B=3, H=8, d_h=32, d_v=32, d_c=64, d_r=16)
    r = lambda x: (x + 255) // 256 * 256  # noqa: E731
    exp = abi.workspace_bytes(d)
    for n in (3 * 8 * 32 * 4, 3 * 8 * 16 * 4, 3 * 4, 3 * 4, 3 * 8 * 32 * 4):
        exp = r(exp + n)
    assert abi.host_workspace_bytes(d) == exp


def test_host_decode_validation(L):
    d = _dims(dtype="f32", kernel="simt", num_splits=10, B=3, H=8, d_h=32, d_v=32, d_c=64, d_r=16)
    fake = 1 << 20  # never dereferenced: validation fails first
    st = L.mlra_decode_host(ctypes.byref(d), None, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                            abi.host_workspace_bytes(d), None)
    assert st == 1 and "host buffer" in abi.last_error()
    st = L.mlra_decode_host(ctypes.byref(d), fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                            abi.host_workspace_bytes(d) - 1, None)
    assert st == 3


@pytest.mark.parametrize("over,status", [
    (dict(d_r=3), 1), (dict(B=0), 1), (dict(n_branch=3), 1), (dict(dtype="bf16", page_size=32), 2),
    (dict(d_c=520), 2), (dict(d_r=128), 2), (dict(softmax_scale=-1.0), 1), (dict(num_pages=0), 1),
])
def test_bad_dims_rejected(L, over, status):
    page_size = over.pop("page_size", 64)
    d = _dims(**over)
    d.page_size = page_size
    st = _decode(L.mlra_decode, d, 1 << 40)
    assert st == status, abi.last_error()
    assert abi.last_error()


def test_null_and_misaligned_pointers(L):
    d = _dims()
    assert _decode(L.mlra_decode, d, 1 << 40, q_nope=None) == 1
    assert "q_nope" in abi.last_error()
    assert _decode(L.mlra_decode, d, 1 << 40, out=FAKE + 8) == 1
    assert "aligned" in abi.last_error()
    assert _decode(L.mlra_decode, d, 1 << 40, workspace=FAKE + 16) == 1


def test_small_workspace_rejected(L):
    d = _dims()
    need = abi.workspace_bytes(d)
    assert _decode(L.mlra_decode, d, need - 1) == 3
    assert str(need) in abi.last_error()


def test_mla_decode_needs_one_branch(L):
    d = _dims(n_branch=4, branch_scale=0.5)
    assert _decode(L.mla_decode, d, 1 << 40) == 1


def test_tc_request_outside_tc_shapes_is_unsupported(L):
    d = _dims(dtype="f32", kernel="tc")
    assert _decode(L.mlra_decode, d, 1 << 40) == 2


def test_append_and_store_validation(L):
    d = _dims()
    assert L.latent_append_workspace_bytes(ctypes.byref(d), 0) == 0
    # 16-byte column groups: the one-launch form keeps its sums on chip, only the error record
    n = L.latent_append_workspace_bytes(ctypes.byref(d), 5120)
    assert n == 256
    st = L.latent_append(ctypes.byref(d), 5120, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, n - 1, None)
    assert st == 3
    # d_r = 62 does not split into 16-byte groups: the two-kernel form's split-K sums, 80 chunks of 64 rows
    d62 = _dims(d_r=62)
    n62 = L.latent_append_workspace_bytes(ctypes.byref(d62), 5120)
    assert n62 == 256 + (80 * 4 * 574 * 4 + 255) // 256 * 256
    assert L.latent_append(ctypes.byref(d62), 5120, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, n62 - 1,
                           None) == 3
    # fp32 groups are 4 columns wide: d_r = 60 still takes the one-launch form
    assert L.latent_append_workspace_bytes(ctypes.byref(_dims(d_r=60, dtype="f32")), 5120) == 256
    # a hidden width whose chunk (kAppendB rows of ceil(d_model / 8) floats) outgrows shared memory: two kernels
    big = 8 * 10240 + 8
    assert L.latent_append_workspace_bytes(ctypes.byref(d), big) == 256 + ((big + 63) // 64 * 4 * 576 * 4 + 255) // 256 * 256
    st = L.latent_store(ctypes.byref(d), -1, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, None)
    assert st == 1
    st = L.latent_store(ctypes.byref(d), 10, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 256, None)
    assert st == 1


def test_selftest_validation(L):
    assert L.mlra_selftest_wait_timeout(None, 1000, None) == 1
    assert L.mlra_selftest_wait_timeout(1 << 20, 0, None) == 1


def _workload_dims(w, num_splits=74):
    from mlra_latent_kv_b200 import synth  # noqa: F401
    return abi.make_dims(B=w.B, H=w.H, d_h=w.d_h, d_v=w.d_v, d_c=w.d_c, d_r=w.d_r, max_pages_per_seq=8,
                         num_pages=32, n_branch=w.n_branch, branch_scale=w.branch_scale, dtype=w.dtype,
                         num_splits=num_splits)


def test_every_bf16_workload_plans_the_tcgen05_family(L):
    """Kernel AUTO puts every bf16 workload of the decode study on the tcgen05
    kernels (no silent CUDA-core stage); the fp32 tiny workload runs on the
    CUDA-core kernels, which are the ones that take fp32."""
    from mlra_latent_kv_b200 import synth
    for w in synth.WORKLOADS:
        plan = abi.describe_plan(_workload_dims(w))
        if w.dtype == "bf16":
            assert plan["family"] == "tcgen05", (w.name, plan)
            assert plan["attention"].startswith("attend_tc_"), (w.name, plan)
            assert plan["kernels"] == 3, (w.name, plan)
        else:
            assert plan["family"] == "cuda-core", (w.name, plan)
            assert plan["kernels"] == 4, (w.name, plan)
        assert plan["splits"] == 74


def test_describe_plan_follows_the_kernel_switch(L):
    from mlra_latent_kv_b200 import synth
    w = synth.workload("mlra4")
    d = _workload_dims(w)
    d.kernel = 1
    assert abi.describe_plan(d)["family"] == "cuda-core"
    d.kernel = 2
    assert abi.describe_plan(d)["attention"] == "attend_tc_branch_kernel<mlra-4, one branch per cta, two-page units>"
    # MLRA-4 over 128-dim branches and a branch-parallel rank's share (one 128-dim branch) run on the
    # branch kernel
    d1 = _workload_dims(w.with_(d_c=128, n_branch=1))
    assert abi.describe_plan(d1)["attention"] == "attend_tc_branch_kernel<mla over a 128-dim latent, two-page units>"
    assert abi.describe_plan(d1)["family"] == "tcgen05"
    buf = ctypes.create_string_buffer(8)
    assert L.mlra_describe_plan(ctypes.byref(d), buf, len(buf)) == 1  # MLRA_ERR_INVALID_ARG
