"""ctypes binding of libmlra (include/mlra.h): argument marshalling only.

Every computation runs in the CUDA library; this module turns torch tensors
into device pointers and status codes into exceptions.  It fails loudly if the
library is missing -- there is no other implementation behind these names.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmlra.so")

MLRA_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA",
                5: "DEVICE_CHECK", 6: "TIMEOUT"}
DTYPES = {"f32": 0, "bf16": 1}
KERNELS = {"auto": 0, "simt": 1, "tc": 2}


class MlraError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libmlra {STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d_h", ctypes.c_int), ("d_v", ctypes.c_int),
                ("d_c", ctypes.c_int), ("d_r", ctypes.c_int), ("n_branch", ctypes.c_int),
                ("page_size", ctypes.c_int), ("max_pages_per_seq", ctypes.c_int), ("num_pages", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("branch_scale", ctypes.c_float),
                ("rope_base", ctypes.c_float), ("dtype", ctypes.c_int), ("num_splits", ctypes.c_int),
                ("kernel", ctypes.c_int)]


def make_dims(*, B, H, d_h, d_v, d_c, d_r, max_pages_per_seq, num_pages, n_branch=1, page_size=64,
              softmax_scale=0.0, branch_scale=1.0, rope_base=0.0, dtype="bf16", num_splits=0,
              kernel="auto") -> Dims:
    return Dims(B, H, d_h, d_v, d_c, d_r, n_branch, page_size, max_pages_per_seq, num_pages,
                float(softmax_scale), float(branch_scale), float(rope_base), DTYPES[dtype], num_splits,
                KERNELS[kernel])


_lib = None
_P = ctypes.c_void_p
_I32P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_DIMS = ctypes.POINTER(Dims)
_DECODE_ARGS = [_DIMS, _P, _P, _I32P, _P, _P, _P, _P, _I32P, _I32P, _P, _P, _SZ, _P]

SIGNATURES = {
    "mlra_workspace_bytes": (_SZ, [_DIMS]),
    "mla_decode": (ctypes.c_int, _DECODE_ARGS),
    "mlra_decode": (ctypes.c_int, _DECODE_ARGS),
    "mlra_decode_profiled": (ctypes.c_int, _DECODE_ARGS + [_P]),
    "mlra_decode_host_workspace_bytes": (_SZ, [_DIMS]),
    "mlra_decode_host": (ctypes.c_int, _DECODE_ARGS),
    "latent_append_workspace_bytes": (_SZ, [_DIMS, ctypes.c_int]),
    "latent_append": (ctypes.c_int, [_DIMS, ctypes.c_int, _P, _P, _P, _I32P, _I32P, _P, _P, _P, _SZ, _P]),
    "latent_store": (ctypes.c_int, [_DIMS, ctypes.c_int, _P, _P, _I32P, _I32P, _I32P, _P, _P, _P, _SZ, _P]),
    "latent_append_noalloc": (ctypes.c_int, [_DIMS, ctypes.c_int, _P, _P, _P, _I32P, _I32P, _P, _P, _P]),
    "mlra_describe_plan": (ctypes.c_int, [_DIMS, ctypes.c_char_p, _SZ]),
    "mlra_attend_partial": (ctypes.c_int, [_DIMS, _P, _P, _I32P, _P, _P, _P, _I32P, _I32P, _P, _P, _P, _SZ, _P]),
    "mlra_merge_workspace_bytes": (_SZ, [_DIMS]),
    "mlra_merge_upproj": (ctypes.c_int, [_DIMS, ctypes.c_int, _P, _P, _P, _P, _P, _SZ, _P]),
    "mlra_quantize_pages_fp8": (ctypes.c_int, [_DIMS, _P, _P, _P, _P, _P, _P, _P]),
    "mlra_decode_fp8": (ctypes.c_int, [_DIMS, _P, _P, _I32P, _P, _P, _P, _P, _P, _P, _I32P, _I32P, _P, _P, _SZ, _P]),
    "mlra_check_status": (ctypes.c_int, [_P, _P]),
    "mlra_selftest_wait_timeout": (ctypes.c_int, [_P, ctypes.c_longlong, _P]),
    "mlra_last_error": (ctypes.c_char_p, []),
    "mlra_shutdown": (None, []),
    "mlra_version": (ctypes.c_int, []),
}


def lib() -> ctypes.CDLL:
    """The loaded library (raises if libmlra.so has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m mlra_latent_kv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def last_error() -> str:
    return lib().mlra_last_error().decode()


def _check(status: int):
    if status != MLRA_OK:
        raise MlraError(status, last_error())


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def describe_plan(dims: Dims) -> dict:
    """The kernels a decode call launches for ``dims`` (family, splits,
    launches per call, and the kernel of each stage), as the library plans them."""
    buf = ctypes.create_string_buffer(512)
    _check(lib().mlra_describe_plan(ctypes.byref(dims), buf, len(buf)))
    out = dict(kv.split("=", 1) for kv in buf.value.decode().split(";"))
    out["splits"], out["kernels"] = int(out["splits"]), int(out["kernels"])
    return out


def attend_partial(dims, q_nope, q_rope, q_pos, W_UK, latent_cache, rope_cache, page_table, seq_lens, o, lse,
                   workspace, stream=None):
    """A sequence-sharded rank's partial: o [B,H,d_c] fp32 and lse [B,n_branch,H] fp32 (see include/mlra.h)."""
    _check(lib().mlra_attend_partial(ctypes.byref(dims), _ptr(q_nope), _ptr(q_rope), _ptr(q_pos), _ptr(W_UK),
                                     _ptr(latent_cache), _ptr(rope_cache), _ptr(page_table), _ptr(seq_lens),
                                     _ptr(o), _ptr(lse), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream)))


def merge_workspace_bytes(dims: Dims) -> int:
    n = lib().mlra_merge_workspace_bytes(ctypes.byref(dims))
    if n == 0:
        raise MlraError(1, last_error())
    return int(n)


def merge_upproj(dims, o_parts, lse_parts, W_UV, out, workspace, stream=None):
    """Merges R gathered partials ([R,B,H,d_c], [R,B,n_branch,H]) and applies W_UV into out."""
    _check(lib().mlra_merge_upproj(ctypes.byref(dims), int(o_parts.shape[0]), _ptr(o_parts), _ptr(lse_parts),
                                   _ptr(W_UV), _ptr(out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)))


def quantize_pages_fp8(dims, latent_cache, rope_cache, latent_fp8, rope_fp8, latent_scale, rope_scale,
                       stream=None):
    """FP8 E4M3 codes and per-page fp32 scales of a bf16/fp32 pool (see include/mlra.h)."""
    _check(lib().mlra_quantize_pages_fp8(ctypes.byref(dims), _ptr(latent_cache), _ptr(rope_cache), _ptr(latent_fp8),
                                         _ptr(rope_fp8), _ptr(latent_scale), _ptr(rope_scale), _stream(stream)))


def decode_fp8(dims, q_nope, q_rope, q_pos, W_UK, W_UV, latent_fp8, rope_fp8, latent_scale, rope_scale, page_table,
               seq_lens, out, workspace, stream=None):
    """mlra_decode over an FP8 cache (CUDA-core kernels; the workspace is sized for kernel SIMT)."""
    nbytes = workspace.numel() * workspace.element_size()
    _check(lib().mlra_decode_fp8(ctypes.byref(dims), _ptr(q_nope), _ptr(q_rope), _ptr(q_pos), _ptr(W_UK), _ptr(W_UV),
                                 _ptr(latent_fp8), _ptr(rope_fp8), _ptr(latent_scale), _ptr(rope_scale),
                                 _ptr(page_table), _ptr(seq_lens), _ptr(out), _ptr(workspace), nbytes,
                                 _stream(stream)))


def workspace_bytes(dims: Dims) -> int:
    n = lib().mlra_workspace_bytes(ctypes.byref(dims))
    if n == 0:
        raise MlraError(1, last_error())
    return int(n)


def _decode(fn, dims, q_nope, q_rope, q_pos, W_UK, W_UV, latent_cache, rope_cache, page_table, seq_lens, out,
            workspace, workspace_nbytes=None, stream=None, extra=()):
    nbytes = workspace_nbytes if workspace_nbytes is not None else \
        workspace.numel() * workspace.element_size()
    _check(fn(ctypes.byref(dims), _ptr(q_nope), _ptr(q_rope), _ptr(q_pos), _ptr(W_UK), _ptr(W_UV),
              _ptr(latent_cache), _ptr(rope_cache), _ptr(page_table), _ptr(seq_lens), _ptr(out),
              _ptr(workspace), nbytes, _stream(stream), *extra))


def mla_decode(dims, q_nope, q_rope, q_pos, W_UK, W_UV, latent_cache, rope_cache, page_table, seq_lens, out,
               workspace, workspace_nbytes=None, stream=None):
    _decode(lib().mla_decode, dims, q_nope, q_rope, q_pos, W_UK, W_UV, latent_cache, rope_cache, page_table,
            seq_lens, out, workspace, workspace_nbytes, stream)


def mlra_decode(dims, q_nope, q_rope, q_pos, W_UK, W_UV, latent_cache, rope_cache, page_table, seq_lens, out,
                workspace, workspace_nbytes=None, stream=None):
    _decode(lib().mlra_decode, dims, q_nope, q_rope, q_pos, W_UK, W_UV, latent_cache, rope_cache, page_table,
            seq_lens, out, workspace, workspace_nbytes, stream)


def mlra_decode_profiled(dims, q_nope, q_rope, q_pos, W_UK, W_UV, latent_cache, rope_cache, page_table, seq_lens,
                         out, workspace, events, workspace_nbytes=None, stream=None):
    """``events``: five torch.cuda.Event(enable_timing=True), already recorded once (so they exist)."""
    arr = (ctypes.c_void_p * 5)(*[e.cuda_event for e in events])
    _decode(lib().mlra_decode_profiled, dims, q_nope, q_rope, q_pos, W_UK, W_UV, latent_cache, rope_cache,
            page_table, seq_lens, out, workspace, workspace_nbytes, stream, extra=(ctypes.cast(arr, _P),))


def host_workspace_bytes(dims: Dims) -> int:
    n = lib().mlra_decode_host_workspace_bytes(ctypes.byref(dims))
    if n == 0:
        raise MlraError(1, last_error())
    return int(n)


def mlra_decode_host(dims, h_q_nope, h_q_rope, h_q_pos, W_UK, W_UV, latent_cache, rope_cache, page_table,
                     h_seq_lens, h_out, workspace, workspace_nbytes=None, stream=None):
    """Per-step inputs and the output are host (pinned) tensors; the rest is device-resident."""
    _decode(lib().mlra_decode_host, dims, h_q_nope, h_q_rope, h_q_pos, W_UK, W_UV, latent_cache, rope_cache,
            page_table, h_seq_lens, h_out, workspace, workspace_nbytes, stream)


def append_workspace_bytes(dims: Dims, d_model: int) -> int:
    n = lib().latent_append_workspace_bytes(ctypes.byref(dims), d_model)
    if n == 0:
        raise MlraError(1, last_error())
    return int(n)


def latent_append(dims, d_model, h, W_DKV, W_KR, pos, page_table, latent_cache, rope_cache, workspace,
                  workspace_nbytes=None, stream=None):
    nbytes = workspace_nbytes if workspace_nbytes is not None else workspace.numel() * workspace.element_size()
    _check(lib().latent_append(ctypes.byref(dims), int(d_model), _ptr(h), _ptr(W_DKV), _ptr(W_KR), _ptr(pos),
                               _ptr(page_table), _ptr(latent_cache), _ptr(rope_cache), _ptr(workspace), nbytes,
                               _stream(stream)))


def latent_store(dims, n_tokens, c_kv, k_rope, tok_seq, tok_pos, page_table, latent_cache, rope_cache, workspace,
                 workspace_nbytes=None, stream=None):
    nbytes = workspace_nbytes if workspace_nbytes is not None else workspace.numel() * workspace.element_size()
    _check(lib().latent_store(ctypes.byref(dims), int(n_tokens), _ptr(c_kv), _ptr(k_rope), _ptr(tok_seq),
                              _ptr(tok_pos), _ptr(page_table), _ptr(latent_cache), _ptr(rope_cache),
                              _ptr(workspace), nbytes, _stream(stream)))


def latent_append_noalloc(dims, d_model, h, W_DKV, W_KR, pos, page_table, latent_cache, rope_cache, stream=None):
    """latent_append without a workspace, for callers that cannot allocate
    device memory; its scratch is a fixed array inside the library (see
    include/mlra.h for the size limit and the sharing rules)."""
    _check(lib().latent_append_noalloc(ctypes.byref(dims), int(d_model), _ptr(h), _ptr(W_DKV), _ptr(W_KR),
                                       _ptr(pos), _ptr(page_table), _ptr(latent_cache), _ptr(rope_cache),
                                       _stream(stream)))


def check_status(workspace, stream=None) -> None:
    _check(lib().mlra_check_status(_ptr(workspace), _stream(stream)))


def selftest_wait_timeout(workspace, limit_cycles: int, stream=None) -> None:
    """Runs the bounded-wait self-test kernel (see include/mlra.h); read the outcome with check_status."""
    _check(lib().mlra_selftest_wait_timeout(_ptr(workspace), int(limit_cycles), _stream(stream)))


def version() -> int:
    return int(lib().mlra_version())
