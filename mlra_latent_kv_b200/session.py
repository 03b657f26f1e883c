"""Device state of one decode workload, driven through the C ABI.

A DecodeSession uploads a workload's inputs, builds the paged cache with
``latent_store`` (after poisoning every slot with NaN, so that a read of an
unwritten slot shows up in the output), and runs decode steps
(``latent_append`` first when the workload appends, then ``mlra_decode``).
PyTorch is used for device memory and the stream only.
"""
from __future__ import annotations

import torch

from . import abi
from .synth import PAGE_SIZE, Workload, nan_bits

_UPLOAD_ROWS = 1 << 17


def torch_dtype(w: Workload):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


class DecodeSession:
    def __init__(self, w: Workload, inp: dict, device="cuda", kernel: str = "auto", num_splits: int = 0,
                 poison: bool = True):
        self.w = w
        self.device = torch.device(device)
        dev = self.device
        tdt = torch_dtype(w)
        self.num_pages = int(inp["num_pages"])
        self.maxp = int(inp["page_table"].shape[1])
        self.dims = abi.make_dims(B=w.B, H=w.H, d_h=w.d_h, d_v=w.d_v, d_c=w.d_c, d_r=w.d_r,
                                  max_pages_per_seq=self.maxp, num_pages=self.num_pages, n_branch=w.n_branch,
                                  branch_scale=w.branch_scale, rope_base=w.rope_base, dtype=w.dtype,
                                  num_splits=num_splits, kernel=kernel)
        self.q_nope = inp["q_nope"].to(dev)
        self.q_rope = inp["q_rope"].to(dev)
        self.q_pos = inp["q_pos"].to(dev)
        self.W_UK = inp["W_UK"].to(dev)
        self.W_UV = inp["W_UV"].to(dev)
        self.page_table = inp["page_table"].to(dev)
        self.seq_lens = inp["attn_lens"].to(dev)
        itype = torch.int16 if w.dtype == "bf16" else torch.int32
        self.latent_cache = torch.empty((self.num_pages, PAGE_SIZE, w.d_c), dtype=tdt, device=dev)
        self.rope_cache = torch.empty((self.num_pages, PAGE_SIZE, w.d_r), dtype=tdt, device=dev)
        if poison:
            bits = nan_bits(w.dtype)
            if w.dtype == "bf16":
                bits = bits - (1 << 16) if bits >= (1 << 15) else bits
            self.latent_cache.view(itype).fill_(bits)
            self.rope_cache.view(itype).fill_(bits)
        else:
            self.latent_cache.zero_()
            self.rope_cache.zero_()
        self.ws_bytes = abi.workspace_bytes(self.dims)
        self.workspace = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.out = torch.empty((w.B, w.H, w.d_v), dtype=tdt, device=dev)
        self._store(inp)
        self.appends = bool(w.append_d_model)
        if self.appends:
            self.d_model = w.append_d_model
            self.h = inp["h"].to(dev)
            self.W_DKV = inp["W_DKV"].to(dev)
            self.W_KR = inp["W_KR"].to(dev)
            self.pos = inp["pos"].to(dev)
            self.app_ws = torch.zeros(abi.append_workspace_bytes(self.dims, self.d_model), dtype=torch.uint8,
                                      device=dev)
        abi.check_status(self.workspace)

    def _store(self, inp: dict):
        T = int(inp["c_kv"].shape[0])
        for r0 in range(0, T, _UPLOAD_ROWS):
            r1 = min(T, r0 + _UPLOAD_ROWS)
            c = inp["c_kv"][r0:r1].to(self.device)
            k = inp["k_rope"][r0:r1].to(self.device)
            ts = inp["tok_seq"][r0:r1].to(self.device)
            tp = inp["tok_pos"][r0:r1].to(self.device)
            abi.latent_store(self.dims, r1 - r0, c, k, ts, tp, self.page_table, self.latent_cache,
                             self.rope_cache, self.workspace)
        torch.cuda.synchronize(self.device)

    def append(self, stream=None):
        abi.latent_append(self.dims, self.d_model, self.h, self.W_DKV, self.W_KR, self.pos, self.page_table,
                          self.latent_cache, self.rope_cache, self.app_ws, stream=stream)

    def decode(self, stream=None, events=None):
        if events is not None:
            abi.mlra_decode_profiled(self.dims, self.q_nope, self.q_rope, self.q_pos, self.W_UK, self.W_UV,
                                     self.latent_cache, self.rope_cache, self.page_table, self.seq_lens, self.out,
                                     self.workspace, events, stream=stream)
        else:
            abi.mlra_decode(self.dims, self.q_nope, self.q_rope, self.q_pos, self.W_UK, self.W_UV,
                            self.latent_cache, self.rope_cache, self.page_table, self.seq_lens, self.out,
                            self.workspace, stream=stream)

    def quantize_fp8(self, stream=None):
        """Quantize the cache pools to FP8 E4M3 with per-page scales (mlra_quantize_pages_fp8) and size
        the CUDA-core workspace that mlra_decode_fp8 needs."""
        dev = self.device
        self.lat8 = torch.empty(self.latent_cache.shape, dtype=torch.uint8, device=dev)
        self.rop8 = torch.empty(self.rope_cache.shape, dtype=torch.uint8, device=dev)
        self.lat_scale = torch.empty(self.num_pages, dtype=torch.float32, device=dev)
        self.rop_scale = torch.empty(self.num_pages, dtype=torch.float32, device=dev)
        abi.quantize_pages_fp8(self.dims, self.latent_cache, self.rope_cache, self.lat8, self.rop8, self.lat_scale,
                               self.rop_scale, stream=stream)
        d = self.dims
        self.dims_fp8 = abi.make_dims(B=d.B, H=d.H, d_h=d.d_h, d_v=d.d_v, d_c=d.d_c, d_r=d.d_r,
                                      max_pages_per_seq=d.max_pages_per_seq, num_pages=d.num_pages,
                                      n_branch=d.n_branch, branch_scale=d.branch_scale, rope_base=d.rope_base,
                                      dtype=self.w.dtype, num_splits=d.num_splits, kernel="simt")
        self.ws_fp8 = torch.zeros(abi.workspace_bytes(self.dims_fp8), dtype=torch.uint8, device=dev)

    def decode_fp8(self, stream=None):
        """One decode over the FP8 pools made by quantize_fp8 (into self.out)."""
        abi.decode_fp8(self.dims_fp8, self.q_nope, self.q_rope, self.q_pos, self.W_UK, self.W_UV, self.lat8, self.rop8,
                       self.lat_scale, self.rop_scale, self.page_table, self.seq_lens, self.out, self.ws_fp8,
                       stream=stream)

    def decode_host(self, h_q_nope, h_q_rope, h_q_pos, h_seq_lens, h_out, stream=None):
        """One decode through the host-buffer entry point (inputs in, output out, on `stream`)."""
        if getattr(self, "host_ws", None) is None:
            self.host_ws = torch.zeros(abi.host_workspace_bytes(self.dims), dtype=torch.uint8, device=self.device)
        abi.mlra_decode_host(self.dims, h_q_nope, h_q_rope, h_q_pos, self.W_UK, self.W_UV, self.latent_cache,
                             self.rope_cache, self.page_table, h_seq_lens, h_out, self.host_ws, stream=stream)

    def step(self, stream=None, events=None):
        """One decode step: append the new token (if the workload does), then attend."""
        if self.appends:
            self.append(stream)
        self.decode(stream, events)
        return self.out

    def check(self):
        abi.check_status(self.workspace)
        if getattr(self, "host_ws", None) is not None:
            abi.check_status(self.host_ws)
        if self.appends:
            abi.check_status(self.app_ws)

    def append_kernels(self) -> int:
        """Kernels one latent_append launches: one for the one-launch form,
        whose workspace is the 256-byte error record alone, two for the
        two-kernel form (partial sums in the workspace, then the finalize)."""
        if not self.appends:
            return 0
        return 1 if abi.append_workspace_bytes(self.dims, self.d_model) == 256 else 2

    def kernels_per_step(self) -> int:
        """Kernels one step launches: the append's (when it appends) plus the
        decode call's own launches, as the library plans them."""
        return self.append_kernels() + abi.describe_plan(self.dims)["kernels"]

    def plan(self) -> dict:
        """The decode call's kernel plan (family and per-stage kernel names)."""
        return abi.describe_plan(self.dims)
