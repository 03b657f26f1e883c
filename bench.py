"""Decode-step benchmark of the latent-KV (MLA / MLRA-n) hot path on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|INDEX] [--impl ours|reference]

One step = the whole hot path of one decode step over one batch: latent_append
(when the workload appends a token) -> query absorption -> split-KV latent
attention -> split combine -> output up-projection, all through the C ABI.
Inputs are seeded synthetic tensors resident in HBM; L2 is flushed (256 MiB
write) before every timed step; each step is timed with CUDA events on the
launching stream and the job time is the max over ranks.  With N > 1 (one
process per GPU, torchrun) every rank decodes its own batch: weak scaling, no
data-path collective.

The default workload is the paged variable-length batch at H = 32 (the
largest single-GPU workload); the same run also times the split-KV attention
kernel of the MLRA-4 workload (reported under roofline_by_workload).

--impl reference times the fp64 CPU oracle on the host cores instead (a
bounded sample of (sequence, head) pairs per step, extrapolated to the step),
with the same sampler as the cpu_baseline leg.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mlra_latent_kv_b200 import dist as mdist  # noqa: E402
from mlra_latent_kv_b200 import synth  # noqa: E402

METRIC = "latent decode attention µs/step, achieved HBM GB/s and % of 1×B200 roofline"
DEFAULT_WORKLOAD = "paged_varlen_h32"
COMPANION_WORKLOADS = ("mlra4",)   # attention roofline also reported for these (1-GPU runs)
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def step_bytes(w, inp) -> dict:
    """Algorithmic HBM bytes of one step: every cached token attended once,
    the absorption and up-projection weights once, the append weights once."""
    e = 2 if w.dtype == "bf16" else 4
    tokens = int(inp["attn_lens"].sum())
    cache = tokens * (w.d_c + w.d_r) * e
    weights = 2 * w.H * w.d_h * w.d_c * e if w.d_h == w.d_v else w.H * w.d_c * (w.d_h + w.d_v) * e
    app = w.append_d_model * (w.d_c + w.d_r) * e if w.append_d_model else 0
    # algorithmic attention flops: QK over d_c + d_r (rope counted once) and PV over d_c
    flops = 2 * w.H * tokens * (w.d_c + w.d_r + w.d_c)
    return dict(tokens=tokens, cache=cache, weights=weights, append=app, total=cache + weights + app,
                attn_flops=flops)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - clocks are reported as unknown
            self._nv = None
            return self
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()
        return self

    def _run(self):
        nv = self._nv
        names = {getattr(nv, k): k for k in dir(nv) if k.startswith("nvmlClocksEventReason") and
                 isinstance(getattr(nv, k), int) and k not in ("nvmlClocksEventReasonNone", "nvmlClocksEventReasonAll")}
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in names.items():
                    if r & bit:
                        self.reasons.add(name.replace("nvmlClocksEventReason", ""))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()
        return False

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples), "reasons": sorted(self.reasons)}


ATTN_SOURCES = ("attn_tc.cu", "attn_small.cu", "attn_branch.cu", "attn_common.cuh", "attn_tc.h", "ptx.cuh",
                "common.cuh", "launch.h", "host_cache.cu", "host_cache.h")


def source_digest() -> str:
    """Digest of the code the attention kernel is built from, with `//`
    comments and blank lines left out (a stored ncu traffic figure is used
    only while it matches; a comment does not change the kernel)."""
    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        with open(os.path.join(ROOT, "mlra_latent_kv_b200", "csrc", name), encoding="utf-8") as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode("utf-8") + b"\n")
    return h.hexdigest()[:16]


def captured_traffic(workload: str):
    """DRAM bytes per attention launch from the committed ncu capture, if it
    was taken on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("source_digest") != source_digest():
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# oracle timing (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def host_cores() -> int:
    """Host cores this process may run on (the oracle's thread pool size)."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


class OracleSampler:
    """Times the fp64 oracle, as it stands, on random (sequence, head) pairs of
    one workload step: the pairs are split into chunks that a pool of one
    thread per host core runs through ``oracle.decode`` (its BLAS calls held
    to one thread each, so the pool is the parallelism).  The wall time of a
    sample scales to a full step by B*H / pairs."""

    def __init__(self, w, inp):
        import oracle
        from oracle.inputs import oracle_inputs
        self._decode = oracle.decode
        self.w = w
        self.oi = oracle_inputs(w, inp)
        self.cores = host_cores()
        self.total = w.B * w.H

    def pairs(self, n, seed):
        rng = np.random.default_rng(12345 + seed)
        idx = rng.choice(self.total, size=n, replace=False)
        return [(int(i) // self.w.H, int(i) % self.w.H) for i in idx]

    def time(self, pairs) -> float:
        from threadpoolctl import threadpool_limits
        n_chunks = min(len(pairs), 4 * self.cores)
        chunks = [pairs[i::n_chunks] for i in range(n_chunks)]
        with threadpool_limits(1), ThreadPoolExecutor(self.cores) as ex:
            t0 = time.perf_counter()
            list(ex.map(lambda c: self._decode(self.oi, c), chunks))
            return time.perf_counter() - t0

    def grow(self, budget_s, seed=1):
        """Sample size whose timing takes at least half of budget_s (or the whole
        step); returns (pairs, seconds)."""
        n = min(self.total, 4 * self.cores)
        t = self.time(self.pairs(n, seed))
        while t < 0.5 * budget_s and n < self.total:
            n = min(self.total, max(n + 1, int(n * budget_s / max(t, 1e-3))))
            t = self.time(self.pairs(n, seed))
        return n, t

    def sample_text(self, n):
        return (f"{n} random (sequence, head) pairs of the {self.w.name} step per timing, run by "
                f"{self.cores} threads (one per host core, BLAS single-threaded), scaled by "
                f"{self.total}/{n} to one step")


def cpu_baseline(w, inp, budget_s: float = 15.0) -> dict:
    """The oracle (as it stands) on a bounded sample of (b, h) pairs, scaled to a full step."""
    smp = OracleSampler(w, inp)
    smp.time(smp.pairs(min(smp.total, smp.cores), seed=6))  # first-touch costs are not the oracle's rate
    n, t = smp.grow(budget_s)
    step_s = t * smp.total / n
    sb = step_bytes(w, inp)
    return {"value": sb["total"] / step_s / 1e9, "unit": "GB/s", "cores": smp.cores, "kind": "oracle",
            "sample": smp.sample_text(n) + f" ({t:.1f} s for the sample, {step_s:.1f} s/step)",
            "s_per_step": step_s}


def run_reference(args, w):
    rank, ws, _ = mdist.world()
    if rank != 0:
        return 0
    inp = synth.make_inputs(w)
    sb = step_bytes(w, inp)
    smp = OracleSampler(w, inp)
    # the cpu_baseline leg's sampler and growth rule, with a per-step budget that keeps the
    # whole --steps/--warmup run to a few minutes
    budget = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    n, _ = smp.grow(budget, seed=99)
    for i in range(args.warmup):
        smp.time(smp.pairs(n, seed=100 + i))
    tot = 0.0
    for i in range(args.steps):
        tot += smp.time(smp.pairs(n, seed=1000 + i))
    step_s = tot / args.steps * smp.total / n
    value = sb["total"] / step_s / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, inp, args.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": smp.cores, "kind": "oracle",
                         "sample": smp.sample_text(n) + "; one fresh sample per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, inp, n):
    lens = inp["attn_lens"]
    return {"workload": w.name, "B": w.B, "H": w.H, "d_h": w.d_h, "d_v": w.d_v, "d_c": w.d_c, "d_r": w.d_r,
            "n_branch": w.n_branch, "branch_scale": w.branch_scale,
            "seq_len": int(lens[0]) if bool((lens == lens[0]).all()) else
            {"min": int(lens.min()), "max": int(lens.max()), "mean": float(lens.float().mean())},
            "tokens_attended": int(lens.sum()), "paged": w.paged, "append_d_model": w.append_d_model,
            "dtype": w.dtype, "parallelism": f"replica x{n} (independent batches per GPU)",
            "l2": "flushed: 256 MiB written before every timed step"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def roofline_of(sb, attn_us, peaks, src) -> dict:
    """Roofline of the split-KV attention kernel from its event-timed duration:
    the bound is whichever of cache bytes / HBM peak and attention flops /
    bf16 tensor peak is longer (burst peaks: the kernel is timed on its own,
    well under a second); achieved, peak and frac are reported for that bound,
    the other pipe's figures beside them."""
    hbm = float(peaks["hbm_gbs"])
    tc = float(peaks["bf16_tflops"])
    attn_s = attn_us * 1e-6
    t_hbm = sb["cache"] / (hbm * 1e9)
    t_tc = sb["attn_flops"] / (tc * 1e12)
    gbs = sb["cache"] / attn_s / 1e9
    tfs = sb["attn_flops"] / attn_s / 1e12
    hbm_bound = t_hbm >= t_tc
    note = "of measured" if src == "measured" else "of fallback"
    return {"kernel": "split-KV latent attention", "bound": "hbm" if hbm_bound else "tensor",
            "achieved": gbs if hbm_bound else tfs, "peak": hbm if hbm_bound else tc,
            "unit": "GB/s" if hbm_bound else "TFLOP/s", "frac": (gbs / hbm) if hbm_bound else (tfs / tc),
            "peak_source": f"{note} (MEASURED_PEAKS.json hbm_gbs / bf16_tflops burst)",
            "algorithmic_bytes_per_launch": sb["cache"], "algorithmic_flops_per_launch": sb["attn_flops"],
            "attn_us": attn_us, "hbm_gbs": gbs, "hbm_frac": gbs / hbm, "tensor_tflops": tfs, "tensor_frac": tfs / tc,
            "tensor_peak_tflops": tc, "hbm_peak_gbs": hbm,
            "roofline_us": max(t_hbm, t_tc) * 1e6, "frac_of_roofline_time": max(t_hbm, t_tc) / attn_s}


def _events(n):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def staged_timing(sess, stream, flush, K, W, graph=True):
    """Per-stage device times (µs, mean over K steps) of one decode step with
    events recorded between its kernels (which serialises them), L2 flushed
    before every step."""
    stage = _events(5)
    for e in stage:  # materialise the raw events before handing them to the library
        e.record(stream)
    # the step's first event, recorded inside the captured step (an event record node), so that the
    # append stage does not include the graph's launch latency
    first = torch.cuda.Event(enable_timing=True, external=True)
    first.record(stream)

    def staged_step():
        first.record()  # on the current stream: the capture stream while the graph is captured
        sess.step(events=stage)

    g = None
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            staged_step()
    for _ in range(W):
        flush.fill_(3)
        g.replay() if g else staged_step()
    torch.cuda.synchronize()
    acc = {"absorb": 0.0, "attention": 0.0, "combine": 0.0, "upproj_incl_fused_combine": 0.0,
           "launch_to_first_kernel": 0.0}
    if sess.appends:
        acc["append"] = 0.0
    starts = _events(K)
    for i in range(K):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        g.replay() if g else staged_step()
        stage[4].synchronize()
        for name, a, b in (("absorb", 0, 1), ("attention", 1, 2), ("combine", 2, 3),
                           ("upproj_incl_fused_combine", 3, 4)):
            acc[name] += stage[a].elapsed_time(stage[b])
        acc["launch_to_first_kernel"] += starts[i].elapsed_time(first)
        if sess.appends:
            acc["append"] += first.elapsed_time(stage[0])
    torch.cuda.synchronize()
    del g
    out = {k: v / K * 1e3 for k, v in acc.items()}
    if sess.plan().get("combine", "").startswith("fused"):
        # no kernel runs between events 2 and 3: what they measure is the cost
        # of two back-to-back event records, which every stage above includes
        out["event_gap_no_kernel"] = out.pop("combine")
    return out


def run_ours(args, w):
    from mlra_latent_kv_b200.session import DecodeSession
    rank, ws, local = mdist.world()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    mdist.init("nccl" if ws > 1 else "gloo")
    wr = w.with_(seed=mdist.rank_seed(w.seed, rank))
    inp = synth.make_inputs(wr)
    sess = DecodeSession(wr, inp, device=dev, kernel=args.kernel)
    sb = step_bytes(wr, inp)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    K, W = args.steps, args.warmup
    starts, ends = _events(K), _events(K)
    for _ in range(W):
        flush.fill_(1)
        sess.step()
    torch.cuda.synchronize(dev)
    sess.check()
    # The headline pass replays one decode step captured as a CUDA graph (its
    # kernels chained by programmatic dependent launches); a second timed pass
    # (staged_timing) records events between the kernels for the per-kernel
    # times and the attention roofline.
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            sess.step()
        for _ in range(W):
            flush.fill_(1)
            graph.replay()
        torch.cuda.synchronize(dev)

    mdist.barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(K):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            graph.replay() if graph is not None else sess.step()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        mdist.barrier(dev)
        stage_us = staged_timing(sess, stream, flush, K, W, graph=not args.no_graph)
    mdist.barrier(dev)
    torch.cuda.synchronize(dev)
    sess.check()
    del graph

    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(step_ms)
    max_total_ms = mdist.max_over_ranks(total_ms, dev)
    value = mdist.throughput(sb["total"] * K, ws, max_total_ms / 1e3) / 1e9

    # end to end through the public API with host buffers: every step hands pinned host
    # inputs to the library (mlra_decode_host copies them in, decodes and copies the output
    # back on the stream; an appending step first copies h and pos and calls latent_append)
    host = {k: inp[k].pin_memory() for k in ("q_nope", "q_rope", "q_pos")}
    host["seq_lens"] = inp["attn_lens"].pin_memory()
    app_host = {}
    if sess.appends:
        app_host = {"h": inp["h"].pin_memory(), "pos": inp["pos"].pin_memory()}
    out_host = torch.empty(sess.out.shape, dtype=sess.out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in list(host.values()) + list(app_host.values()))
    d2h = out_host.numel() * out_host.element_size()

    def e2e_step():
        if sess.appends:
            sess.h.copy_(app_host["h"], non_blocking=True)
            sess.pos.copy_(app_host["pos"], non_blocking=True)
            sess.append()
        sess.decode_host(host["q_nope"], host["q_rope"], host["q_pos"], host["seq_lens"], out_host)

    # the same host<->device copies alone, for the split of the e2e step
    dev_in = {k: torch.empty_like(v, device=dev) for k, v in list(host.items()) + list(app_host.items())}
    dev_out = torch.empty(sess.out.shape, dtype=sess.out.dtype, device=dev)

    def copies_only():
        for k, v in list(host.items()) + list(app_host.items()):
            dev_in[k].copy_(v, non_blocking=True)
        out_host.copy_(dev_out, non_blocking=True)

    e_s, e_e = _events(K), _events(K)
    for _ in range(W):
        flush.fill_(2)
        e2e_step()
    torch.cuda.synchronize(dev)
    mdist.barrier(dev)
    for i in range(K):
        flush.fill_(i & 0xFF)
        e_s[i].record(stream)
        e2e_step()
        e_e[i].record(stream)
    torch.cuda.synchronize(dev)
    sess.check()
    e2e_ms = mdist.max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(e_s, e_e)), dev)
    e2e_value = mdist.throughput(sb["total"] * K, ws, e2e_ms / 1e3) / 1e9
    c_s, c_e = _events(K), _events(K)
    for i in range(K):
        c_s[i].record(stream)
        copies_only()
        c_e[i].record(stream)
    torch.cuda.synchronize(dev)
    copy_ms = sum(a.elapsed_time(b) for a, b in zip(c_s, c_e)) / K

    peaks, src = load_peaks()
    roof = roofline_of(sb, stage_us["attention"], peaks, src)
    roof["traffic"] = captured_traffic(w.name)
    plan = sess.plan()
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": W,
        "ms_per_step": max_total_ms / K, "us_per_step": max_total_ms / K * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded per workload, shapes of the workload configuration)",
        "config": config_of(w, inp, ws),
        "stage_us": stage_us,
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "mlra_decode_host (host buffers; copies inside the timed region)",
                "ms_per_step": e2e_ms / K,
                "copies_alone_ms_per_step": copy_ms},
        "gpu_launches": K * sess.kernels_per_step(),
        "kernels": plan,
        "timed_as": ("eager API calls" if args.no_graph else "CUDA graph replay of one decode step per timed step")
                    + "; stage_us and roofline from a second timed pass with events between the kernels",
        "clocks": clk.summary(),
        "step_bytes": sb,
    }
    del sess
    torch.cuda.empty_cache()

    # the split-KV attention of the other target workloads, timed the same way (1-GPU runs)
    if ws == 1 and not args.no_companions:
        by = {}
        for name in COMPANION_WORKLOADS:
            if name == w.name:
                continue
            cw = synth.workload(name)
            cinp = synth.make_inputs(cw)
            cs = DecodeSession(cw, cinp, device=dev, kernel=args.kernel)
            with ClockSampler(local) as cclk:
                cst = staged_timing(cs, stream, flush, min(K, 50), W, graph=not args.no_graph)
            cs.check()
            csb = step_bytes(cw, cinp)
            r = roofline_of(csb, cst["attention"], peaks, src)
            r["traffic"] = captured_traffic(name)
            by[name] = {"roofline": r, "stage_us": cst, "kernels": cs.plan(), "clocks": cclk.summary(),
                        "config": config_of(cw, cinp, ws)}
            del cs
            torch.cuda.empty_cache()
        line["roofline_by_workload"] = by

    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wr, inp)
    elif rank == 0:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    mdist.shutdown()
    return 0


def run_fp8(args, w):
    """The step over an FP8 E4M3 cache (one fp32 scale per page and tensor), quantized from the workload's
    bf16 cache by mlra_quantize_pages_fp8 and decoded by mlra_decode_fp8 on the CUDA-core kernels.
    Timed as whole steps (no stage events in that entry point); the roofline is the one of the FP8 cache
    bytes, half of the bf16 ones, against the whole step's time."""
    from mlra_latent_kv_b200 import abi
    from mlra_latent_kv_b200.session import DecodeSession
    rank, ws, local = mdist.world()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    mdist.init("nccl" if ws > 1 else "gloo")
    wr = w.with_(seed=mdist.rank_seed(w.seed, rank))
    if wr.append_d_model:
        raise SystemExit("--cache fp8 takes a workload without append")
    inp = synth.make_inputs(wr)
    sess = DecodeSession(wr, inp, device=dev)
    sess.quantize_fp8()
    sb = step_bytes(wr, inp)
    cache8 = sb["tokens"] * (wr.d_c + wr.d_r) + 2 * 4 * int(inp["num_pages"])  # codes + per-page scales
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    K, W = args.steps, args.warmup
    for _ in range(W):
        flush.fill_(1)
        sess.decode_fp8()
    torch.cuda.synchronize(dev)
    abi.check_status(sess.ws_fp8)
    starts, ends = _events(K), _events(K)
    mdist.barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(K):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            sess.decode_fp8()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / K
    ms = mdist.max_over_ranks(ms, dev)
    peaks, src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    gbs = cache8 / (ms * 1e-3) / 1e9
    plan = abi.describe_plan(sess.dims_fp8)
    line = {
        "metric": "latent decode over an FP8 latent cache: µs/step, achieved HBM GB/s of the FP8 cache bytes",
        "value": (cache8 + sb["weights"]) * ws / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": ws, "steps": K,
        "warmup": W, "ms_per_step": ms, "us_per_step": ms * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8 e4m3 cache, fp32 compute",
        "data": "synthetic (seeded per workload), the bf16 cache quantized per page",
        "config": {"workload": wr.name, "cache": "fp8_e4m3, one fp32 scale per page and tensor", "B": wr.B,
                   "H": wr.H, "d_c": wr.d_c, "d_r": wr.d_r, "n_branch": wr.n_branch,
                   "tokens_attended": sb["tokens"], "l2": "flushed: 256 MiB written before every timed step"},
        "roofline": {"kernel": "whole decode step over the FP8 cache (CUDA-core kernels)", "bound": "hbm",
                     "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "peak_source": ("of measured" if src == "measured" else "of fallback") + " (hbm_gbs)",
                     "algorithmic_bytes_per_launch": cache8, "bf16_cache_bytes": sb["cache"],
                     "roofline_us": cache8 / (hbm * 1e9) * 1e6, "traffic": None},
        "gpu_launches": K * int(plan.get("kernels", 4)), "kernels": plan, "clocks": clk.summary(),
        "timed_as": "eager steps, CUDA events around each step",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    mdist.shutdown()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-companions", action="store_true",
                    help="skip the attention timing of the other target workloads")
    ap.add_argument("--no-graph", action="store_true", help="launch each timed step eagerly instead of as a graph")
    ap.add_argument("--cache", default="bf16", choices=["bf16", "fp8"],
                    help="fp8: time the step over the cache quantized to FP8 E4M3 (CUDA-core kernels)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    name = args.workload
    w = synth.workload(int(name) if name.isdigit() else name)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.cache == "fp8":
        return run_fp8(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
