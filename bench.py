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

--impl reference times the fp64 CPU oracle on the host cores instead (a
bounded sample of (sequence, head) pairs per step, extrapolated to the step).
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mlra_latent_kv_b200 import dist as mdist  # noqa: E402
from mlra_latent_kv_b200 import synth  # noqa: E402

METRIC = "latent decode attention µs/step, achieved HBM GB/s and % of 1×B200 roofline"
DEFAULT_WORKLOAD = "dsv2_contiguous"
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


ATTN_SOURCES = ("attn_tc.cu", "attn_tc.h", "ptx.cuh", "common.cuh", "launch.h", "host_cache.cu", "host_cache.h")


def source_digest() -> str:
    """Digest of the sources the attention kernel is built from (a stored ncu
    traffic figure is used only while it matches)."""
    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        with open(os.path.join(ROOT, "mlra_latent_kv_b200", "csrc", name), "rb") as f:
            h.update(f.read())
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

def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def time_oracle_pairs(w, inp, pairs) -> float:
    import oracle
    from oracle.inputs import oracle_inputs
    oi = oracle_inputs(w, inp)
    t0 = time.perf_counter()
    oracle.decode(oi, pairs)
    return time.perf_counter() - t0


def pick_pairs(w, n, seed=0):
    rng = np.random.default_rng(12345 + seed)
    bs = rng.integers(0, w.B, n)
    hs = rng.integers(0, w.H, n)
    return [(int(b), int(h)) for b, h in zip(bs, hs)]


def cpu_baseline(w, inp, budget_s: float = 15.0) -> dict:
    """The oracle (as it stands) on a bounded sample of (b, h) pairs, scaled to a full step."""
    time_oracle_pairs(w, inp, pick_pairs(w, 8, seed=6))  # warm (first-touch costs are not the oracle's rate)
    # grow the sample until it takes about half the budget or covers the whole step (the
    # oracle's per-pair cost falls with the sample size, so one small calibration overshoots)
    n = min(w.B * w.H, 64)
    t = time_oracle_pairs(w, inp, pick_pairs(w, n, seed=1))
    while t < 0.5 * budget_s and n < w.B * w.H:
        n = min(w.B * w.H, max(n + 1, int(n * budget_s / max(t, 1e-3))))
        t = time_oracle_pairs(w, inp, pick_pairs(w, n, seed=1))
    per_pair = t / n
    step_s = per_pair * w.B * w.H
    sb = step_bytes(w, inp)
    return {"value": sb["total"] / step_s / 1e9, "unit": "GB/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{n} random (sequence, head) pairs of the {w.name} step in {t:.1f} s, "
                      f"scaled by {w.B * w.H}/{n} to one step ({step_s:.1f} s/step)",
            "s_per_step": step_s}


def run_reference(args, w):
    rank, ws, _ = mdist.world()
    if rank != 0:
        return 0
    inp = synth.make_inputs(w)
    sb = step_bytes(w, inp)
    t1 = time_oracle_pairs(w, inp, pick_pairs(w, 1))
    budget = 120.0 / max(1, args.steps + args.warmup)
    per_step = max(1, min(w.B * w.H, int(budget / max(t1, 1e-6))))
    for i in range(args.warmup):
        time_oracle_pairs(w, inp, pick_pairs(w, per_step, seed=100 + i))
    tot = 0.0
    for i in range(args.steps):
        tot += time_oracle_pairs(w, inp, pick_pairs(w, per_step, seed=1000 + i))
    step_s = tot / (args.steps * per_step) * w.B * w.H
    value = sb["total"] / step_s / 1e9
    cores = oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, inp, args.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} random (sequence, head) pairs per step, scaled by "
                                   f"{w.B * w.H}/{per_step} to the full step"},
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

    def mk(n):
        return [torch.cuda.Event(enable_timing=True) for _ in range(n)]

    K, W = args.steps, args.warmup
    starts, ends = mk(K), mk(K)
    stage = mk(5)
    for e in stage:  # materialise the raw events before handing them to the library
        e.record(stream)
    for _ in range(W):
        flush.fill_(1)
        sess.step()
    torch.cuda.synchronize(dev)
    sess.check()
    # One decode step captured as a CUDA graph, replayed once per timed step.
    # The headline pass replays the plain step (its kernels chained by
    # programmatic dependent launches); a second timed pass replays a step with
    # the stage events recorded between the kernels (which also serialises
    # them) for the per-kernel times and the attention roofline.
    graphs = {}
    if not args.no_graph:
        for name, evs in (("plain", None), ("staged", stage)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                sess.step(events=evs)
            for _ in range(W):
                flush.fill_(1)
                g.replay()
            graphs[name] = g
        torch.cuda.synchronize(dev)

    def one_step(staged: bool):
        if graphs:
            graphs["staged" if staged else "plain"].replay()
        else:
            sess.step(events=stage if staged else None)

    stage_acc = {"absorb": 0.0, "attention": 0.0, "combine": 0.0, "upproj_incl_fused_combine": 0.0}
    if sess.appends:
        stage_acc["append"] = 0.0
    mdist.barrier(dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(K):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            one_step(False)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
        mdist.barrier(dev)
        s_starts = mk(K)
        for i in range(K):
            flush.fill_(i & 0xFF)
            s_starts[i].record(stream)
            one_step(True)
            stage[4].synchronize()
            for name, a, b in (("absorb", 0, 1), ("attention", 1, 2), ("combine", 2, 3),
                               ("upproj_incl_fused_combine", 3, 4)):
                stage_acc[name] += stage[a].elapsed_time(stage[b])
            if sess.appends:
                stage_acc["append"] += s_starts[i].elapsed_time(stage[0])
        torch.cuda.synchronize(dev)
    mdist.barrier(dev)
    torch.cuda.synchronize(dev)
    sess.check()

    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(step_ms)
    stage_ms = {k: v / K for k, v in stage_acc.items()}
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

    e_s, e_e = mk(K), mk(K)
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

    peaks, src = load_peaks()
    attn_s = stage_ms["attention"] / 1e3
    hbm_peak = float(peaks["hbm_gbs"])
    achieved = sb["cache"] / attn_s / 1e9
    tflops = sb["attn_flops"] / attn_s / 1e12
    tensor_peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    roofline_t = max(sb["cache"] / (hbm_peak * 1e9), sb["attn_flops"] / (float(peaks["bf16_tflops"]) * 1e12))
    traffic = captured_traffic(w.name)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": W,
        "ms_per_step": max_total_ms / K, "us_per_step": max_total_ms / K * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded per workload, shapes of the workload configuration)",
        "config": config_of(w, inp, ws),
        "stage_us": {k: v * 1e3 for k, v in stage_ms.items()},
        "roofline": {"kernel": "split-KV latent attention", "bound": "hbm", "achieved": achieved,
                     "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": traffic,
                     "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else src,
                     "algorithmic_bytes_per_launch": sb["cache"], "attn_us": stage_ms["attention"] * 1e3,
                     "tensor_tflops": tflops, "tensor_peak_tflops": tensor_peak,
                     "roofline_us": roofline_t * 1e6, "frac_of_roofline_time": roofline_t / attn_s},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "mlra_decode_host (host buffers; copies inside the timed region)",
                "ms_per_step": e2e_ms / K},
        "gpu_launches": K * sess.kernels_per_step(),
        "timed_as": ("eager API calls" if args.no_graph else "CUDA graph replay of one decode step per timed step")
                    + "; stage_us and roofline from a second timed pass with events between the kernels",
        "clocks": clk.summary(),
        "step_bytes": sb,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wr, inp)
    elif rank == 0:
        line["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    del sess
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
    ap.add_argument("--no-graph", action="store_true", help="launch each timed step eagerly instead of as a graph")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    name = args.workload
    w = synth.workload(int(name) if name.isdigit() else name)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
