"""Benchmark of the decode step: query encode + Hamming scan + top-k + sparse
attention + LSE merge, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
                    [--main-only] [--no-cpu-baseline]

One step = one pass of the whole decode path over every layer of the
workload (28 sequential layers for the default Qwen2.5-7B-shaped 512K-token
case), captured in one CUDA graph.  Inputs are synthetic, drawn on the device
(same distributions as the parity tests), and larger than L2: every layer has
its own codes and K/V buffers.  Timing: CUDA events on the launching stream
between consecutive replays after W warm-up replays; the reported step time
is the median replay (the mean is reported beside it), max over ranks.  After
the main workload, every other workload's decode step and fused kernel are
timed the same way and reported under "configs".  With N > 1 (torchrun) each
rank runs its own replica (independent sequences: weak scaling, no
collective on the data path).

--impl reference times the oracle (CPU) on the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch

import synth

L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--prefetch-hint", action="store_true",
                    help="time the step with each layer passing the next layer's codes as the L2 prefetch hint")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="qwen7b_512k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="hkv", choices=["hkv", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0)
    ap.add_argument("--split", action="store_true",
                    help="token split: one sequence per layer cut across the ranks (decode_step_split, "
                         "NCCL all-gathers), strong scaling")
    ap.add_argument("--main-only", action="store_true",
                    help="measure only --workload (skip the other workloads' decode steps)")
    ap.add_argument("--layers", type=int, default=0,
                    help="number of layer buffers (default: the workload's layers, at least 3x L2 of data); "
                         "a small value makes a small case for profiling")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world, local, backend="nccl"):
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, ms_local: float, world: int, device):
    """Whole-job throughput: every rank processes units_per_rank_step per step;
    the step time is the slowest rank's.  Returns (units/s, max ms)."""
    ms = max_over_ranks(ms_local, world, device)
    return units_per_rank_step * world / (ms * 1e-3), ms


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_tflops():
    """Burst dense bf16 peak (a kernel timed alone)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def encode_roofline(w: synth.Workload, n_layers: int, encode_ms: float):
    """Prefill key encode: LSH and sign are bound by HBM (keys in, codes out),
    the MLP hash by the tensor cores (2 (d hidden + hidden bits) flops a key)."""
    keys = w.B * w.Hkv * w.N * n_layers
    elt = 2 if w.dtype == "bf16" else 4
    sec = encode_ms * 1e-3
    out = {"keys_per_s": keys / sec, "ms_all_layers": encode_ms,
           "gbs": keys * (w.d * elt + w.bits // 8) / sec / 1e9}
    if w.hash == "mlp":
        peak, kind = measured_bf16_tflops()
        tf = keys * 2.0 * (w.d * w.hidden + w.hidden * w.bits) / sec / 1e12
        out.update({"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                    "peak_kind": kind})
    else:
        peak, kind = measured_peaks()
        out.update({"bound": "hbm", "achieved": out["gbs"], "peak": peak, "unit": "GB/s", "frac": out["gbs"] / peak,
                    "peak_kind": kind})
    return out


class ClockSampler:
    """SM clock and clock-event reasons, polled through NVML every few
    milliseconds on a thread while the timed region runs (read-only queries)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, device_index: int, period_s: float = 0.004):
        self.device_index = device_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.error = None

    def _handle(self, nv):
        props = torch.cuda.get_device_properties(self.device_index)
        uuid = getattr(props, "uuid", None)
        if uuid is not None:
            try:
                return nv.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
            except Exception:  # noqa: BLE001 - fall back to the ordinal
                pass
        return nv.nvmlDeviceGetHandleByIndex(self.device_index)

    def _poll(self, nv, h):
        import time
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), int(get_reasons(h))))
            except Exception as e:  # noqa: BLE001
                self.error = str(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 - no NVML: report no samples
            self.error = str(e)
            self._thread = None
            return self
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)

    def summary(self):
        sm = [c for c, _ in self.samples]
        reasons = sorted({n for _, r in self.samples for n, bit in self.REASONS.items() if r & bit})
        out = {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz, "reasons": reasons,
               "samples": len(sm), "source": "nvml"}
        if self.error and not sm:
            out["error"] = self.error
        return out


# ------------------------------------------------------------------ GPU arm --

class Layer:
    """Device buffers of one layer: inputs, key codes, outputs."""

    def __init__(self, w: synth.Workload, layer: int, dev, hkv):
        inp = synth.device_layer_inputs(w, layer, dev)
        self.q, self.K, self.V = inp["q"], inp["K"], inp["V"]
        code = hkv.HKV_BF16 if w.dtype == "bf16" else hkv.HKV_F32
        if w.hash == "lsh":
            self.R = inp["R"]
            self.kh = self.qh = hkv.HashParams.lsh(self.R)
        elif w.hash == "mlp":
            self.kmlp, self.qmlp = inp["k_mlp"], inp["q_mlp"]
            self.kh = hkv.HashParams.mlp(*self.kmlp, dtype=code)
            self.qh = hkv.HashParams.mlp(*self.qmlp, dtype=code)
        else:
            self.kh = self.qh = hkv.HashParams.sign(code)
        self.codes = torch.empty(w.B, w.Hkv, w.N, w.words, dtype=torch.int32, device=dev)
        self.norms = torch.empty(w.B, w.Hkv, w.N, dtype=torch.float16, device=dev) if w.hash == "sign" else None
        self.q_codes = torch.empty(w.B, w.Hq, w.words, dtype=torch.int32, device=dev)
        self.idx = torch.empty(w.B, w.Hkv, w.top_k, dtype=torch.int32, device=dev)
        self.out = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=dev)

    def encode_keys(self, hkv):
        hkv.hkv_encode_keys(self.kh, self.K.view(-1, self.K.shape[-1]), self.codes.view(-1, self.codes.shape[-1]),
                            None if self.norms is None else self.norms.view(-1))


def paged_roofline(w: synth.Workload, n_layers: int, ms: float, step_ms: float, page: int, peak: float,
                   peak_kind: str) -> dict:
    """Paged cache: the retrieval launch (fused scan + select through the page
    table; the candidates' codes are its algorithmic bytes, the page table is
    negligible) and the paged decode step (the layer's algorithmic bytes)."""
    nbytes = w.B * w.Hkv * w.candidates() * w.bits // 8
    launch_s = ms * 1e-3 / n_layers
    step_s = step_ms * 1e-3 / n_layers
    return {"kernel": "fused_kernel, paged (retrieval only: scan + select through the page table)",
            "page_size": page, "bound": "hbm", "achieved": nbytes / launch_s / 1e9, "peak": peak, "unit": "GB/s",
            "frac": nbytes / launch_s / 1e9 / peak, "bytes_per_launch": nbytes, "launch_us": launch_s * 1e6,
            "step_us_per_layer": step_s * 1e6, "step_frac": w.algorithmic_bytes() / step_s / 1e9 / peak,
            "launches_per_layer": 1 if w.hash in ("lsh", "sign") else 2, "peak_kind": peak_kind, "traffic": None}


def normw_bytes_step(w: synth.Workload) -> int:
    """Algorithmic bytes of one norm-weighted decode step on one layer: codes and norms of every candidate,
    the K and V rows of the selected, sink and local tokens, the queries and the fp32 outputs."""
    elt = 2 if w.dtype == "bf16" else 4
    rows = w.B * w.Hkv * (min(w.top_k, w.candidates()) + w.n_sink + w.n_local)
    return (w.B * w.Hkv * w.candidates() * (w.bits // 8 + 2) + rows * w.d * 2 * elt
            + w.B * w.Hq * w.d * elt + w.B * w.Hq * w.d * 4)


def normw_roofline(w: synth.Workload, n_layers: int, ms: float, step_ms: float, peak: float, peak_kind: str) -> dict:
    """Norm-weighted sign-VQ retrieval: codes and fp16 norms of every candidate
    are the algorithmic bytes of one launch."""
    nbytes = w.B * w.Hkv * w.candidates() * (w.bits // 8 + 2)
    launch_s = ms * 1e-3 / n_layers
    return {"kernel": "normw_kernel (scan, lists at the threshold bin, select, ordered compaction)", "bound": "hbm",
            "achieved": nbytes / launch_s / 1e9, "peak": peak, "unit": "GB/s",
            "frac": nbytes / launch_s / 1e9 / peak, "bytes_per_launch": nbytes, "launch_us": launch_s * 1e6,
            "step_us_per_layer": step_ms * 1e3 / n_layers, "launches_per_layer": 3,
            "step": "query encode + norm-weighted retrieval + sparse attention (three launches); "
                    "decode_step_us_per_layer: hkv_decode_step_normw (one launch)", "peak_kind": peak_kind,
            "traffic": traffic_record([os.path.join(ROOT, "hash_sparse_kv_b200", "csrc", f)
                                       for f in ("normw.cu", "normw_select.cuh")], w.name)}


def graph_of(fn, warm=1):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(warm):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def time_graph(g, steps, warmup, world):
    """Replays g: W untimed warm-up replays, then K timed replays bracketed by
    a barrier and a synchronize on both sides, with CUDA events recorded on
    the launching stream between consecutive replays.  Returns (mean ms,
    median ms) per replay; the max over ranks is taken by the caller."""
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        g.replay()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    return ev[0].elapsed_time(ev[-1]) / steps, statistics.median(per)


def timed_ms(g, args, world, dev):
    """Median ms per replay, max over ranks."""
    return max_over_ranks(time_graph(g, args.steps, args.warmup, world)[1], world, dev)


def source_digest(paths):
    """First 16 hex digits of the SHA-256 of the files' contents, concatenated in order."""
    h = hashlib.sha256()
    for path in [paths] if isinstance(paths, str) else paths:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel_files, workload: str):
    """DRAM traffic per launch from the committed ncu summary, if it was taken
    on the current source of the kernel (one file, or the list of files its
    code lives in, keyed by the first one's name); else None."""
    files = [kernel_files] if isinstance(kernel_files, str) else list(kernel_files)
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(workload, {}).get(os.path.basename(files[0]))
    if not rec or rec.get("source_sha256_16") != source_digest(files):
        return None
    return rec.get("bytes_per_launch")


def build_layers(w: synth.Workload, dev, hkv, n_layers: int):
    """Device buffers of n_layers layers.  The layers' query rows live in one
    contiguous tensor and their outputs in another, so the end-to-end step
    moves them with one copy each way."""
    layers = [Layer(w, l % w.layers if w.layers > 1 else 0, dev, hkv) for l in range(n_layers)]
    q_all = torch.empty((n_layers,) + tuple(layers[0].q.shape), dtype=layers[0].q.dtype, device=dev)
    out_all = torch.empty((n_layers,) + tuple(layers[0].out.shape), dtype=torch.float32, device=dev)
    for i, L in enumerate(layers):
        q_all[i].copy_(L.q)
        L.q = q_all[i]
        L.out = out_all[i]
    return layers, q_all, out_all


def step_fn(w, layers, ws, status, hkv, hint=False):
    """One decode step over every layer: hkv_decode_step per layer (query
    encode + scan + select + attend + merge).  hint: each layer names the next
    layer's codes for the library's L2 prefetch."""
    def step():
        for i, L in enumerate(layers):
            nxt = layers[(i + 1) % len(layers)].codes if hint and len(layers) > 1 else None
            hkv.hkv_decode_step(L.qh, L.q, L.codes, L.K, L.V, w.N, w.n_sink, w.n_local, w.top_k, L.out,
                                q_codes=L.q_codes, idx=L.idx, ws=ws, status=status, next_k_codes=nxt)
    return step


def check(hkv, status, what):
    rc = hkv.hkv_check(status)
    if rc != hkv.HKV_OK:
        raise RuntimeError(f"{what} reported status {rc}: {hkv.hkv_last_error()}")


def measure_workload(w: synth.Workload, args, dev, world, hkv, full: bool):
    """Times the decode step of workload w (all of its layers, one CUDA graph)
    and the fused decode kernel alone; with full=True also the other entry
    points, the encode and the end-to-end step.  Returns (dict, layers)."""
    per_layer_bytes = w.algorithmic_bytes()
    n_layers = args.layers or max(w.layers, math.ceil(3 * L2_BYTES / per_layer_bytes))
    layers, q_all, out_all = build_layers(w, dev, hkv, n_layers)
    # prefill: encode the keys of every layer (timed separately, reported as encode)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for L in layers:
        L.encode_keys(hkv)
    e1.record()
    torch.cuda.synchronize()
    encode_ms = e0.elapsed_time(e1)
    new_ws = lambda: hkv.workspace(w.B, w.Hq, w.Hkv, w.N, w.bits, w.top_k, w.n_sink, w.n_local, device=dev)
    ws = new_ws()
    status = hkv.status_word(dev)
    peak, peak_kind = measured_peaks()
    step = step_fn(w, layers, ws, status, hkv, hint=args.prefetch_hint)
    g_step = graph_of(step)
    check(hkv, status, "decode step")
    with ClockSampler(dev.index) as clk:
        mean_ms, med_ms = time_graph(g_step, args.steps, args.warmup, world)
    ms = max_over_ranks(med_ms, world, dev)
    mean_ms = max_over_ranks(mean_ms, world, dev)
    check(hkv, status, "decode step")
    del g_step
    keys_per_layer = w.B * w.Hkv * w.candidates()
    value, ms = job_throughput(keys_per_layer * len(layers), ms, world, dev)
    # the fused kernel alone: query codes given, one hkv_decode_step launch per layer
    given = hkv.HashParams.given(hkv.HKV_BF16 if w.dtype == "bf16" else hkv.HKV_F32, w.bits)
    ws_f = new_ws()
    for L in layers:
        hkv.hkv_encode_keys(L.qh, L.q.view(-1, w.d), L.q_codes.view(-1, w.words))

    def fused_only():
        for L in layers:
            hkv.hkv_decode_step(given, L.q, L.codes, L.K, L.V, w.N, w.n_sink, w.n_local, w.top_k, L.out,
                                q_codes=L.q_codes, idx=L.idx, ws=ws_f, status=status)

    g_fused = graph_of(fused_only)
    fused_ms = timed_ms(g_fused, args, world, dev)
    del g_fused
    check(hkv, status, "fused decode")
    fused_launch_ms = fused_ms / len(layers)
    achieved = per_layer_bytes / (fused_launch_ms * 1e-3) / 1e9
    step_gbs = per_layer_bytes * len(layers) / (ms * 1e-3) / 1e9
    res = {
        "workload": w.name, "layers_per_step": len(layers), "ms_per_step": ms, "ms_per_step_mean": mean_ms,
        "us_per_layer": ms * 1e3 / len(layers), "keys_per_s": value,
        "step_hbm": {"achieved_gbs": step_gbs, "peak_gbs": peak, "frac": step_gbs / peak,
                     "frac_of_nominal_8tbs": step_gbs / 8000.0, "bytes_per_layer": per_layer_bytes,
                     "peak_kind": peak_kind},
        "roofline": {"bound": "hbm", "kernel": "fused_kernel (scan + select + attend + merge, one layer)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic_record(os.path.join(ROOT, "hash_sparse_kv_b200", "csrc", "retrieve.cu"),
                                               w.name),
                     "algorithmic_bytes_per_launch": per_layer_bytes, "launch_us": fused_launch_ms * 1e3,
                     "peak_kind": peak_kind},
        "encode": dict(encode_roofline(w, len(layers), encode_ms),
                       traffic=traffic_record(os.path.join(ROOT, "hash_sparse_kv_b200", "csrc", "encode_tc.cu"),
                                              w.name) if w.hash == "lsh" else None),
        # decode with an LSH or sign query hash (query heads per KV head <= 32) is one
        # fused launch a layer; an MLP query hash adds the separate query encode launch
        "launches_per_step": (1 if w.hash in ("lsh", "sign") and w.g <= 32 else 2) * len(layers),
        "clocks": clk.summary(),
    }

    status_ok = lambda what: check(hkv, status, what)
    if full:
        g_other = graph_of(step_fn(w, layers, ws, status, hkv, hint=not args.prefetch_hint))
        other_ms = timed_ms(g_other, args, world, dev)
        del g_other
        res["us_per_layer_without_prefetch_hint" if args.prefetch_hint else "us_per_layer_with_prefetch_hint"] = \
            other_ms * 1e3 / len(layers)
        # each entry point alone, one launch per layer (own workspaces: each has its own layout)
        ws_r, ws_a = new_ws(), new_ws()

        def scan_only():
            for L in layers:
                hkv.hkv_retrieve_topk(L.q_codes, L.codes, w.N, w.n_sink, w.n_local, w.top_k, L.idx, ws=ws_r,
                                      status=status)

        def qenc_only():
            for L in layers:
                hkv.hkv_encode_keys(L.qh, L.q.view(-1, w.d), L.q_codes.view(-1, w.words))

        def attend_only():
            for L in layers:
                hkv.hkv_sparse_attend(L.q, L.K, L.V, w.N, L.idx, w.n_sink, w.n_local, L.out, ws=ws_a, status=status)

        victims = [torch.zeros(w.B, w.Hkv, dtype=torch.int32, device=dev) for _ in layers]
        ws_e = torch.zeros(8 * w.B * w.Hkv, dtype=torch.uint8, device=dev)

        def evict_only():
            for L, vic in zip(layers, victims):
                hkv.hkv_evict_select(L.q_codes, L.codes, w.N, w.n_sink, w.n_local, vic, ws=ws_e)

        times = {}
        for name, fn in (("retrieve_only", scan_only), ("encode_q", qenc_only), ("sparse_attend_only", attend_only),
                         ("evict_select", evict_only)):
            g = graph_of(fn)
            times[name] = timed_ms(g, args, world, dev) * 1e3 / len(layers)
            del g
        status_ok("stand-alone entry points")
        times["fused_decode"] = fused_launch_ms * 1e3
        res["kernels_us_per_launch"] = times
        code_bytes = w.B * w.Hkv * w.candidates() * w.bits // 8
        ev_gbs = code_bytes / (times["evict_select"] * 1e-6) / 1e9
        res["evict"] = {"bound": "hbm", "achieved": ev_gbs, "peak": peak, "unit": "GB/s", "frac": ev_gbs / peak,
                        "bytes_per_launch": code_bytes, "launches_per_layer": 2,
                        "traffic": traffic_record(os.path.join(ROOT, "hash_sparse_kv_b200", "csrc", "evict.cu"),
                                                  w.name)}
        # end to end: every layer's queries in from pinned host memory and every
        # output back, one copy each way per step, inside the timed region
        q_host = torch.empty(q_all.shape, dtype=q_all.dtype, device="cpu").pin_memory()
        o_host = torch.empty(out_all.shape, dtype=out_all.dtype, device="cpu").pin_memory()
        q_host.copy_(q_all.cpu())

        def e2e_step():
            q_all.copy_(q_host, non_blocking=True)
            step()
            o_host.copy_(out_all, non_blocking=True)

        g_e2e = graph_of(e2e_step)
        e2e_ms = timed_ms(g_e2e, args, world, dev)
        del g_e2e
        status_ok("end-to-end step")
        keys_step = keys_per_layer * len(layers) * world
        res["e2e"] = {"value": keys_step / (e2e_ms * 1e-3), "unit": "keys/s",
                      "h2d_bytes_per_step": q_host.numel() * q_host.element_size(),
                      "d2h_bytes_per_step": o_host.numel() * o_host.element_size(), "ms_per_step": e2e_ms,
                      "copies_per_step": 2}
    # paged cache (pages of 256 tokens scattered through a pool): the fused
    # multi-block retrieval and the fused decode step read through the page table
    res["paged"] = None
    PAGE = 256
    if w.N % PAGE == 0:
        ws_p = new_ws()
        pages = w.N // PAGE
        gen = torch.Generator(device=dev).manual_seed(1234)
        paged_layers = []
        for L in layers:
            perm = torch.randperm(w.B * pages, generator=gen, device=dev)
            table = perm.view(w.B, pages).to(torch.int32)

            def to_pool(x):
                # [B, Hkv, N, ...] -> pool page perm[b * pages + j] = tokens [j * PAGE, (j + 1) * PAGE) of b
                tail = tuple(x.shape[3:])
                src = x.view((w.B, w.Hkv, pages, PAGE) + tail).transpose(1, 2).reshape((w.B * pages, w.Hkv, PAGE) + tail)
                pool = torch.empty(src.shape, dtype=src.dtype, device=src.device)  # contiguous
                pool[perm.long()] = src
                return pool

            paged_layers.append((L, table, to_pool(L.codes), to_pool(L.K), to_pool(L.V)))

        def paged_only():
            for L, table, cpool, _, _ in paged_layers:
                hkv.hkv_retrieve_topk_paged(L.q_codes, cpool, table, w.N, w.n_sink, w.n_local, w.top_k, L.idx,
                                            status=status, ws=ws_p)

        def paged_step():
            for L, table, cpool, kpool, vpool in paged_layers:
                hkv.hkv_decode_step_paged(L.qh, L.q, cpool, kpool, vpool, table, w.N, w.n_sink, w.n_local, w.top_k,
                                          L.out, q_codes=L.q_codes, idx=L.idx, ws=ws_p, status=status)

        g = graph_of(paged_only)
        paged_ms = timed_ms(g, args, world, dev)
        del g
        g = graph_of(paged_step)
        paged_step_ms = timed_ms(g, args, world, dev)
        del g, paged_layers
        torch.cuda.empty_cache()
        status_ok("paged calls")
        res["paged"] = paged_roofline(w, len(layers), paged_ms, paged_step_ms, PAGE, peak, peak_kind)
    # sign-VQ only: retrieval by the norm-weighted sign score (its own kernel),
    # then the standalone sparse attention
    res["normw"] = None
    if w.hash == "sign" and w.candidates() <= 65536:
        ws_a = new_ws()

        def normw_only():
            for L in layers:
                hkv.hkv_retrieve_topk_normw(L.q_codes, L.codes, L.norms, w.N, w.n_sink, w.n_local, w.top_k, L.idx)

        def normw_step():
            for L in layers:
                hkv.hkv_encode_keys(L.qh, L.q.view(-1, w.d), L.q_codes.view(-1, w.words))
                hkv.hkv_retrieve_topk_normw(L.q_codes, L.codes, L.norms, w.N, w.n_sink, w.n_local, w.top_k, L.idx)
                hkv.hkv_sparse_attend(L.q, L.K, L.V, w.N, L.idx, w.n_sink, w.n_local, L.out, ws=ws_a, status=status)

        def normw_decode():
            for L in layers:
                hkv.hkv_decode_step_normw(L.q, L.codes, L.norms, L.K, L.V, w.N, w.n_sink, w.n_local, w.top_k, L.idx,
                                          L.out, q_codes=L.q_codes, status=status)

        g = graph_of(normw_only)
        normw_ms = timed_ms(g, args, world, dev)
        del g
        g = graph_of(normw_step)
        normw_step_ms = timed_ms(g, args, world, dev)
        del g
        g = graph_of(normw_decode)
        normw_decode_ms = timed_ms(g, args, world, dev)
        del g
        status_ok("norm-weighted calls")
        res["normw"] = normw_roofline(w, len(layers), normw_ms, normw_step_ms, peak, peak_kind)
        res["normw"]["decode_step_us_per_layer"] = normw_decode_ms * 1e3 / len(layers)
        res["normw"]["decode_step_frac"] = normw_bytes_step(w) / (normw_decode_ms * 1e-3 / len(layers)) / 1e9 / peak
    return res, layers

def run_gpu(args, rank, world, local):
    """The main workload in full, then every other workload's decode step and
    fused kernel (each workload's buffers freed before the next)."""
    import hash_sparse_kv_b200 as hkv

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hkv.lib()
    w = synth.WORKLOADS[args.workload]
    main, layers = measure_workload(w, args, dev, world, hkv, full=True)
    cpu_layer = oracle_inputs_from_device(w, layers[0]) if rank == 0 and world == 1 and not args.no_cpu_baseline \
        else None
    del layers
    torch.cuda.empty_cache()
    others = {}
    if not args.main_only:
        for name in sorted(synth.WORKLOADS):
            if name == w.name:
                continue
            r, lay = measure_workload(synth.WORKLOADS[name], args, dev, world, hkv, full=False)
            del lay
            torch.cuda.empty_cache()
            others[name] = r
    peak, peak_kind = measured_peaks()
    out = {
        "metric": "decode retrieval+sparse-attn keys scanned/s (also us/layer and % HBM roofline)",
        "value": main["keys_per_s"],
        "unit": "keys/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": main["ms_per_step"],
        "ms_per_step_mean": main["ms_per_step_mean"],
        "us_per_layer": main["us_per_layer"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u32 codes + " + ("bf16" if w.dtype == "bf16" else "f32") + " K/V, f32 accumulate",
        "data": "synthetic (two-cone Gaussian keys/queries, drawn on device)",
        "config": {
            "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": w.d, "n_tokens": w.N,
            "hash": w.hash, "code_bits": w.bits, "top_k": w.top_k, "n_sink": w.n_sink, "n_local": w.n_local,
            "layers_per_step": main["layers_per_step"], "parallelism": f"replica x{world}",
            "next_layer_prefetch_hint": args.prefetch_hint,
            "timing": "median of the per-replay CUDA-event times (max over ranks)",
            "l2": f"inputs larger than L2: {main['layers_per_step']} distinct layer buffers, "
                  f"{w.algorithmic_bytes() * main['layers_per_step'] / 1e9:.2f} GB algorithmic per step",
        },
        "step_hbm": main["step_hbm"],
        "roofline": main["roofline"],
        "e2e": main["e2e"],
        "encode": main["encode"],
        "kernels_us_per_launch": main["kernels_us_per_launch"],
        "evict": main["evict"],
        "paged": main["paged"],
        "normw": main["normw"],
        "configs": {n: {k: v for k, v in r.items() if k != "clocks"} for n, r in others.items()},
        "gpu_launches": main["launches_per_step"] * args.steps,
        "clocks": main["clocks"],
    }
    for k in ("us_per_layer_with_prefetch_hint", "us_per_layer_without_prefetch_hint"):
        if k in main:
            out[k] = main[k]
    out["peak_kind"] = peak_kind
    return out, cpu_layer, w


def run_split(args, rank, world, local):
    """Token split of the workload's sequence across the ranks: rank r holds
    tokens token_range(N, world, r) of every layer (K, V, codes) and a copy of
    the queries; one step is decode_step_split on every layer (the ranks'
    top-k candidates and partial outputs exchanged by NCCL all-gathers),
    captured in one CUDA graph."""
    import socket
    import torch.distributed as dist
    import hash_sparse_kv_b200 as hkv
    from hash_sparse_kv_b200 import split as hsplit

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if not dist.is_initialized():
        # one rank: a process group of one, for the same collective calls
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        import datetime
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120))
    hkv.lib()
    w = synth.WORKLOADS[args.workload]
    r0, r1 = hsplit.token_range(w.N, world, rank)
    wr = w.with_(N=r1 - r0)
    n_layers = args.layers or w.layers
    layers = [Layer(wr, l % w.layers if w.layers > 1 else 0, dev, hkv) for l in range(n_layers)]
    for L in layers:
        L.encode_keys(hkv)
    st = hsplit.SplitState.make(world, rank, w.B, w.Hq, w.Hkv, w.bits, w.top_k, w.N, w.n_sink, w.n_local, dev)

    def step():
        for L in layers:
            hsplit.decode_step_split(st, L.qh, L.q, L.codes, L.K, L.V, w.N, w.n_sink, w.n_local, w.bits, L.out)

    g = graph_of(step)
    check(hkv, st.status, "split decode step")
    with ClockSampler(dev.index) as clk:
        mean_ms, med_ms = time_graph(g, args.steps, args.warmup, world)
    ms = max_over_ranks(med_ms, world, dev)
    check(hkv, st.status, "split decode step")
    del g
    keys = w.B * w.Hkv * w.candidates() * n_layers  # the whole sequence, all ranks together
    out = {
        "metric": "decode retrieval+sparse-attn keys scanned/s (also us/layer and % HBM roofline)",
        "value": keys / (ms * 1e-3), "unit": "keys/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "us_per_layer": ms * 1e3 / n_layers, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "u32 codes + " + ("bf16" if w.dtype == "bf16" else "f32") + " K/V, f32 accumulate",
        "data": "synthetic (two-cone Gaussian keys/queries, drawn on device)",
        "config": {"workload": w.name, "n_tokens": w.N, "tokens_per_rank": r1 - r0, "layers_per_step": n_layers,
                   "parallelism": f"token split x{world} (NCCL all-gathers of candidates and partials)",
                   "timing": "median of the per-replay CUDA-event times (max over ranks)"},
        # per layer: query encode, retrieval, global selection, attention and
        # the G-way merge, one launch each at this shape (the all-gathers are NCCL's)
        "gpu_launches": 5 * n_layers * args.steps, "clocks": clk.summary(), "cpu_baseline": None,
    }
    dist.barrier()
    return out


# ------------------------------------------------------------------ oracle arm --

def oracle_inputs_from_device(w: synth.Workload, L):
    """One layer's host copies, from the bench's device buffers."""
    q, K, V = L.q.cpu(), L.K.cpu(), L.V.cpu()
    if w.hash == "lsh":
        return q, K, V, L.R.cpu(), L.R.cpu()
    if w.hash == "mlp":
        return q, K, V, tuple(t.cpu() for t in L.qmlp), tuple(t.cpu() for t in L.kmlp)
    return q, K, V, None, None


def oracle_inputs_host(w: synth.Workload):
    inp = synth.layer_inputs(w, 0, pad_junk=False)
    if w.hash == "lsh":
        return inp["q"], inp["K"], inp["V"], inp["R"], inp["R"]
    if w.hash == "mlp":
        return inp["q"], inp["K"], inp["V"], inp["q_mlp"], inp["k_mlp"]
    return inp["q"], inp["K"], inp["V"], None, None


def host_cpu():
    """(usable cores, CPU model name) of this host."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return cores, model


class OracleLayer:
    """The oracle's decode step on one layer of the workload.  The cache's key
    codes are computed once by the oracle itself (setup, not timed).  (batch,
    KV head) pairs are independent, so the step can also run as one oracle
    call per pair on a pool of host threads (numpy releases the interpreter
    lock inside its array operations; each call keeps BLAS to one thread)."""

    def __init__(self, w: synth.Workload, q, K, V, qparams, kparams):
        import oracle
        self.w, self.q, self.K, self.V, self.qparams = w, q, K, V, qparams
        kc = oracle.encode(w.hash, K, kparams)
        self.kc = kc[0] if w.hash == "sign" else kc

    def _pair(self, b, h):
        import oracle
        w, g = self.w, self.w.g
        oracle.decode_step(self.q[b:b + 1, h * g:(h + 1) * g], self.K[b:b + 1, h:h + 1], self.V[b:b + 1, h:h + 1],
                           self.kc[b:b + 1, h:h + 1], w.N, w.n_sink, w.n_local, w.top_k, w.hash, self.qparams)

    def run(self, threads: int = 1) -> float:
        """Seconds for one decode step of this layer on `threads` host threads."""
        import oracle
        from threadpoolctl import threadpool_limits
        w = self.w
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            if threads <= 1:
                oracle.decode_step(self.q, self.K, self.V, self.kc, w.N, w.n_sink, w.n_local, w.top_k, w.hash,
                                   self.qparams)
            else:
                import concurrent.futures
                pairs = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
                with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
                    list(ex.map(lambda bh: self._pair(*bh), pairs))
            return time.perf_counter() - t0


def oracle_sample(w: synth.Workload, budget_s: float, layer_inputs):
    """Time the oracle's decode step on one whole layer on one thread and on a
    thread per (batch, KV head) pair (up to the host's cores), each repeated
    until its share of the budget is spent (at most 64 times)."""
    ol = OracleLayer(w, *layer_inputs)
    cores, model = host_cpu()
    pool = max(1, min(cores, w.B * w.Hkv))
    keys_step = w.B * w.Hkv * w.candidates()
    out = {}
    for threads in (pool, 1):
        elapsed, n = 0.0, 0
        while n < 1 or (elapsed < budget_s / 2 and n < 64):
            elapsed += ol.run(threads)
            n += 1
        out[threads] = (keys_step * n / elapsed, n, elapsed)
    v, n, el = out[pool]
    v1, n1, el1 = out[1]
    return {"value": v, "unit": "keys/s", "cores": pool, "kind": "oracle",
            "sample": f"{n} decode step(s) of one {w.name} layer ({keys_step} keys each) on {pool} host thread(s), "
                      f"one per (batch, KV head) pair, {el:.2f} s; single thread: {n1} step(s), {el1:.2f} s",
            "value_1_core": v1, "host_cores": cores, "cpu_model": model}


def run_reference(args, rank, world):
    """The reference arm: the oracle's decode step of one layer per step, on a
    host thread per (batch, KV head) pair (up to the host's cores)."""
    w = synth.WORKLOADS[args.workload]
    if rank != 0:
        return None
    ol = OracleLayer(w, *oracle_inputs_host(w))
    cores, model = host_cpu()
    pool = max(1, min(cores, w.B * w.Hkv))
    keys_per_step = w.B * w.Hkv * w.candidates()
    for _ in range(args.warmup):
        ol.run(pool)
    per_step_s = [ol.run(pool) for _ in range(args.steps)]
    med = statistics.median(per_step_s)
    value = keys_per_step / med
    sample = (f"each step: one decode step of one {w.name} layer ({keys_per_step} keys) on {pool} host thread(s), "
              f"one per (batch, KV head) pair; median of {args.steps}")
    return {
        "impl": "reference",
        "metric": "decode retrieval+sparse-attn keys scanned/s (also us/layer and % HBM roofline)",
        "value": value, "unit": "keys/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": med * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (two-cone Gaussian, host generator)",
        "config": {"workload": w.name, "layers_per_step": 1},
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": pool, "kind": "oracle", "sample": sample,
                         "host_cores": cores, "cpu_model": model},
        "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    init_dist(world, local)
    if args.split:
        res = run_split(args, rank, world, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
        import torch.distributed as dist
        dist.destroy_process_group()
        return
    res, cpu_layer, w = run_gpu(args, rank, world, local)
    if rank == 0:
        res["cpu_baseline"] = oracle_sample(w, args.cpu_budget_s, cpu_layer) if cpu_layer is not None else None
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
