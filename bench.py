"""Benchmark of the decode step: query encode + Hamming scan + top-k + sparse
attention + LSE merge, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole decode path over every layer of the
workload (28 sequential layers for the default Qwen2.5-7B-shaped 512K-token
case), captured in one CUDA graph.  Inputs are synthetic, drawn on the device
(same distributions as the parity tests), and larger than L2: every layer has
its own codes and K/V buffers.  Timing uses CUDA events on the launching
stream after W warm-up steps; the value is the max over ranks.  With N > 1
(torchrun) each rank runs its own replica of the workload (independent
sequences: weak scaling, no collective on the data path).

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
    """Retrieval over a paged code pool: the candidates' codes are the
    algorithmic bytes of one launch (the page table is negligible)."""
    nbytes = w.B * w.Hkv * w.candidates() * w.bits // 8
    launch_s = ms * 1e-3 / n_layers
    return {"kernel": "paged_topk_kernel (scan through the page table + select + ordered compaction)",
            "page_size": page, "bound": "hbm", "achieved": nbytes / launch_s / 1e9, "peak": peak, "unit": "GB/s",
            "frac": nbytes / launch_s / 1e9 / peak, "bytes_per_launch": nbytes, "launch_us": launch_s * 1e6,
            "step_us_per_layer": step_ms * 1e3 / n_layers, "launches_per_layer": 3, "peak_kind": peak_kind,
            "traffic": None}


def normw_roofline(w: synth.Workload, n_layers: int, ms: float, step_ms: float, peak: float, peak_kind: str) -> dict:
    """Norm-weighted sign-VQ retrieval: codes and fp16 norms of every candidate
    are the algorithmic bytes of one launch."""
    nbytes = w.B * w.Hkv * w.candidates() * (w.bits // 8 + 2)
    launch_s = ms * 1e-3 / n_layers
    return {"kernel": "normw_kernel (scan + radix select + ordered compaction)", "bound": "hbm",
            "achieved": nbytes / launch_s / 1e9, "peak": peak, "unit": "GB/s",
            "frac": nbytes / launch_s / 1e9 / peak, "bytes_per_launch": nbytes, "launch_us": launch_s * 1e6,
            "step_us_per_layer": step_ms * 1e3 / n_layers, "launches_per_layer": 3, "peak_kind": peak_kind,
            "traffic": traffic_record(os.path.join(ROOT, "hash_sparse_kv_b200", "csrc", "normw.cu"), w.name)}


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
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    start.record(stream)
    for _ in range(steps):
        g.replay()
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / steps  # ms per replay


def source_digest(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_record(kernel_file: str, workload: str):
    """DRAM traffic per launch from the committed ncu summary, if it was taken
    on the current source of the kernel; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(workload, {}).get(os.path.basename(kernel_file))
    if not rec or rec.get("source_sha256_16") != source_digest(kernel_file):
        return None
    return rec.get("bytes_per_launch")


def run_gpu(args, rank, world, local):
    import hash_sparse_kv_b200 as hkv

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hkv.lib()
    w = synth.WORKLOADS[args.workload]
    per_layer_bytes = w.algorithmic_bytes()
    n_layers = args.layers or max(w.layers, math.ceil(3 * L2_BYTES / per_layer_bytes))
    layers = [Layer(w, l % w.layers if w.layers > 1 else 0, dev, hkv) for l in range(n_layers)]
    # prefill: encode the keys of every layer (timed separately, reported as encode)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for L in layers:
        L.encode_keys(hkv)
    e1.record()
    torch.cuda.synchronize()
    encode_ms = e0.elapsed_time(e1)
    ws = hkv.workspace(w.B, w.Hq, w.Hkv, w.N, w.bits, w.top_k, w.n_sink, w.n_local, device=dev)
    status = hkv.status_word(dev)

    def step(hint=args.prefetch_hint):
        # layer i tells the library that layer i + 1 (wrapping to the next
        # step's layer 0) scans next, so its codes stream into L2 during layer
        # i's selection and attention
        for i, L in enumerate(layers):
            nxt = layers[(i + 1) % len(layers)].codes if hint and len(layers) > 1 else None
            hkv.hkv_decode_step(L.qh, L.q, L.codes, L.K, L.V, w.N, w.n_sink, w.n_local, w.top_k, L.out,
                                q_codes=L.q_codes, idx=L.idx, ws=ws, status=status, next_k_codes=nxt)

    # standalone calls get their own workspaces (each entry point has its own layout)
    ws_r = hkv.workspace(w.B, w.Hq, w.Hkv, w.N, w.bits, w.top_k, w.n_sink, w.n_local, device=dev)
    ws_a = hkv.workspace(w.B, w.Hq, w.Hkv, w.N, w.bits, w.top_k, w.n_sink, w.n_local, device=dev)
    ws_f = hkv.workspace(w.B, w.Hq, w.Hkv, w.N, w.bits, w.top_k, w.n_sink, w.n_local, device=dev)

    given = hkv.HashParams.given(hkv.HKV_BF16 if w.dtype == "bf16" else hkv.HKV_F32, w.bits)

    def fused_only():
        for L in layers:
            hkv.hkv_decode_step(given, L.q, L.codes, L.K, L.V, w.N, w.n_sink, w.n_local, w.top_k, L.out,
                                q_codes=L.q_codes, idx=L.idx, ws=ws_f, status=status)

    def scan_only():
        for L in layers:
            hkv.hkv_retrieve_topk(L.q_codes, L.codes, w.N, w.n_sink, w.n_local, w.top_k, L.idx, ws=ws_r,
                                  status=status)

    g_step = graph_of(step)
    rc = hkv.hkv_check(status)
    if rc != hkv.HKV_OK:
        raise RuntimeError(f"decode step reported status {rc}")
    with ClockSampler(local) as clk:
        ms = time_graph(g_step, args.steps, args.warmup, world)
    rc = hkv.hkv_check(status)
    if rc != hkv.HKV_OK:
        raise RuntimeError(f"decode step reported status {rc}")
    keys_per_layer = w.B * w.Hkv * w.candidates()
    value, ms = job_throughput(keys_per_layer * len(layers), ms, world, dev)
    g_other = graph_of(lambda: step(hint=not args.prefetch_hint))
    other_ms = max_over_ranks(time_graph(g_other, args.steps, args.warmup, world), world, dev)
    del g_other
    # each kernel alone, one launch per layer
    def qenc_only():
        for L in layers:
            hkv.hkv_encode_keys(L.qh, L.q.view(-1, w.d), L.q_codes.view(-1, w.words))

    def attend_only():
        for L in layers:
            hkv.hkv_sparse_attend(L.q, L.K, L.V, w.N, L.idx, w.n_sink, w.n_local, L.out, ws=ws_a, status=status)

    g_fused = graph_of(fused_only)
    fused_ms = max_over_ranks(time_graph(g_fused, args.steps, args.warmup, world), world, dev)
    del g_fused
    g_scan = graph_of(scan_only)
    scan_ms = max_over_ranks(time_graph(g_scan, args.steps, args.warmup, world), world, dev)
    g_qenc = graph_of(qenc_only)
    qenc_ms = max_over_ranks(time_graph(g_qenc, args.steps, args.warmup, world), world, dev)
    g_att = graph_of(attend_only)
    att_ms = max_over_ranks(time_graph(g_att, args.steps, args.warmup, world), world, dev)
    # HashEvict eviction choice for every layer (one scan of the codes each)
    victims = [torch.zeros(w.B, w.Hkv, dtype=torch.int32, device=dev) for _ in layers]
    ws_e = torch.zeros(8 * w.B * w.Hkv, dtype=torch.uint8, device=dev)

    def evict_only():
        for L, vic in zip(layers, victims):
            hkv.hkv_evict_select(L.q_codes, L.codes, w.N, w.n_sink, w.n_local, vic, ws=ws_e)

    g_ev = graph_of(evict_only)
    ev_ms = max_over_ranks(time_graph(g_ev, args.steps, args.warmup, world), world, dev)
    del g_ev
    del g_qenc, g_att
    # paged cache (pages of 256 tokens scattered through a pool): retrieval
    # and attention read through the page table, after the query encode
    paged_ms = paged_step_ms = None
    PAGE = 256
    if w.candidates() <= 65536 and w.N % PAGE == 0:
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
                pool = torch.empty_like(src)
                pool[perm.long()] = src
                return pool

            paged_layers.append((L, table, to_pool(L.codes), to_pool(L.K), to_pool(L.V)))

        def paged_only():
            for L, table, cpool, _, _ in paged_layers:
                hkv.hkv_retrieve_topk_paged(L.q_codes, cpool, table, w.N, w.n_sink, w.n_local, w.top_k, L.idx,
                                            status=status)

        def paged_step():
            for L, table, cpool, kpool, vpool in paged_layers:
                hkv.hkv_encode_keys(L.qh, L.q.view(-1, w.d), L.q_codes.view(-1, w.words))
                hkv.hkv_retrieve_topk_paged(L.q_codes, cpool, table, w.N, w.n_sink, w.n_local, w.top_k, L.idx,
                                            status=status)
                hkv.hkv_sparse_attend_paged(L.q, kpool, vpool, table, w.N, L.idx, w.n_sink, w.n_local, L.out,
                                            ws=ws_a, status=status)

        g_pg = graph_of(paged_only)
        paged_ms = max_over_ranks(time_graph(g_pg, args.steps, args.warmup, world), world, dev)
        del g_pg
        g_pg = graph_of(paged_step)
        paged_step_ms = max_over_ranks(time_graph(g_pg, args.steps, args.warmup, world), world, dev)
        del g_pg, paged_layers
        rc = hkv.hkv_check(status)
        if rc != hkv.HKV_OK:
            raise RuntimeError(f"paged calls reported status {rc}")
    # sign-VQ only: retrieval by the norm-weighted sign score (its own kernel),
    # then the standalone sparse attention
    normw_ms = normw_step_ms = None
    if w.hash == "sign" and w.candidates() <= 65536:
        def normw_only():
            for L in layers:
                hkv.hkv_retrieve_topk_normw(L.q_codes, L.codes, L.norms, w.N, w.n_sink, w.n_local, w.top_k, L.idx)

        def normw_step():
            for L in layers:
                hkv.hkv_encode_keys(L.qh, L.q.view(-1, w.d), L.q_codes.view(-1, w.words))
                hkv.hkv_retrieve_topk_normw(L.q_codes, L.codes, L.norms, w.N, w.n_sink, w.n_local, w.top_k, L.idx)
                hkv.hkv_sparse_attend(L.q, L.K, L.V, w.N, L.idx, w.n_sink, w.n_local, L.out, ws=ws_a, status=status)

        g_nw = graph_of(normw_only)
        normw_ms = max_over_ranks(time_graph(g_nw, args.steps, args.warmup, world), world, dev)
        del g_nw
        g_nw = graph_of(normw_step)
        normw_step_ms = max_over_ranks(time_graph(g_nw, args.steps, args.warmup, world), world, dev)
        del g_nw
    # end to end: host q in, host out back, every step
    q_host = [torch.empty_like(L.q, device="cpu").pin_memory() for L in layers]
    o_host = [torch.empty_like(L.out, device="cpu").pin_memory() for L in layers]
    for qh, L in zip(q_host, layers):
        qh.copy_(L.q.cpu())

    def e2e_step():
        for qh, L in zip(q_host, layers):
            L.q.copy_(qh, non_blocking=True)
        step()
        for oh, L in zip(o_host, layers):
            oh.copy_(L.out, non_blocking=True)

    g_e2e = graph_of(e2e_step)
    e2e_ms = max_over_ranks(time_graph(g_e2e, args.steps, args.warmup, world), world, dev)
    h2d = sum(t.numel() * t.element_size() for t in q_host)
    d2h = sum(t.numel() * t.element_size() for t in o_host)
    rc = hkv.hkv_check(status)
    if rc != hkv.HKV_OK:
        raise RuntimeError(f"e2e step reported status {rc}")

    keys_step = keys_per_layer * len(layers) * world
    peak, peak_kind = measured_peaks()
    fused_launch_ms = fused_ms / len(layers)
    achieved = per_layer_bytes / (fused_launch_ms * 1e-3) / 1e9
    traffic = traffic_record(os.path.join(ROOT, "hash_sparse_kv_b200", "csrc", "retrieve.cu"), w.name)
    code_bytes = w.B * w.Hkv * w.candidates() * w.bits // 8
    step_gbs = per_layer_bytes * len(layers) / (ms * 1e-3) / 1e9
    out = {
        "metric": "decode retrieval+sparse-attn keys scanned/s (also us/layer and % HBM roofline)",
        "value": value,
        "unit": "keys/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "us_per_layer": ms * 1e3 / len(layers),
        ("us_per_layer_without_prefetch_hint" if args.prefetch_hint else "us_per_layer_with_prefetch_hint"):
            other_ms * 1e3 / len(layers),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u32 codes + " + ("bf16" if w.dtype == "bf16" else "f32") + " K/V, f32 accumulate",
        "data": "synthetic (two-cone Gaussian keys/queries, drawn on device)",
        "config": {
            "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "head_dim": w.d, "n_tokens": w.N,
            "hash": w.hash, "code_bits": w.bits, "top_k": w.top_k, "n_sink": w.n_sink, "n_local": w.n_local,
            "layers_per_step": len(layers), "parallelism": f"replica x{world}",
            "next_layer_prefetch_hint": args.prefetch_hint,
            "l2": f"inputs larger than L2: {len(layers)} distinct layer buffers, "
                  f"{per_layer_bytes * len(layers) / 1e9:.2f} GB algorithmic per step",
        },
        "step_hbm": {"achieved_gbs": step_gbs, "peak_gbs": peak, "frac": step_gbs / peak,
                     "frac_of_nominal_8tbs": step_gbs / 8000.0,
                     "bytes_per_layer": per_layer_bytes, "peak_kind": peak_kind},
        "roofline": {"bound": "hbm", "kernel": "fused_kernel (scan + select + attend + merge, one layer)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "algorithmic_bytes_per_launch": per_layer_bytes,
                     "launch_us": fused_launch_ms * 1e3, "peak_kind": peak_kind},
        "e2e": {"value": keys_step / (e2e_ms * 1e-3), "unit": "keys/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "encode": dict(encode_roofline(w, len(layers), encode_ms),
                       traffic=traffic_record(os.path.join(ROOT, "hash_sparse_kv_b200", "csrc", "encode_tc.cu"),
                                              w.name) if w.hash == "lsh" else None),
        "kernels_us_per_launch": {"encode_q": qenc_ms * 1e3 / len(layers),
                                  "fused_decode": fused_launch_ms * 1e3,
                                  "retrieve_only": scan_ms * 1e3 / len(layers),
                                  "sparse_attend_only": att_ms * 1e3 / len(layers),
                                  "evict_select": ev_ms * 1e3 / len(layers)},
        "evict": {"bound": "hbm", "achieved": code_bytes / (ev_ms * 1e-3 / len(layers)) / 1e9, "peak": peak,
                  "unit": "GB/s", "frac": code_bytes / (ev_ms * 1e-3 / len(layers)) / 1e9 / peak,
                  "bytes_per_launch": code_bytes, "launches_per_layer": 2,
                  "traffic": traffic_record(os.path.join(ROOT, "hash_sparse_kv_b200", "csrc", "evict.cu"), w.name)},
        "paged": None if paged_ms is None else paged_roofline(w, len(layers), paged_ms, paged_step_ms, PAGE, peak,
                                                              peak_kind),
        "normw": None if normw_ms is None else normw_roofline(w, len(layers), normw_ms, normw_step_ms, peak, peak_kind),
        # decode with an LSH or sign query hash (query heads per KV head <= 32) is one
        # fused launch a layer; an MLP query hash adds the separate query encode launch
        "gpu_launches": (1 if w.hash in ("lsh", "sign") and w.g <= 32 else 2) * len(layers) * args.steps,
        "clocks": clk.summary(),
    }
    del g_step, g_scan, g_e2e
    return out, layers, w


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


class OracleLayer:
    """The oracle's decode step on one layer of the workload.  The cache's key
    codes are computed once by the oracle itself (setup, not timed)."""

    def __init__(self, w: synth.Workload, q, K, V, qparams, kparams):
        import oracle
        self.w, self.q, self.K, self.V, self.qparams = w, q, K, V, qparams
        kc = oracle.encode(w.hash, K, kparams)
        self.kc = kc[0] if w.hash == "sign" else kc

    def run(self) -> float:
        """Seconds for one decode step of this layer (single thread)."""
        import oracle
        from threadpoolctl import threadpool_limits
        w = self.w
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            oracle.decode_step(self.q, self.K, self.V, self.kc, w.N, w.n_sink, w.n_local, w.top_k, w.hash,
                               self.qparams)
            return time.perf_counter() - t0


def oracle_sample(w: synth.Workload, budget_s: float, layer_inputs):
    """Time the oracle's decode step on one whole layer, repeated until the
    budget is spent (at most 64 times).  Returns (keys/s, sample, threads)."""
    ol = OracleLayer(w, *layer_inputs)
    elapsed, n = 0.0, 0
    while n < 1 or (elapsed < budget_s and n < 64):
        elapsed += ol.run()
        n += 1
    keys = n * w.B * w.Hkv * w.candidates()
    return keys / elapsed, f"{n} decode step(s) of one {w.name} layer ({w.B * w.Hkv * w.candidates()} keys each), " \
                           f"{elapsed:.2f} s", 1


def run_reference(args, rank, world):
    w = synth.WORKLOADS[args.workload]
    if rank != 0:
        return None
    ol = OracleLayer(w, *oracle_inputs_host(w))
    keys_per_step = w.B * w.Hkv * w.candidates()
    for _ in range(args.warmup):
        ol.run()
    per_step_s = [ol.run() for _ in range(args.steps)]
    value = keys_per_step / statistics.mean(per_step_s)
    sample = f"each step: one decode step of one {w.name} layer ({keys_per_step} keys), single thread"
    return {
        "impl": "reference",
        "metric": "decode retrieval+sparse-attn keys scanned/s (also us/layer and % HBM roofline)",
        "value": value, "unit": "keys/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.mean(per_step_s) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (two-cone Gaussian, host generator)",
        "config": {"workload": w.name, "layers_per_step": 1},
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": 1, "kind": "oracle", "sample": sample},
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
    res, layers, w = run_gpu(args, rank, world, local)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            v, sample, cores = oracle_sample(w, args.cpu_budget_s, oracle_inputs_from_device(w, layers[0]))
            res["cpu_baseline"] = {"value": v, "unit": "keys/s", "cores": cores, "kind": "oracle", "sample": sample}
        else:
            res["cpu_baseline"] = None
        print(json.dumps(res), flush=True)
    del layers
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
