#!/usr/bin/env python
"""DSA hot-path throughput on B200 through libdsa's C ABI.

One step = one pass of the whole hot path (Lightning Indexer logits -> top-k ->
sparse MLA (+ split merge)) over one batch of synthetic input.  The default workload
is decode: 32 sequences x 8192 context, one query each, FP8 indexer 64 x 128 (page
64), top-k 2048, 128-head MLA over bf16 576-d latent KV (page 1).

Timing: W untimed warm-up steps, then exactly K timed steps of the fused call
(dsa_decode / the prefill sequence), each bracketed by CUDA events on the launching
stream, with a 256 MiB write between steps to flush L2 (inputs here are ~120 MB,
below the 126 MB L2).  A second K-step loop times the same kernels stage by stage
for the roofline.  Multi-GPU runs are independent replicas (one batch per rank, no
data-path collective): value = all ranks' tokens / the slowest rank's time.

`--impl reference` times the CPU oracle on a bounded sample of the same workload.

`--workload store_L131072_fp8` times the cache writes instead: one step writes a
131072-token prompt's indexer keys (page 64) and latent-KV rows (page 1) into FP8
caches (dsa_cache_store, twice).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import long_context_sparse_fp8_b200 as L  # noqa: E402
from long_context_sparse_fp8_b200 import chunked as CH  # noqa: E402
from long_context_sparse_fp8_b200 import replicas as R  # noqa: E402
from long_context_sparse_fp8_b200 import workloads as W  # noqa: E402

METRIC = "DSA tokens/s (decode & prefill) on 1 B200; % of HBM / tensor-core roofline"
FLUSH_BYTES = 256 << 20

WORKLOADS = {
    "chunked_prefill_L131072_16x8192": (W.ChunkedSpec, "chunked"),
    "decode_b32_ctx8192": (W.decode_b32_8k, "decode"),
    "prefill_L32768_q8192": (W.prefill_32k, "prefill"),
    "decode_b64_ctx64k-128k_fp8kv": (W.decode_b64_128k, "decode"),
    "decode_mtp2_b32_ctx8192": (W.decode_mtp_b32_8k, "decode"),
    "prefill_L131072_chunk15": (lambda: W.chunked_prefill_128k(15), "prefill"),
    "store_L131072_fp8": (W.store_prompt_128k, "store"),
}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["dsa", "reference"], default="dsa")
    p.add_argument("--workload", choices=sorted(WORKLOADS),
                   default="chunked_prefill_L131072_16x8192")
    p.add_argument("--no-extras", action="store_true",
                   help="chunked prefill only: skip the decode lines reported beside it")
    p.add_argument("--no-e2e", action="store_true", help="skip the end-to-end measurement")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--fp8-peak", action="store_true",
                   help="measure the dense FP8 GEMM rate (torch._scaled_mm, e4m3, 8192^3, "
                        "best of 10) and print it as one JSON line")
    return p.parse_args()


# ----------------------------------------------------------------------------- plumbing
class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, read through NVML every
    millisecond or so by a background thread while the timed loop runs (the loop lasts
    only milliseconds, so nvidia-smi's 200 ms period would miss it).  Falls back to
    nvidia-smi when NVML is unavailable."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.thread = None
        self.samples = []        # (sm_mhz, reason bits)
        self.lines = []
        self.smax = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        pr = torch.cuda.get_device_properties(self.gpu)
        bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop = threading.Event()

            def poll():
                while not self.stop.is_set():
                    try:
                        self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                             nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
                    except Exception:  # noqa: BLE001 -- sampling must never fail the run
                        pass
                    time.sleep(0.001)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            time.sleep(0.005)
            return self
        except Exception:  # noqa: BLE001
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
            "sw_power_cap": 0x4}

    def summary(self):
        sm, smax, reasons = [], self.smax, set()
        for mhz, bits in self.samples:
            sm.append(float(mhz))
            for n, b in self.BITS.items():
                if bits & b:
                    reasons.add(n)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvml" if self.samples else "nvidia-smi"}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def fp8_peak():
    """The FP8 denominator: the measured figure recorded in profiles/fp8_peak.json (from
    `bench.py --fp8-peak` on this pool), else 2x the measured bf16 peak (nominal ratio)."""
    try:
        with open(os.path.join(ROOT, "profiles", "fp8_peak.json")) as f:
            return float(json.load(f)["fp8_tflops"]), "measured fp8 (torch._scaled_mm e4m3 8192^3)"
    except (OSError, KeyError, ValueError):
        return 2.0 * measured_peaks()[1], "2x measured bf16 (nominal ratio)"


def measure_fp8_peak():
    n = 8192
    a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    one = torch.ones((), device="cuda")
    run = lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one,  # noqa: E731
                                   out_dtype=torch.bfloat16)
    for _ in range(3):
        run()
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    return {"fp8_tflops": round(2 * n ** 3 / (best / 1e3) / 1e12, 1), "ms": round(best, 4),
            "method": "torch._scaled_mm e4m3 x e4m3 -> bf16, 8192^3, best of 10 (CUDA events)",
            "gpu": torch.cuda.get_device_name()}


def ncu_traffic(workload: str, kernel_file: str):
    """DRAM bytes per launch from the committed ncu summary of this workload, if the
    kernel source is unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    src = os.path.join(ROOT, "long_context_sparse_fp8_b200", "csrc", kernel_file)
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    entry = rec.get(workload, {}).get(kernel_file)
    if not entry or entry.get("source_sha") != sha:
        return None
    return entry.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- workload
class Step:
    """Buffers and calls of one hot-path step on one GPU."""

    def __init__(self, wl: W.Workload, mode: str):
        s = wl.spec
        self.wl, self.mode, self.s = wl, mode, s
        self.batch = L.Batch(wl.cu_q, wl.seq_lens, s.total_q, s.max_seq_len)
        self.kc = L.PagedCache(wl.k_pages, wl.k_block_table, W.INDEXER_PAGE, wl.k_scale)
        self.kv = L.PagedCache(wl.kv, wl.kv_slot_table, 1, wl.kv_scale)
        dev = wl.device
        self.ld = (s.max_seq_len + 63) // 64 * 64
        self.logits = torch.empty(s.total_q, self.ld, device=dev)
        self.idx = torch.empty(s.total_q, s.topk, dtype=torch.int32, device=dev)
        self.out = torch.empty(s.total_q, s.heads, s.d_v, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(s.total_q, s.heads, device=dev)
        n = L.dsa_decode_workspace_size(self.batch, s.topk, s.heads, s.d_v)
        self.ws = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
        m = L.dsa_sparse_mla_decode_workspace_size(s.total_q, s.heads, s.d_v, s.topk)
        self.mla_ws = torch.empty(max(m, 16), dtype=torch.uint8, device=dev)
        self.has_combine = m > 0   # the decode MLA splits each row's list and merges

    def fused(self):
        s = self.s
        if self.mode == "decode":
            L.dsa_decode(self.wl.q_idx, None, self.wl.w, self.kc, s.topk, self.wl.q, self.kv,
                         self.batch, s.d_v, s.softmax_scale, self.out, self.lse, self.idx,
                         self.ws)
        else:
            for f in self.stages():
                f()

    def stages(self):
        s, wl = self.s, self.wl
        mla = (lambda: L.dsa_sparse_mla_decode(wl.q, self.kv, self.batch, self.idx, s.d_v,
                                               s.softmax_scale, self.out, self.lse, self.mla_ws)) \
            if self.mode == "decode" else \
            (lambda: L.dsa_sparse_mla_prefill(wl.q, self.kv, self.batch, self.idx, s.d_v,
                                              s.softmax_scale, self.out, self.lse))
        return [lambda: L.dsa_indexer_logits(wl.q_idx, None, wl.w, self.kc, self.batch,
                                             self.logits),
                lambda: L.dsa_topk(self.logits, self.batch, s.topk, self.idx),
                mla]

    def launches_per_step(self) -> int:
        combine = 1 if (self.mode == "decode" and self.has_combine) else 0
        return 3 + combine

    # algorithmic bytes / flops per stage (what the method must touch)
    def work(self):
        s, wl = self.s, self.wl
        T, k = s.total_q, s.topk
        pos = []
        for b in range(s.num_seqs):
            for i in range(s.nq[b]):
                pos.append(s.seq_lens[b] - s.nq[b] + i)
        n_pairs = sum(p + 1 for p in pos)                     # causal (query, key) pairs
        keys_read = sum(s.seq_lens) if self.mode == "decode" else s.max_seq_len * s.num_seqs
        idx_bytes_key = s.idx_dim * (1 if s.idx_fp8 else 4) + 4
        n_sel = sum(min(k, p + 1) for p in pos)
        kv_row = s.d_qk * (1 if s.kv_fp8 else 2) + (4 if s.kv_fp8 else 0)
        q_bytes = T * s.heads * s.d_qk * 2
        o_bytes = T * s.heads * s.d_v * 2
        return {
            "indexer": {"bytes": keys_read * idx_bytes_key + T * s.idx_heads * (s.idx_dim + 4)
                        + n_pairs * 4,
                        "flops": 2 * n_pairs * s.idx_heads * s.idx_dim},
            "topk": {"bytes": n_pairs * 4 + T * k * 4, "flops": 0},
            "mla": {"bytes": n_sel * (kv_row + 8) + q_bytes + o_bytes + T * s.heads * 4,
                    "flops": 2 * n_sel * s.heads * (s.d_qk + s.d_v)},
        }


def sparse_ratio(spec) -> float:
    """Mean over query rows of the attended fraction of the causal keys, min(k, pos+1) /
    (pos+1) -- what a serving stack reports as its sparse-attention ratio."""
    tot, n = 0.0, 0
    for b in range(spec.num_seqs):
        for i in range(spec.nq[b]):
            pos = spec.seq_lens[b] - spec.nq[b] + i
            tot += min(spec.topk, pos + 1) / (pos + 1)
            n += 1
    return round(tot / max(n, 1), 5)


def timed_loop(fn_list, steps, flush, stream):
    """K steps; before each, a 256 MiB write flushes L2; events around every stage."""
    evs = []
    for _ in range(steps):
        flush.zero_()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(len(fn_list) + 1)]
        e[0].record(stream)
        for j, f in enumerate(fn_list):
            f()
            e[j + 1].record(stream)
        evs.append(e)
    torch.cuda.synchronize()
    return [[e[j].elapsed_time(e[j + 1]) for j in range(len(fn_list))] for e in evs]


def run_dsa(args, rank, world, dev):
    spec_fn, mode = WORKLOADS[args.workload]
    if mode == "store":
        return run_store(args, rank, world, dev)
    if mode == "chunked":
        return run_chunked(args, rank, world, dev)
    spec = spec_fn()
    spec.seed = R.replica_seed(spec.seed, rank)  # independent replica inputs per rank
    wl = W.make(spec, device=dev)
    st = Step(wl, mode)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    for _ in range(max(3, args.warmup)):
        st.fused()
    torch.cuda.synchronize()
    if L.dsa_device_check() != 0:
        raise RuntimeError("device check recorded an error during warm-up")

    # ---- headline: K fused steps
    R.barrier(world, dev)
    with ClockSampler(torch.cuda.current_device()) as clk:
        step_ms = [sum(x) for x in timed_loop([st.fused], args.steps, flush, stream)]
    R.barrier(world, dev)
    ms = statistics.mean(step_ms)
    ms_max = R.max_over_ranks(ms, world, dev)
    tokens = spec.total_q
    value = R.job_throughput(tokens, ms_max, world)

    # ---- per-stage breakdown of the same kernels (roofline)
    R.barrier(world, dev)
    stage_ms = timed_loop(st.stages(), args.steps, flush, stream)
    R.barrier(world, dev)
    names = ["indexer", "topk", "mla"]
    mean_stage = {n: statistics.mean(r[j] for r in stage_ms) for j, n in enumerate(names)}
    work = st.work()
    hbm_gbs, bf16_tf, peak_kind = measured_peaks()
    dom = max(mean_stage, key=mean_stage.get)
    if mode == "decode" or dom == "topk":
        achieved = work[dom]["bytes"] / (mean_stage[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_gbs, "unit": "GB/s"}
    else:
        fl = work[dom]["flops"] / (mean_stage[dom] / 1e3) / 1e12
        peak = fp8_peak()[0] if dom == "indexer" else bf16_tf
        roof = {"bound": "tensor", "achieved": round(fl, 1), "peak": peak, "unit": "TFLOP/s"}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
    kernel_file = {"indexer": "indexer_tc.cu", "topk": "topk.cu", "mla": "mla_tc.cu"}[dom]
    roof["traffic"] = ncu_traffic(args.workload, kernel_file)
    roof["kernel"] = dom
    roof["peak_source"] = (f"{peak_kind} ({'burst' if roof['unit'] == 'GB/s' else 'burst bf16'})"
                           if not (roof["unit"] == "TFLOP/s" and dom == "indexer") else fp8_peak()[1])
    if mode == "prefill":
        ix = work["indexer"]["flops"] / (mean_stage["indexer"] / 1e3) / 1e12
        roof["indexer_fp8"] = {"achieved": round(ix, 1), "peak": fp8_peak()[0],
                               "frac": round(ix / fp8_peak()[0], 4), "peak_source": fp8_peak()[1]}
    roof["stage_ms"] = {n: round(v, 4) for n, v in mean_stage.items()}
    roof["algorithmic_bytes_per_launch"] = work[dom]["bytes"]
    if mode == "prefill":
        # the same selection without the [T][L] logits: dsa_indexer_topk over L2-sized
        # row blocks (reported beside the staged calls the step uses)
        ws_n = L.dsa_indexer_topk_workspace_size(st.batch)
        ws_fused = torch.empty(max(ws_n, 16), dtype=torch.uint8, device=dev)
        idx_f = torch.empty_like(st.idx)
        fused_call = lambda: L.dsa_indexer_topk(wl.q_idx, None, wl.w, st.kc, st.batch,  # noqa: E731
                                                spec.topk, idx_f, workspace=ws_fused)
        for _ in range(2):
            fused_call()
        R.barrier(world, dev)
        f_ms = statistics.mean(r[0] for r in timed_loop([fused_call], args.steps, flush, stream))
        roof["indexer_topk_fused"] = {
            "ms": round(f_ms, 4), "staged_ms": round(mean_stage["indexer"] + mean_stage["topk"], 4),
            "logits_bytes_staged": int(st.logits.numel() * 4), "logits_bytes_fused": int(ws_n),
            "same_selection": bool(torch.equal(idx_f, st.idx))}

    # ---- end to end through host buffers: every step uploads its queries (q_idx, w, q)
    # from pinned host memory and downloads o, as a serving loop does -- the uploads of
    # step i+1 and the download of step i-1 overlap step i on two copy streams.  Two
    # independent batches (different seeds, together larger than L2) alternate, so no
    # step finds its inputs in L2 from the step before.
    e2e = None
    if mode == "decode" and not args.no_e2e:
        spec_b = spec_fn()
        spec_b.seed = R.replica_seed(spec.seed + 7, rank)
        sts = [st, Step(W.make(spec_b, device=dev), mode)]
        host = []
        for x in sts:
            host.append({"q_idx": x.wl.q_idx.cpu().pin_memory(), "w": x.wl.w.cpu().pin_memory(),
                         "q": x.wl.q.cpu().pin_memory(),
                         "out": torch.empty(x.out.shape, dtype=x.out.dtype).pin_memory()})
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_ready, comp_done, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def pipelined(n, cs):
            for i in range(n):
                x, hb = sts[i & 1], host[i & 1]
                with torch.cuda.stream(h2d_s):
                    if i >= 2:
                        h2d_s.wait_event(comp_done[i & 1])   # step i-2 done with these inputs
                    x.wl.q_idx.copy_(hb["q_idx"], non_blocking=True)
                    x.wl.w.copy_(hb["w"], non_blocking=True)
                    x.wl.q.copy_(hb["q"], non_blocking=True)
                    in_ready[i & 1].record(h2d_s)
                cs.wait_event(in_ready[i & 1])
                if i >= 2:
                    cs.wait_event(out_free[i & 1])         # o of step i-2 downloaded
                x.fused()
                comp_done[i & 1].record(cs)
                with torch.cuda.stream(d2h_s):
                    d2h_s.wait_event(comp_done[i & 1])
                    hb["out"].copy_(x.out, non_blocking=True)
                    out_free[i & 1].record(d2h_s)
            for e in out_free:
                cs.wait_event(e)

        h2d_s.wait_stream(stream)
        d2h_s.wait_stream(stream)
        pipelined(4, stream)
        torch.cuda.synchronize(dev)
        # the K steps are captured once as a CUDA graph (all copies and kernels of every
        # step), so that host-side enqueue speed does not set the rate; eager fallback
        graph = None
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                cs = torch.cuda.current_stream()
                h2d_s.wait_stream(cs)
                d2h_s.wait_stream(cs)
                pipelined(args.steps, cs)
            g.replay()
            torch.cuda.synchronize(dev)
            graph = g
        except RuntimeError:
            torch.cuda.synchronize(dev)
        R.barrier(world, dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        if graph is not None:
            graph.replay()
        else:
            h2d_s.wait_stream(stream)
            d2h_s.wait_stream(stream)
            pipelined(args.steps, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = R.max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
        h2d = sum(host[0][k].numel() * host[0][k].element_size() for k in ("q_idx", "w", "q"))
        e2e = {"value": round(R.job_throughput(tokens, e_ms, world), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": host[0]["out"].numel() * 2,
               "ms_per_step": round(e_ms, 4),
               "method": "pinned H2D of q_idx, w, q and D2H of o every step; copies of "
                         "neighbouring steps overlap on two copy streams; two batches "
                         "alternate (inputs larger than L2); "
                         + ("the K steps replayed as one CUDA graph" if graph is not None
                            else "eager launches (graph capture unavailable)")}
        if graph is not None:
            del graph

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, mode, args.cpu_seconds)
        cpu["kind"] = "oracle"

    if L.dsa_device_check() != 0:
        raise RuntimeError("device check recorded an error in the timed region")
    return {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8 e4m3 (indexer) + bf16 (MLA), fp32 accumulate",
        "data": "synthetic (seeded N(0,1) caches and queries)",
        "config": {"workload": spec.name, "mode": mode, "num_seqs": spec.num_seqs,
                   "context": spec.max_seq_len, "queries": spec.total_q, "topk": spec.topk,
                   "indexer": f"{'fp8 e4m3' if spec.idx_fp8 else 'fp32'} {spec.idx_heads}x"
                              f"{spec.idx_dim}, page 64, per-token scale",
                   "mla": f"{spec.heads} heads, d_qk {spec.d_qk}, d_v {spec.d_v}, "
                          f"{'fp8' if spec.kv_fp8 else 'bf16'} latent KV page 1",
                   "l2": "flushed between steps (256 MiB write)",
                   "sparse_attention_ratio": sparse_ratio(spec),
                   "parallelism": f"replicas x{world}"},
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.summary(),
        "gpu_launches": st.launches_per_step() * args.steps,
        "gpu_launches_note": "fused decode steps in the timed loop (indexer, top-k, attention, merge)",
    }


# ----------------------------------------------------------------------------- chunked prefill
def chunked_work(spec):
    """Algorithmic work of one whole chunked prefill, per stage: causal (query, key) pairs
    for the indexer, min(k, pos+1) selected rows per query for the attention."""
    Lt, k = spec.seq_len, spec.topk
    n_pairs = Lt * (Lt + 1) // 2
    n_sel = sum(min(k, t + 1) for t in range(Lt))
    kv_row = spec.d_qk + 4                                  # fp8 codes + scale
    store = Lt * (spec.idx_dim * 2 + spec.idx_dim + 4 + 8) + Lt * (spec.d_qk * 2 + spec.d_qk + 4 + 8)
    return {
        "store": {"bytes": store, "flops": 0},
        "indexer": {"flops": 2 * n_pairs * spec.idx_heads * spec.idx_dim},
        "topk": {"bytes": n_pairs * 4 + Lt * k * 4, "flops": 0},
        "mla": {"flops": 2 * n_sel * spec.heads * (spec.d_qk + spec.d_v),
                "bytes": n_sel * (kv_row + 8) + Lt * spec.heads * (spec.d_qk + spec.d_v) * 2},
        "n_pairs": n_pairs, "n_sel": n_sel,
    }


def run_chunked(args, rank, world, dev):
    spec = W.ChunkedSpec()
    spec.seed = R.replica_seed(spec.seed, rank)
    cw = W.make_chunked(spec, device=dev)
    cp = CH.ChunkedPrefill(cw)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    for _ in range(max(3, args.warmup)):
        cp.step()
    torch.cuda.synchronize()
    if L.dsa_device_check() != 0:
        raise RuntimeError("device check recorded an error during warm-up")

    # ---- headline: K whole prefills (16 chunks each)
    R.barrier(world, dev)
    with ClockSampler(torch.cuda.current_device()) as clk:
        step_ms = [sum(x) for x in timed_loop([cp.step], args.steps, flush, stream)]
    R.barrier(world, dev)
    ms_max = R.max_over_ranks(statistics.mean(step_ms), world, dev)
    tokens = spec.seq_len
    value = R.job_throughput(tokens, ms_max, world)

    # ---- per stage over all chunks: the step's own calls (store, indexer + top-k in
    # row blocks, attention), then the indexer and the top-k staged through a full logits
    # buffer, which times the indexer kernel alone
    R.barrier(world, dev)
    stage_ms = timed_loop(cp.stages(), args.steps, flush, stream)
    names = ["store", "select", "mla"]
    mean_stage = {n: statistics.mean(r[j] for r in stage_ms) for j, n in enumerate(names)}
    ld = (spec.seq_len + 63) // 64 * 64
    logits = torch.empty(spec.chunk_q, ld, device=dev)
    idx_s = torch.empty(spec.chunk_q, spec.topk, dtype=torch.int32, device=dev)

    def staged(which):
        def f():
            for c in range(spec.n_chunks):
                if which == "indexer":
                    L.dsa_indexer_logits(cw.q_idx[c], None, cw.w[c], cp.kc, cp.batches[c], logits)
                else:
                    L.dsa_topk(logits, cp.batches[c], spec.topk, idx_s)
        return f
    # the top-k of every chunk reads the last chunk's logits rows (same shape of work)
    staged("indexer")()
    sm = timed_loop([staged("indexer"), staged("topk")], max(2, args.steps // 2), flush, stream)
    R.barrier(world, dev)
    mean_stage["indexer"] = statistics.mean(r[0] for r in sm)
    mean_stage["topk"] = statistics.mean(r[1] for r in sm)
    # the selection again with the minimum workspace: L2-sized row blocks (no chunk-sized
    # logits buffer, hundreds of launches per step)
    ws_l2 = torch.empty(max(max(L.dsa_indexer_topk_workspace_size(b) for b in cp.batches), 16),
                        dtype=torch.uint8, device=dev)

    def select_l2():
        for c in range(spec.n_chunks):
            L.dsa_indexer_topk(cw.q_idx[c], None, cw.w[c], cp.kc, cp.batches[c], spec.topk,
                               idx_s, workspace=ws_l2)
    select_l2()
    sl = timed_loop([select_l2], max(2, args.steps // 2), flush, stream)
    R.barrier(world, dev)
    mean_stage["select_l2_blocks"] = statistics.mean(r[0] for r in sl)
    del logits, idx_s, ws_l2
    work = chunked_work(spec)
    hbm_gbs, bf16_tf, peak_kind = measured_peaks()
    fp8_tf, fp8_src = fp8_peak()
    ix = work["indexer"]["flops"] / (mean_stage["indexer"] / 1e3) / 1e12
    mla = work["mla"]["flops"] / (mean_stage["mla"] / 1e3) / 1e12
    per = {"indexer": {"achieved": round(ix, 1), "peak": fp8_tf, "frac": round(ix / fp8_tf, 4),
                       "unit": "TFLOP/s", "peak_source": fp8_src},
           "mla": {"achieved": round(mla, 1), "peak": bf16_tf, "frac": round(mla / bf16_tf, 4),
                   "unit": "TFLOP/s", "peak_source": f"{peak_kind} (burst bf16)"}}
    dom = "indexer" if mean_stage["indexer"] >= mean_stage["mla"] else "mla"
    kernel_file = {"indexer": "indexer_tc.cu", "mla": "mla_tc.cu"}[dom]
    roof = {"bound": "tensor", **per[dom], "kernel": dom,
            "traffic": ncu_traffic(args.workload, kernel_file),
            "indexer_fp8": per["indexer"], "mla_bf16": per["mla"],
            "stage_ms": {n: round(v, 3) for n, v in mean_stage.items()},
            "stage_note": "store / select (dsa_indexer_topk, one row block per chunk) / mla are "
                          "the step's calls over all 16 chunks; indexer and topk are the same "
                          "work as two separate calls; select_l2_blocks is dsa_indexer_topk "
                          "with the minimum workspace (L2-sized row blocks)",
            "flops_per_step": {"indexer": work["indexer"]["flops"], "mla": work["mla"]["flops"]},
            "store": {"achieved_gbs": round(work["store"]["bytes"] / (mean_stage["store"] / 1e3)
                                            / 1e9, 1), "peak": hbm_gbs}}

    # ---- end to end through host buffers: every chunk's inputs (new key / KV rows, slot
    # maps, q_idx, w, q) are uploaded from pinned host memory and its output o is read
    # back; the uploads of chunk c+1 and the download of chunk c-1 overlap chunk c on two
    # copy streams (two device input sets and two pinned output buffers alternate)
    e2e = None
    if not args.no_e2e:
        try:
            e2e = _chunked_e2e(args, cw, cp, stream, world, dev, tokens)
        except RuntimeError as ex:   # e.g. pinned host memory unavailable
            torch.cuda.synchronize(dev)
            e2e = {"value": None, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0, "error": str(ex)[:200]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = chunked_cpu_baseline(cw, args.cpu_seconds)
    if L.dsa_device_check() != 0:
        raise RuntimeError("device check recorded an error in the timed region")
    launches = cp.launches_per_step()
    res = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8 e4m3 (indexer, latent KV cache) + bf16 q (MLA), fp32 accumulate",
        "data": "synthetic (seeded N(0,1) key / latent-KV rows and queries)",
        "config": {"workload": spec.name, "mode": "chunked prefill", "context": spec.seq_len,
                   "chunks": spec.n_chunks, "chunk_queries": spec.chunk_q, "topk": spec.topk,
                   "indexer": f"fp8 e4m3 {spec.idx_heads}x{spec.idx_dim}, page 64, per-token "
                              "scale (written by dsa_cache_store each chunk)",
                   "mla": f"{spec.heads} heads, d_qk {spec.d_qk}, d_v {spec.d_v}, fp8 latent "
                          "KV page 1 (written by dsa_cache_store each chunk)",
                   "step": "per chunk: dsa_cache_store x2, dsa_indexer_topk (workspace for "
                           "the chunk's whole logits: one indexer and one top-k launch), "
                           "dsa_sparse_mla_prefill",
                   "l2": "flushed between steps (256 MiB write); the inputs (~21 GB) exceed L2",
                   "sparse_attention_ratio": round(work["n_sel"] / work["n_pairs"], 5),
                   "parallelism": f"replicas x{world}"},
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.summary(),
        "gpu_launches": launches * args.steps,
        "gpu_launches_note": f"{launches} launches per whole prefill (per chunk: 2 stores, "
                             "indexer and top-k per row block, attention)",
    }
    del cp, cw
    torch.cuda.empty_cache()
    if not args.no_extras:
        res["extra"] = {}
        for wname in ("decode_b32_ctx8192", "decode_b64_ctx64k-128k_fp8kv"):
            sub = argparse.Namespace(**vars(args))
            sub.workload, sub.no_cpu_baseline, sub.no_e2e = wname, True, True
            r = run_dsa(sub, rank, world, dev)
            res["extra"][wname] = {k: r[k] for k in ("value", "unit", "ms_per_step", "config")}
            rf = r["roofline"]
            res["extra"][wname]["roofline"] = {k: rf.get(k) for k in (
                "bound", "kernel", "achieved", "peak", "unit", "frac", "stage_ms")}
            res["extra"][wname]["clocks"] = r["clocks"]
            res["gpu_launches"] += r["gpu_launches"]
            torch.cuda.empty_cache()
        res["gpu_launches_note"] += "; plus the two decode lines under 'extra'"
    return res


def _chunked_e2e(args, cw, cp, stream, world, dev, tokens):
    s = cw.spec
    C = s.n_chunks
    names = ("k_new", "kv_new", "k_slots", "kv_slots")
    host = {n: [getattr(cw, n)[cp.rows(c)].cpu().pin_memory() for c in range(C)] for n in names}
    for n in ("q_idx", "w", "q"):
        host[n] = [getattr(cw, n)[c].cpu().pin_memory() for c in range(C)]
    dev_in = [{n: torch.empty_like(host[n][0], device=dev) for n in host} for _ in range(2)]
    out_host = [torch.empty(cp.out.shape[1:], dtype=cp.out.dtype).pin_memory() for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, comp_done, out_free = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def run(n_steps, cs):
        i = 0
        for _ in range(n_steps):
            for c in range(C):
                b = i & 1
                d = dev_in[b]
                with torch.cuda.stream(h2d_s):
                    if i >= 2:
                        h2d_s.wait_event(comp_done[b])   # chunk i-2 done with this input set
                    for n in host:
                        d[n].copy_(host[n][c], non_blocking=True)
                    in_ready[b].record(h2d_s)
                cs.wait_event(in_ready[b])
                if i >= 2:
                    cs.wait_event(out_free[b])          # output of chunk i-2 read back
                cp.store(c, d["k_new"], d["kv_new"], d["k_slots"], d["kv_slots"], stream=cs)
                cp.select(c, d["q_idx"], d["w"], cp.idx[b], stream=cs)
                cp.attend(c, d["q"], cp.idx[b], cp.out[b], cp.lse[b], stream=cs)
                comp_done[b].record(cs)
                with torch.cuda.stream(d2h_s):
                    d2h_s.wait_event(comp_done[b])
                    out_host[b].copy_(cp.out[b], non_blocking=True)
                    out_free[b].record(d2h_s)
                i += 1
        for e in out_free:
            cs.wait_event(e)

    h2d_s.wait_stream(stream)
    d2h_s.wait_stream(stream)
    run(1, stream)
    torch.cuda.synchronize(dev)
    R.barrier(world, dev)
    n_steps = max(1, min(args.steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h2d_s.wait_stream(stream)
    d2h_s.wait_stream(stream)
    e0.record(stream)
    run(n_steps, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e_ms = R.max_over_ranks(e0.elapsed_time(e1) / n_steps, world, dev)
    h2d = sum(t.numel() * t.element_size() for n in host for t in host[n])
    d2h = C * out_host[0].numel() * out_host[0].element_size()
    return {"value": round(R.job_throughput(tokens, e_ms, world), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e_ms, 3),
            "steps": n_steps,
            "method": "per chunk: pinned H2D of the new key / latent-KV rows, slot maps, q_idx, "
                      "w and q, D2H of o; the next chunk's uploads and the previous chunk's "
                      "download overlap the chunk on two copy streams; eager launches"}


def _chunked_oracle_setup(cw):
    """The oracle's own FP8 caches for the whole prompt (its cache_store on the rows), as
    the inputs of its per-row indexer and attention."""
    import numpy as np
    from oracle import oracle as O
    s = cw.spec
    kx = cw.k_new.view(torch.int16).cpu().numpy().view(np.uint16)
    vx = cw.kv_new.view(torch.int16).cpu().numpy().view(np.uint16)
    slots = np.arange(s.seq_len, dtype=np.int64)
    kd, ks = O.cache_store(kx, O.BF16, slots, np.zeros((s.seq_len, s.idx_dim), np.uint8), O.E4M3,
                           np.zeros(s.seq_len, np.float32))
    vd, vs = O.cache_store(vx, O.BF16, slots, np.zeros((s.seq_len, s.d_qk), np.uint8), O.E4M3,
                           np.zeros(s.seq_len, np.float32))
    dev = cw.device
    return (torch.from_numpy(kd).to(dev).view(W.FP8).reshape(-1, W.INDEXER_PAGE, s.idx_dim),
            torch.from_numpy(ks).to(dev).reshape(-1, W.INDEXER_PAGE),
            torch.from_numpy(vd).to(dev).view(W.FP8), torch.from_numpy(vs).to(dev))


def _chunked_oracle_rows(cw, caches, positions):
    """Oracle indexer + top-k + attention for the query rows at the given prompt positions."""
    import numpy as np
    s = cw.spec
    for c in np.unique(positions // s.chunk_q):
        rows = positions[positions // s.chunk_q == c] - c * s.chunk_q
        wl = W.chunk_view(cw, int(c), *caches)
        _oracle_rows(wl, "prefill", rows)


def _chunk7_rows(cw, n, seed):
    """n query rows of chunk 7 (prompt positions 57344..65535): a row's oracle cost grows
    linearly with its position, and this chunk's mean position (61440) is within 7% of the
    whole prompt's (65535.5), so its rows/s estimates the whole prefill's tokens/s; rows
    of one chunk also run in parallel in the oracle."""
    import numpy as np
    s = cw.spec
    rng = np.random.default_rng(seed)
    return 7 * s.chunk_q + np.sort(rng.choice(s.chunk_q, n, replace=False))


def chunked_cpu_baseline(cw, seconds):
    """The oracle on a bounded row sample (chunk 7, one row per host thread at least)."""
    from oracle import oracle as O
    caches = _chunked_oracle_setup(cw)
    threads = O.num_threads()
    t0 = time.perf_counter()
    _chunked_oracle_rows(cw, caches, _chunk7_rows(cw, threads, 1))
    first = time.perf_counter() - t0
    n = int(max(threads, min(256, threads * round(seconds / max(first, 1e-3)))))
    pos = _chunk7_rows(cw, n, 2)
    t0 = time.perf_counter()
    _chunked_oracle_rows(cw, caches, pos)
    dt = time.perf_counter() - t0
    return {"value": round(len(pos) / dt, 3), "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{len(pos)} query rows of chunk 7 (positions 57344-65535, mean cost within "
                      f"7% of the whole {cw.spec.seq_len}-token prompt's) -- indexer + top-k + MLA "
                      f"per row in fp64 over the oracle's own FP8 caches, {dt:.1f} s; rows/s "
                      "estimates the whole prefill's tokens/s"}


# ----------------------------------------------------------------------------- cache writes
def _store_bytes(x, out_elem):
    """Algorithmic bytes of one store call: rows in, codes + scale out, the slot map."""
    n, dim = x.shape
    return n * (dim * x.element_size() + dim * out_elem + (4 if out_elem == 1 else 0) + 8)


def run_store(args, rank, world, dev):
    spec = W.store_prompt_128k()
    spec.seed = R.replica_seed(spec.seed, rank)
    wl = W.make_store(spec, device=dev)
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    calls = [lambda: L.dsa_cache_store(wl.k_new, wl.k_slots, wl.k_pages, wl.k_scale),
             lambda: L.dsa_cache_store(wl.kv_new, wl.kv_slots, wl.kv, wl.kv_scale)]

    def step():
        for c in calls:
            c()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if L.dsa_device_check() != 0:
        raise RuntimeError("device check recorded an error during warm-up")
    R.barrier(world, dev)
    with ClockSampler(torch.cuda.current_device()) as clk:
        step_ms = [sum(x) for x in timed_loop([step], args.steps, flush, stream)]
    R.barrier(world, dev)
    ms_max = R.max_over_ranks(statistics.mean(step_ms), world, dev)
    n = spec.n_tokens
    value = R.job_throughput(n, ms_max, world)
    stage_ms = timed_loop(calls, args.steps, flush, stream)
    mean_stage = {nm: statistics.mean(r[j] for r in stage_ms)
                  for j, nm in enumerate(["key_store", "kv_store"])}
    kv_elem = wl.kv.element_size()
    work = {"key_store": _store_bytes(wl.k_new, 1), "kv_store": _store_bytes(wl.kv_new, kv_elem)}
    hbm_gbs, _, peak_kind = measured_peaks()
    dom = "kv_store"
    achieved = work[dom] / (mean_stage[dom] / 1e3) / 1e9
    roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_gbs, "unit": "GB/s",
            "frac": round(achieved / hbm_gbs, 4),
            "traffic": ncu_traffic(args.workload, "cache_store.cu"), "kernel": dom,
            "peak_source": f"{peak_kind} (burst)",
            "stage_ms": {k: round(v, 4) for k, v in mean_stage.items()},
            "algorithmic_bytes_per_launch": work[dom]}

    # end to end: the rows and slot maps come from pinned host memory each step and
    # the written per-token scales go back (neighbouring steps overlap on copy streams)
    names = ("k_new", "kv_new", "k_slots", "kv_slots")
    host = {k: getattr(wl, k).cpu().pin_memory() for k in names}
    back = {"k_scale": torch.empty(wl.k_scale.shape).pin_memory(),
            "kv_scale": torch.empty(wl.kv_scale.shape).pin_memory()}
    h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    R.barrier(world, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    done, ready = torch.cuda.Event(), torch.cuda.Event()
    h2d_s.wait_stream(stream)
    d2h_s.wait_stream(stream)
    e0.record(stream)
    for i in range(args.steps):
        with torch.cuda.stream(h2d_s):
            if i:
                h2d_s.wait_event(done)
            for k in names:
                getattr(wl, k).copy_(host[k], non_blocking=True)
            ready.record(h2d_s)
        stream.wait_event(ready)
        step()
        done.record(stream)
        with torch.cuda.stream(d2h_s):
            d2h_s.wait_event(done)
            back["k_scale"].copy_(wl.k_scale, non_blocking=True)
            back["kv_scale"].copy_(wl.kv_scale, non_blocking=True)
    stream.wait_stream(d2h_s)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e_ms = R.max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    e2e = {"value": round(R.job_throughput(n, e_ms, world), 1), "unit": "tokens/s",
           "h2d_bytes_per_step": sum(host[k].numel() * host[k].element_size() for k in names),
           "d2h_bytes_per_step": sum(b.numel() * 4 for b in back.values()),
           "ms_per_step": round(e_ms, 4),
           "method": "pinned H2D of the new rows and slot maps, D2H of the written scales, "
                     "every step; eager launches"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = _store_oracle(wl, args.cpu_seconds)
    if L.dsa_device_check() != 0:
        raise RuntimeError("device check recorded an error in the timed region")
    return {
        "metric": "cache-write tokens/s (indexer key + latent KV into FP8 caches) on 1 B200",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, fp8 e4m3 + fp32 scale out",
        "data": "synthetic (seeded N(0,1) rows, 1% x4)",
        "config": {"workload": spec.name, "mode": "store", "tokens": n,
                   "key": f"{spec.idx_dim} dims -> page-64 fp8 cache",
                   "kv": f"{spec.d_qk} dims -> page-1 fp8 cache",
                   "l2": "flushed between steps (256 MiB write)",
                   "parallelism": f"replicas x{world}"},
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.summary(),
        "gpu_launches": 2 * args.steps, "gpu_launches_note": "two cache_store launches per step",
    }


def _store_oracle(wl, seconds, rows=None):
    """The oracle's cache write on a bounded token sample (both caches)."""
    import numpy as np
    from oracle import oracle as O
    n = wl.spec.n_tokens
    if rows is None:
        rows = 4096
    sel = np.arange(min(rows, n))
    kd = wl.k_pages.view(torch.uint8).reshape(-1, wl.spec.idx_dim).cpu().numpy()
    vd = wl.kv.view(torch.uint8).cpu().numpy()
    ks, vs = wl.k_scale.reshape(-1).cpu().numpy(), wl.kv_scale.cpu().numpy()
    kx = wl.k_new[sel].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    vx = wl.kv_new[sel].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    kslot, vslot = wl.k_slots[sel].cpu().numpy(), wl.kv_slots[sel].cpu().numpy()
    t0 = time.perf_counter()
    O.cache_store(kx, O.BF16, kslot, kd, O.E4M3, ks)
    O.cache_store(vx, O.BF16, vslot, vd, O.E4M3, vs)
    dt = time.perf_counter() - t0
    return {"value": round(len(sel) / dt, 1), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{len(sel)} of {n} tokens of {wl.spec.name} (key + KV rows), {dt:.2f} s"}


# ----------------------------------------------------------------------------- oracle arm
def _oracle_rows(wl, mode, rows):
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import _helpers as H
    from oracle import oracle as O
    logits = H.oracle_logits(wl, rows)
    cu = H.np_bits(wl.cu_q)
    lens = H.np_bits(wl.seq_lens)
    sel = O.topk(logits, cu, lens, wl.spec.topk, rows=rows)
    H.oracle_mla(wl, sel, rows)


def cpu_baseline(wl, mode, seconds):
    """The oracle, as it stands, on a bounded row sample of the same workload."""
    import numpy as np
    from oracle import oracle as O
    T = wl.spec.total_q
    t0 = time.perf_counter()
    _oracle_rows(wl, mode, np.array([T - 1]))
    one = time.perf_counter() - t0
    threads = O.num_threads()
    n = int(max(1, min(T, seconds / max(one, 1e-3) * threads)))
    rows = np.linspace(0, T - 1, n).round().astype(np.int64)
    rows = np.unique(rows)
    t0 = time.perf_counter()
    _oracle_rows(wl, mode, rows)
    dt = time.perf_counter() - t0
    return {"value": round(len(rows) / dt, 3), "unit": "tokens/s", "cores": threads,
            "sample": f"{len(rows)} of {T} query rows of {wl.spec.name} (indexer + top-k + MLA "
                      f"per row, fp64), {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import numpy as np
    from oracle import oracle as O
    spec_fn, mode = WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    if mode == "store":
        return _store_reference(args, world, dev)
    if mode == "chunked":
        return _chunked_reference(args, world, dev)
    spec = spec_fn()
    wl = W.make(spec, device=dev)
    T = spec.total_q
    # size each step's sample so the whole run stays within a few minutes
    t0 = time.perf_counter()
    _oracle_rows(wl, mode, np.array([T - 1]))
    one = time.perf_counter() - t0
    threads = O.num_threads()
    budget = 150.0 / max(1, args.steps + args.warmup)
    per_step = int(max(1, min(T, budget / max(one, 1e-3) * threads)))
    rng = np.random.default_rng(0)
    for _ in range(args.warmup):
        _oracle_rows(wl, mode, np.sort(rng.choice(T, per_step, replace=False)))
    times = []
    for _ in range(args.steps):
        rows = np.sort(rng.choice(T, per_step, replace=False))
        t0 = time.perf_counter()
        _oracle_rows(wl, mode, rows)
        times.append(time.perf_counter() - t0)
    ms = statistics.mean(times) * 1e3
    value = per_step / (ms / 1e3)
    sample = (f"{per_step} of {T} query rows per step of {spec.name} (indexer + top-k + MLA, "
              f"fp64)")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded N(0,1) caches and queries)",
        "config": {"workload": spec.name, "mode": mode, "queries": T, "topk": spec.topk},
        "cpu_baseline": {"kind": "oracle", "cores": threads, "sample": sample,
                         "value": round(value, 3), "unit": "tokens/s"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def _chunked_reference(args, world, dev):
    from oracle import oracle as O
    spec = W.ChunkedSpec()
    cw = W.make_chunked(spec, device=dev)
    caches = _chunked_oracle_setup(cw)
    threads = O.num_threads()
    t0 = time.perf_counter()
    _chunked_oracle_rows(cw, caches, _chunk7_rows(cw, threads, 1))
    first = time.perf_counter() - t0
    budget = 150.0 / max(1, args.steps + args.warmup)
    per_step = int(max(1, min(256, threads * budget / max(first, 1e-3))))
    for i in range(args.warmup):
        _chunked_oracle_rows(cw, caches, _chunk7_rows(cw, per_step, 10 + i))
    times = []
    for i in range(args.steps):
        pos = _chunk7_rows(cw, per_step, 100 + i)
        t0 = time.perf_counter()
        _chunked_oracle_rows(cw, caches, pos)
        times.append(time.perf_counter() - t0)
    ms = statistics.mean(times) * 1e3
    value = per_step / (ms / 1e3)
    sample = (f"{per_step} query rows per step of chunk 7 of the {spec.seq_len}-token prompt "
              "(its mean row cost is within 7% of the whole prompt's; indexer + top-k + MLA, "
              "fp64); rows/s estimates the whole prefill's tokens/s")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) key / latent-KV rows and queries)",
        "config": {"workload": spec.name, "mode": "chunked prefill", "context": spec.seq_len,
                   "chunks": spec.n_chunks, "topk": spec.topk},
        "cpu_baseline": {"kind": "oracle", "cores": threads, "sample": sample,
                         "value": round(value, 3), "unit": "tokens/s"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def _store_reference(args, world, dev):
    wl = W.make_store(W.store_prompt_128k(), device=dev)
    for _ in range(args.warmup):
        _store_oracle(wl, 0, rows=2048)
    res = [_store_oracle(wl, 0, rows=2048) for _ in range(args.steps)]
    value = statistics.mean(r["value"] for r in res)
    ms = 2048 / value * 1e3
    return {
        "impl": "reference", "metric": "cache-write tokens/s (indexer key + latent KV into FP8 "
        "caches) on 1 B200", "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded N(0,1) rows, 1% x4)",
        "config": {"workload": wl.spec.name, "mode": "store", "tokens": wl.spec.n_tokens},
        "cpu_baseline": {"kind": "oracle", "cores": 1, "value": round(value, 1),
                         "unit": "tokens/s",
                         "sample": f"2048 of {wl.spec.n_tokens} tokens per step (key + KV)"},
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    if args.fp8_peak:
        print(json.dumps(measure_fp8_peak()), flush=True)
        return
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, dev = R.setup()
    try:
        res = run_dsa(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        R.teardown(world)


if __name__ == "__main__":
    main()
