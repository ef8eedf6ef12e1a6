"""Benchmark of one absorbed-form MLA decode step on B200.

A step is the whole hot path over one batch: mla_cache_append ->
mla_absorb_q -> mla_decode (decode + split combine) -> mla_out_proj, all
through the C ABI (libmla.so). Default workload: DeepSeek-V2 dims, batch 64,
seq_lens ~ U[1024, 8192], paged latent cache (block 64) — the configuration
the >= 70 % roofline target is stated on. Other workloads: --workload NAME.

Usage:
  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
For N > 1 launch under torchrun: every rank runs an independent replica of the
workload on its own GPU (no data-path collective; "scaling": "weak"); the
timing is the max over ranks.
"""
import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mla_latent_kv_33_b200 import synth  # noqa: E402

METRIC = "MLA decode µs/step, latent-cache HBM GB/s and TFLOP/s vs roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def decode_traffic(workload="v2_b64_paged"):
    """DRAM bytes of one k_decode launch on the workload, from the committed ncu
    summary, or None when there is none or the decode source has changed since
    that capture."""
    import hashlib
    here = os.path.dirname(os.path.abspath(__file__))
    try:
        doc = open(os.path.join(here, "profiles", f"k_decode_{workload}.md")).read()
        src = open(os.path.join(here, "mla_latent_kv_33_b200", "csrc", "decode_tc.cuh"), "rb").read()
    except OSError:
        return None
    fields = dict(l.split(": ", 1) for l in doc.splitlines() if l.startswith(("traffic_bytes_per_launch:",
                                                                              "decode_source_sha256_16:")))
    if fields.get("decode_source_sha256_16", "").strip() != hashlib.sha256(src).hexdigest()[:16]:
        return None
    return int(fields["traffic_bytes_per_launch"])


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="v2_b64_paged", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="launch every call from the host (no CUDA graph)")
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch kernels without programmatic dependent launch (mla_set_launch_overlap off)")
    ap.add_argument("--cpu-sample-s", type=float, default=15.0, help="target seconds of oracle work")
    ap.add_argument("--num-splits", type=int, default=0,
                    help="mla_decode num_splits: 0 = automatic plan, S > 0 = each token row in min(S, its tiles) pieces")
    ap.add_argument("--breakdown", action="store_true",
                    help="diagnostic: also time the front of the step (append + query chain) and its tail "
                         "(W_UV readout) with event pairs in the timed graph; the extra nodes add to the step time")
    ap.add_argument("--with-o-proj", action="store_true",
                    help="add the output projection y = W_O o (mla_o_proj) to every step and time it on its own")
    ap.add_argument("--o-proj-absorbed", action="store_true",
                    help="with --with-o-proj: y = W_OV o_lat (mla_o_proj_latent, W_UV absorbed into W_O) in place of "
                         "the W_UV readout and W_O")
    ap.add_argument("--fused-front-end", action="store_true",
                    help="append and absorb in one call (mla_front_end: h read once) instead of two calls on two streams")
    ap.add_argument("--merged-absorb", action="store_true",
                    help="absorb with the merged matrix W_UK_h^T W_UQ_h (mla_absorb_q_merged)")
    ap.add_argument("--order-a", action="store_true",
                    help="attention in order A (mla_query_heads + mla_attend_order_a: decompress K/V per head, then "
                         "192-d attention) in place of absorb + decode + W_UV readout; default workload v2_prefill_c512")
    a = ap.parse_args()
    if a.order_a and (a.fused_front_end or a.merged_absorb or a.with_o_proj or a.num_splits):
        ap.error("--order-a replaces the absorb, the decode and the readout: no other path option applies")
    if a.order_a and "--workload" not in sys.argv:
        a.workload = "v2_prefill_c512"
    if a.o_proj_absorbed and not a.with_o_proj:
        ap.error("--o-proj-absorbed needs --with-o-proj")
    if a.merged_absorb and a.fused_front_end:
        ap.error("--merged-absorb and --fused-front-end are exclusive")
    return a


L2_BYTES = 126 * 1024 * 1024


def cache_copies(cache_bytes):
    """Copies of the latent cache the timed loop rotates through, so that a
    step never finds its cache in L2 left by the step before: one when the cache
    alone exceeds L2, else enough to cover twice the L2 size."""
    if cache_bytes > L2_BYTES:
        return 1
    return min(8, -(-2 * L2_BYTES // cache_bytes))


# ------------------------------------------------------------------ clocks --

class ClockSampler:
    """Samples of SM clock and throttle reasons, each stamped with the host time
    it was taken, so that the summary keeps only the samples taken while the
    timed region ran (mark() brackets it). NVML is read in-process every ~2 ms
    (read-only queries), so that even a timed region of a few tens of
    milliseconds holds a dozen samples; without NVML, nvidia-smi is polled every
    20 ms instead. Both record the same fields in the same line format. The GPU
    is addressed by UUID, which stays right under CUDA_VISIBLE_DEVICES."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    PERIOD_S = 0.002  # NVML polling period

    def __init__(self, gpu_id, nvml=None):
        self.gpu = gpu_id
        self.proc = None
        self.poller = None
        self.stop = threading.Event()
        self.nvml = nvml  # the pynvml module (injectable for tests); None: import it
        self.samples = []  # (host time, line)
        self.window = None

    def _nvml_handle(self):
        nv = self.nvml
        if nv is None:
            import pynvml as nv
        nv.nvmlInit()
        try:
            g = str(self.gpu)
            h = nv.nvmlDeviceGetHandleByUUID(g) if g.startswith("GPU-") else nv.nvmlDeviceGetHandleByIndex(int(g))
            smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception:
            nv.nvmlShutdown()
            raise
        self.nvml = nv
        return h, smax

    def _poll(self, h, smax):
        nv = self.nvml
        bits = (nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap)
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                watts = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
            except Exception:
                break
            flags = ", ".join("Active" if mask & b else "Not Active" for b in bits)
            self.samples.append((time.perf_counter(), f"0, {sm}, {smax}, {watts:.2f}, {mask:#x}, {flags}\n"))
            self.stop.wait(self.PERIOD_S)

    def _read(self):
        for line in self.proc.stdout:
            if line.strip():
                self.samples.append((time.perf_counter(), line))

    def __enter__(self):
        try:
            h, smax = self._nvml_handle()
        except Exception:
            h = None
        if h is not None:
            self.poller = threading.Thread(target=self._poll, args=(h, smax), daemon=True)
            self.poller.start()
            t0 = time.perf_counter()
            while not self.samples and time.perf_counter() - t0 < 5.0 and self.poller.is_alive():
                time.sleep(0.001)
            if self.samples:
                return self
            self.stop.set()  # NVML answered the set-up but not the queries: fall back to nvidia-smi
            self.poller.join(timeout=5)
            self.poller = None
            self.nvml.nvmlShutdown()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        t0 = time.perf_counter()
        while not self.samples and time.perf_counter() - t0 < 5.0 and self.proc.poll() is None:
            time.sleep(0.01)  # sampling is running before the caller starts its timed region
        return self

    def mark(self, t_begin, t_end):
        self.window = (t_begin, t_end)

    def __exit__(self, *a):
        if self.poller is not None:
            self.stop.set()
            self.poller.join(timeout=5)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.reader.join(timeout=5)

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = self.samples
        if self.window is not None:
            a, b = self.window
            inside = [x for x in lines if a <= x[0] <= b]
            # a timed region shorter than the sampling period may hold no sample: keep the nearest one
            lines = inside or sorted(lines, key=lambda x: abs(x[0] - 0.5 * (a + b)))[:1]
        for _, l in lines:
            parts = [x.strip() for x in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_id_for_smi(torch, local_rank):
    """nvidia-smi id of this process's CUDA device (its UUID when torch exposes it)."""
    try:
        u = str(torch.cuda.get_device_properties(local_rank).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(local_rank)


# ----------------------------------------------------------------- our arm --

def upload(x, torch, dev):
    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    w = x.w
    W = {k: bf(v) for k, v in x.weights_bits.items()}
    cache_t = bf(x.cache)
    bt = None if x.block_table is None else torch.from_numpy(x.block_table).to(dev)
    return W, cache_t, bt


def percentiles_us(ms_list):
    """p10, p50 and p90 of per-step durations given in ms, in µs (this rank)."""
    return [float(v) * 1e3 for v in np.percentile(np.asarray(ms_list, dtype=np.float64), [10, 50, 90])]


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings over the process group (every
    rank gets the result): the job is as slow as its slowest replica."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def run_ours(args, rank, world, local_rank):
    import torch
    from mla_latent_kv_33_b200 import mla
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS[args.workload]
    if w.dtype != "bf16":
        raise SystemExit("bench.py times the bf16 tensor-core workloads")
    x = synth.generate(w)
    W, cache_t, bt = upload(x, torch, dev)
    n_copies = cache_copies(cache_t.numel() * cache_t.element_size())
    caches = [mla.Cache(cache_t, bt)] + [mla.Cache(cache_t.clone(), bt) for _ in range(n_copies - 1)]
    p = mla.dims(w.d, w.n_h, w.d_h, w.d_c, w.d_cq, w.d_r, w.rope_base, 0.0, w.dtype)
    T = w.T
    HD = w.n_h * w.d_h
    if args.with_o_proj:  # W_O ~ N(0, 1/(n_h d_h)) from its own seed, rounded to bf16
        rng = np.random.Generator(np.random.PCG64(2000 + w.index))
        W_O = rng.standard_normal((w.d, HD), dtype=np.float32) * np.float32(1.0 / math.sqrt(HD))
        W["W_O"] = torch.from_numpy(synth.bf16_bits(W_O).view(np.int16)).view(torch.bfloat16).to(dev)
        if args.o_proj_absorbed:  # offline: W_OV = W_O blockdiag(W_UV_h), before any timing
            W["W_OV"] = torch.empty((w.d, w.n_h * w.d_c), device=dev, dtype=torch.bfloat16)
            mla.mla_absorb_wo(p, W["W_O"], W["W_UV"], W["W_OV"])
    if args.merged_absorb:  # offline: W_UQK_h = W_UK_h^T W_UQ_h, before any timing
        W["W_UQK"] = torch.empty((w.n_h * w.d_c, w.d_cq), device=dev, dtype=torch.bfloat16)
        mla.mla_absorb_merge(p, W["W_UQ"], W["W_UK"], W["W_UQK"])
    torch.cuda.synchronize()
    # two sets of the step's input and output buffers, so that the end-to-end
    # loop can copy the next step's inputs in while this step computes
    h_host = torch.from_numpy(x.h_bits.view(np.int16)).view(torch.bfloat16)
    bufs = [{"h": h_host.to(dev), "pos": torch.from_numpy(x.positions).to(dev),
             "sidx": torch.from_numpy(x.seq_idx).to(dev), "sl": torch.from_numpy(x.seq_lens).to(dev),
             "o": torch.empty((T, w.n_h * w.d_h), device=dev, dtype=torch.bfloat16),
             "y": torch.empty((T, w.d), device=dev, dtype=torch.bfloat16) if args.with_o_proj else None}
            for _ in range(2)]
    out_key = "y" if args.with_o_proj else "o"  # what a step hands back to the host
    o = bufs[0][out_key]
    q = torch.empty((T, w.n_h, w.D), device=dev, dtype=torch.bfloat16)
    qa = torch.empty((T, w.n_h, w.d_h + w.d_r), device=dev, dtype=torch.bfloat16) if args.order_a else None
    o_lat = torch.empty((T, w.n_h, w.d_c), device=dev, dtype=torch.bfloat16)
    lse = torch.empty((T, w.n_h), device=dev, dtype=torch.float32)
    ws = {op: torch.empty(max(1, mla.workspace_size(p, op, w.B if op == mla.OP_DECODE else T, w.n_q)),
                          dtype=torch.uint8, device=dev)
          for op in (mla.OP_APPEND, mla.OP_ABSORB, mla.OP_DECODE, mla.OP_OUT_PROJ, mla.OP_O_PROJ,
                     mla.OP_O_PROJ_LATENT, mla.OP_ABSORB_MERGED, mla.OP_FRONT_END)}
    if args.order_a:
        ws[mla.OP_QUERY_HEADS] = torch.empty(max(1, mla.workspace_size(p, mla.OP_QUERY_HEADS, T)), dtype=torch.uint8,
                                             device=dev)
        ws[mla.OP_ATTEND_A] = torch.empty(max(1, mla.workspace_size(p, mla.OP_ATTEND_A, w.B, w.n_q,
                                                                    mla.cache_rows(caches[0]))),
                                          dtype=torch.uint8, device=dev)
    ws[mla.OP_DECODE] = torch.empty(max(1, mla.workspace_size(p, mla.OP_DECODE, w.B, w.n_q, mla.cache_capacity(caches[0]),
                                                              args.num_splits)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)  # graph capture needs a non-default stream
    # the decode is bracketed by timing events in every `every`-th timed step
    # (about 20 of them); "external" makes them real event-record nodes when
    # the step is captured in a graph. An event pair costs a step ~10 µs (it
    # breaks the programmatic launch overlap between the kernels it separates),
    # so the other steps run without one.
    every = max(1, args.steps // 20)

    def sampled(i):
        return i is not None and i % every == 0

    ev_dec = [(torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True)) for _ in range(args.steps)]
    ev_op = [(torch.cuda.Event(enable_timing=True, external=True),
              torch.cuda.Event(enable_timing=True, external=True)) for _ in range(args.steps)]
    ev_front = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(args.steps)]
    ev_tail = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(args.steps)]

    # the cache append and the query absorption are independent: the append
    # runs on a side stream, joined before the decode reads the cache
    side = torch.cuda.Stream(device=dev)
    ev_fork, ev_join = torch.cuda.Event(), torch.cuda.Event()

    def step(i=None, b=0, c=None):
        x_ = bufs[b]
        if sampled(i) and args.breakdown:
            ev_front[i].record(stream)
        cache = caches[(i if c is None else c) % n_copies if (i is not None or c is not None) else 0]
        if args.order_a:
            ev_fork.record(stream)
            side.wait_event(ev_fork)
            mla.mla_cache_append(p, x_["h"], W["W_DKV"], W["W_KR"], x_["sidx"], x_["pos"], cache,
                                 ws=ws[mla.OP_APPEND], stream=side)
            ev_join.record(side)
            mla.mla_query_heads(p, x_["h"], W["W_DQ"], W["W_UQ"], W["W_QR"], x_["pos"], qa, ws=ws[mla.OP_QUERY_HEADS],
                                stream=stream)
            stream.wait_event(ev_join)
            if sampled(i):
                ev_dec[i][0].record(stream)
            mla.mla_attend_order_a(p, qa, W["W_UK"], W["W_UV"], cache, x_["sl"], w.n_q, x_["o"].view(T, w.n_h, w.d_h),
                                   ws=ws[mla.OP_ATTEND_A], stream=stream)
            if sampled(i):
                ev_dec[i][1].record(stream)
            return
        if args.fused_front_end:
            mla.mla_front_end(p, x_["h"], W["W_DKV"], W["W_KR"], W["W_DQ"], W["W_UQ"], W["W_QR"], W["W_UK"],
                              x_["sidx"], x_["pos"], cache, q, ws=ws[mla.OP_FRONT_END], stream=stream)
        else:
            ev_fork.record(stream)
            side.wait_event(ev_fork)
            mla.mla_cache_append(p, x_["h"], W["W_DKV"], W["W_KR"], x_["sidx"], x_["pos"], cache,
                                 ws=ws[mla.OP_APPEND], stream=side)
            ev_join.record(side)
            if args.merged_absorb:
                mla.mla_absorb_q_merged(p, x_["h"], W["W_DQ"], W["W_UQK"], W["W_QR"], x_["pos"], q,
                                        ws=ws[mla.OP_ABSORB_MERGED], stream=stream)
            else:
                mla.mla_absorb_q(p, x_["h"], W["W_DQ"], W["W_UQ"], W["W_QR"], W["W_UK"], x_["pos"], q,
                                 ws=ws[mla.OP_ABSORB], stream=stream)
            stream.wait_event(ev_join)
        if sampled(i):
            ev_dec[i][0].record(stream)
        mla.mla_decode(p, q, cache, x_["sl"], w.n_q, o_lat, lse, num_splits=args.num_splits, ws=ws[mla.OP_DECODE],
                       stream=stream)
        if sampled(i):
            ev_dec[i][1].record(stream)
        if not args.o_proj_absorbed:
            mla.mla_out_proj(p, o_lat, W["W_UV"], x_["o"], ws=ws[mla.OP_OUT_PROJ], stream=stream)
        if sampled(i) and args.breakdown:
            ev_tail[i].record(stream)
        if args.with_o_proj:
            if sampled(i):
                ev_op[i][0].record(stream)
            if args.o_proj_absorbed:
                mla.mla_o_proj_latent(p, o_lat, W["W_OV"], x_["y"], ws=ws[mla.OP_O_PROJ_LATENT], stream=stream)
            else:
                mla.mla_o_proj(p, x_["o"], W["W_O"], x_["y"], ws=ws[mla.OP_O_PROJ], stream=stream)
            if sampled(i):
                ev_op[i][1].record(stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    # launch overlap: each tensor-core kernel may be scheduled, set up and
    # start streaming its weights while the kernel ahead of it finishes
    mla.set_launch_overlap(not args.no_overlap)

    # One eager step first (one-time kernel attributes), then the same C-ABI
    # calls captured once into CUDA graphs: graph_1[b] holds one step on buffer
    # set b (warm-up and the end-to-end loop), graph_k the K timed steps.
    # Replays launch every kernel of the step with no host work between them.
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    graph_1 = graph_k = None
    launches_k = 0
    if not args.eager:
        graph_1 = {(b, c): torch.cuda.CUDAGraph() for b in range(2) for c in range(n_copies)}
        graph_k = torch.cuda.CUDAGraph()
        for (b, c), g in graph_1.items():
            with torch.cuda.graph(g, stream=stream):
                step(b=b, c=c)
        n0 = mla.kernel_launches()
        with torch.cuda.graph(graph_k, stream=stream):
            for i in range(args.steps):
                step(i)
        launches_k = mla.kernel_launches() - n0  # the kernels graph_k launches per replay
        torch.cuda.synchronize()

    def one_step(b=0, c=0):
        if graph_1 is not None:
            graph_1[(b, c % n_copies)].replay()
        else:
            step(b=b, c=c)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one_step()
    torch.cuda.synchronize()
    st = mla.mla_get_device_error(stream)
    if st != mla.MLA_OK:
        raise RuntimeError(f"device error after warm-up: {mla.status_string(st)}")

    # device-resident timing
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    launches0 = mla.kernel_launches()
    with ClockSampler(gpu_id_for_smi(torch, local_rank)) as clk, torch.cuda.stream(stream):
        h0 = time.perf_counter()
        t0.record(stream)
        if graph_k is not None:
            graph_k.replay()
        else:
            for i in range(args.steps):
                step(i)
        t1.record(stream)
        torch.cuda.synchronize()
        clk.mark(h0, time.perf_counter())
    launches = mla.kernel_launches() - launches0 + launches_k
    barrier()
    ms_total = t0.elapsed_time(t1)
    idx = [i for i in range(args.steps) if sampled(i)]
    dec_list = [ev_dec[i][0].elapsed_time(ev_dec[i][1]) for i in idx]
    dec_ms = float(np.mean(dec_list))
    dec_pct = percentiles_us(dec_list)
    op_ms = float(np.mean([ev_op[i][0].elapsed_time(ev_op[i][1]) for i in idx])) if args.with_o_proj else None
    breakdown = None
    if args.breakdown and not args.order_a:
        breakdown = {"front_us": float(np.mean([ev_front[i].elapsed_time(ev_dec[i][0]) for i in idx])) * 1e3,
                     "decode_us": dec_ms * 1e3,
                     "tail_us": float(np.mean([ev_dec[i][1].elapsed_time(ev_tail[i]) for i in idx])) * 1e3}

    # End to end through the public API: every step copies its inputs in from
    # pinned host memory and its output o back, inside the timed region. The
    # copies run on their own streams, double-buffered, so that step i + 1's
    # inputs arrive and step i - 1's output leaves while step i computes
    # (the way a serving loop overlaps them); e0/e1 bracket all of it.
    in_host = {"h": h_host.pin_memory(), "pos": torch.from_numpy(x.positions).pin_memory(),
               "sidx": torch.from_numpy(x.seq_idx).pin_memory(), "sl": torch.from_numpy(x.seq_lens).pin_memory()}
    o_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in in_host.values())
    d2h = o_host[0].numel() * o_host[0].element_size()
    h2d_stream, d2h_stream = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of set b landed
    ev_done = [torch.cuda.Event() for _ in range(2)]  # step on set b finished
    ev_out = [torch.cuda.Event() for _ in range(2)]   # o of set b copied out
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    h2d_stream.wait_event(e0)
    d2h_stream.wait_event(e0)
    for i in range(args.steps):
        b = i % 2
        with torch.cuda.stream(h2d_stream):
            if i >= 2:
                h2d_stream.wait_event(ev_done[b])  # step i - 2 no longer reads set b
            for k, t in in_host.items():
                bufs[b][k].copy_(t, non_blocking=True)
            ev_in[b].record(h2d_stream)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # o of step i - 2 has left set b
            one_step(b, i)
            ev_done[b].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(ev_done[b])
            o_host[b].copy_(bufs[b][out_key], non_blocking=True)
            ev_out[b].record(d2h_stream)
    stream.wait_stream(h2d_stream)
    stream.wait_stream(d2h_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    st = mla.mla_get_device_error(stream)
    if st != mla.MLA_OK:
        raise RuntimeError(f"device error during timing: {mla.status_string(st)}")

    step_ms = ms_total / args.steps
    if world > 1:
        step_ms, dec_ms, e2e_ms, op_ms = max_over_ranks([step_ms, dec_ms, e2e_ms, op_ms or 0.0], dev)
        op_ms = op_ms if args.with_o_proj else None
    del graph_1, graph_k
    return {"step_ms": step_ms, "dec_ms": dec_ms, "dec_pct": dec_pct, "e2e_ms": e2e_ms, "h2d": h2d, "d2h": d2h,
            "launch_mode": ("eager" if args.eager else "cuda_graph") + ("" if args.no_overlap else "+overlap"),
            "launches": launches, "clocks": clk.summary(), "x": x, "w": w, "op_ms": op_ms, "breakdown": breakdown, "n_copies": n_copies,
            "timed_calls": f"{len(idx)} of the {args.steps} timed steps (every {every}th) carry the event pair",
            "tc": mla.uses_tensor_cores(p, mla.OP_DECODE)}


# ------------------------------------------------------ oracle (CPU) arm --

def stratified_order(seq_lens):
    """Sequences ordered so that every prefix spans the length distribution:
    sorted by length, then taken alternately from the long and the short end
    of ever finer halvings (a prefix is a fair sample of the batch)."""
    idx = [int(b) for b in np.argsort(seq_lens, kind="stable")]
    out, parts = [], [idx]
    while parts:
        nxt = []
        for p_ in parts:
            if not p_:
                continue
            m = len(p_) // 2
            out.append(p_[m])
            nxt += [p_[:m], p_[m + 1:]]
        parts = nxt
    return out


def oracle_step(w, x, seqs):
    """One step of the fp64 oracle over the token rows of `seqs`: append of
    their new tokens, absorb, decode of all heads over the visible context,
    W_UV readout. Returns (seconds, attended tokens)."""
    import oracle as orc
    po = orc.dims(w.d, w.n_h, w.d_h, w.d_c, w.d_cq, w.d_r, w.rope_base)
    oc = orc.Cache(x.cache, x.block_table)
    rows = [b * w.n_q + j for b in seqs for j in range(w.n_q)]
    t0 = time.perf_counter()
    orc.append_rows(po, x.h[rows], x.weights["W_DKV"], x.weights["W_KR"], x.positions[rows])
    qb = orc.absorb_q(po, x.h[rows], x.weights["W_DQ"], x.weights["W_UQ"], x.weights["W_QR"],
                      x.weights["W_UK"], x.positions[rows])
    q = np.zeros((w.T, w.n_h, w.D))
    q[rows] = qb
    pairs = [(t, hh) for t in rows for hh in range(w.n_h)]
    o_lat, _ = orc.decode(po, q, oc, x.seq_lens, w.n_q, pairs=pairs)
    orc.out_proj(po, o_lat.reshape(len(rows), w.n_h, w.d_c), x.weights["W_UV"])
    seconds = time.perf_counter() - t0
    tokens = sum(int(x.seq_lens[b]) - w.n_q + 1 + j for b in seqs for j in range(w.n_q))
    return seconds, tokens


def oracle_sample(w, x, target_s):
    """Time the fp64 oracle on a bounded sample of the workload: whole steps
    over a growing, length-stratified set of sequences until about target_s of
    work, the whole batch when it fits. Returns (seconds per step, scaled to the
    whole batch by attended tokens when the sample is smaller, sample text,
    cores)."""
    import oracle as orc
    cores = len(os.sched_getaffinity(0))
    orc.set_threads(cores)
    work_total = synth.algorithmic_work(w, x.seq_lens)["tokens_attended"]
    order = stratified_order(x.seq_lens)
    seconds, tokens, n = 0.0, 0, 0
    chunk = max(1, len(order) // 16)
    while n < len(order) and (n == 0 or seconds < target_s):
        s, t = oracle_step(w, x, order[n:n + chunk])
        seconds, tokens, n = seconds + s, tokens + t, min(len(order), n + chunk)
    whole = n == len(order)
    per_step = seconds if whole else seconds * work_total / max(1, tokens)
    sample = (f"full step (append, absorb, decode over all {w.n_h} heads, W_UV readout) for {n} of {w.B} "
              f"sequences ({tokens} attended tokens of {work_total})"
              + ("; the whole batch, no scaling" if whole else
                 "; length-stratified sample, time scaled to the whole batch by attended tokens"))
    return per_step, sample, cores


def run_reference(args, rank, world):
    """The oracle arm: every timed step runs the fp64 oracle over the whole
    batch (all sequences, all heads), so that steps x ms_per_step is the time
    the arm really took. Warm-up steps run one sequence each (they only page
    the oracle and its inputs in)."""
    import oracle as orc
    w = synth.WORKLOADS[args.workload]
    x = synth.generate(w)
    cores = len(os.sched_getaffinity(0))
    orc.set_threads(cores)
    order = stratified_order(x.seq_lens)
    for _ in range(args.warmup):
        oracle_step(w, x, order[:1])
    per_step_s = [oracle_step(w, x, order)[0] for _ in range(args.steps)]
    us = float(np.mean(per_step_s) * 1e6)
    work = synth.algorithmic_work(w, x.seq_lens)
    sample = (f"whole batch every step: full step (append, absorb, decode over all {w.n_h} heads, W_UV readout) "
              f"for all {w.B} sequences ({work['tokens_attended']} attended tokens); warm-up steps: one sequence")
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": "µs/step", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args.gpus, x, None, args), "gpu_launches": 0,
        "cpu_baseline": {"value": us, "unit": "µs/step", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": us, "unit": "µs/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "cache_gbs": work["cache_bytes"] / (us * 1e-6) / 1e9,
    }
    print(json.dumps(line))


def step_text(args):
    if args is None:
        return "append + absorb + decode + W_UV readout"
    front = ("fused front end (append + absorb, h read once)" if args.fused_front_end else
             "append + " + ("merged-matrix absorb" if args.merged_absorb else "absorb"))
    tail = " + decode"
    if args.with_o_proj:
        tail += " + W_OV o_lat (W_UV absorbed into W_O)" if args.o_proj_absorbed else " + W_UV readout + W_O projection"
    else:
        tail += " + W_UV readout"
    return front + tail


def config_of(w, n, x, n_copies=None, args=None):
    L = x.seq_lens
    cache_bytes = int(x.cache.nbytes)
    if n_copies is None:
        n_copies = cache_copies(cache_bytes)
    l2 = ("no flush: the latent cache alone ({:.1f} MB) exceeds the 126 MB L2 (inputs larger than L2)".format(
        cache_bytes / 1e6) if n_copies == 1 else
        "the timed steps rotate through {} copies of the {:.1f} MB latent cache ({:.0f} MB > 2 x L2), so no step "
        "finds its cache in L2".format(n_copies, cache_bytes / 1e6, n_copies * cache_bytes / 1e6))
    return {"workload": w.name, "description": w.note, "batch": w.B, "n_q": w.n_q,
            "seq_len_min": int(L.min()), "seq_len_max": int(L.max()), "seq_len_mean": float(L.mean()),
            "paged": w.paged, "block_size": w.block_size if w.paged else None,
            "dims": {"d": w.d, "n_h": w.n_h, "d_h": w.d_h, "d_c": w.d_c, "d_cq": w.d_cq, "d_r": w.d_r},
            "parallelism": f"replicas{n}", "seed": 1000 + w.index, "l2": l2,
            "num_splits": 0 if args is None else args.num_splits,
            "step": step_text(args)}


def order_a_line(args, r, w, x, work, peaks, peak_kind, world):
    """Bench line of the order-A step. Its dominant call, mla_attend_order_a,
    is a dense contraction: the attention (n_h heads, 2 (d_h + d_r) + 2 d_h flops
    per query row and visible key) and the decompression of K_C and V for every
    physical cache row (2 x 2 d_h d_c flops per head and row); roofline = those
    flops at the measured bf16 tensor peak."""
    rows = int(np.prod(x.cache.shape[:2]))
    attn = 2 * w.n_h * work["tokens_attended"] * (w.d_h + w.d_r + w.d_h)
    decomp = 2 * 2 * w.n_h * w.d_h * w.d_c * rows
    flops = attn + decomp
    dec_s = r["dec_ms"] * 1e-3
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    return {
        "metric": METRIC, "value": r["step_ms"] * 1e3, "unit": "µs/step", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["step_ms"], "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**config_of(w, world, x, r["n_copies"], args),
                   "step": "append + per-head queries + order-A attention (decompress K/V, then 192-d attention)"},
        "attend_order_a_us": r["dec_ms"] * 1e3, "attend_us_p10_p50_p90": r["dec_pct"],
        "attend_timed_on": r["timed_calls"],
        "roofline": {"kernel": "mla_attend_order_a (decompression GEMMs + k_attend_a)", "bound": "tensor",
                     "achieved": flops / dec_s / 1e12, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": t_tc / dec_s, "traffic": None, "peak_source": peak_kind,
                     "algorithmic_flops": flops, "attention_flops": attn, "decompression_flops": decomp,
                     "roofline_us": t_tc * 1e6},
        "e2e": {"value": r["e2e_ms"] * 1e3, "unit": "µs/step", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"], "clocks": r["clocks"],
        "launch": "the step's C-ABI calls captured once into a CUDA graph, replayed",
    }


def o_proj_line(w, op_ms, peaks, absorbed):
    """Timing of the output projection against its weight-streaming roofline:
    W_O (d x n_h d_h) or, absorbed, W_OV (d x n_h d_c), bf16."""
    k = w.n_h * (w.d_c if absorbed else w.d_h)
    wb = w.d * k * 2
    return {"kernel": "mla_o_proj_latent (W_OV o_lat)" if absorbed else "mla_o_proj (W_O o)", "us": op_ms * 1e3,
            "weight_bytes": wb, "gbs": wb / (op_ms * 1e-3) / 1e9,
            "frac": (wb / (peaks["hbm_gbs"] * 1e9)) / (op_ms * 1e-3), "peak_gbs": peaks["hbm_gbs"]}


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        r = run_ours(args, rank, world, local_rank)
    finally:
        pass
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    w, x = r["w"], r["x"]
    work = synth.algorithmic_work(w, x.seq_lens)
    peaks, peak_kind = load_peaks()
    if args.order_a:
        print(json.dumps(order_a_line(args, r, w, x, work, peaks, peak_kind, world)))
        return
    us = r["step_ms"] * 1e3
    dec_s = r["dec_ms"] * 1e-3
    cache_gbs = work["cache_bytes"] / dec_s / 1e9
    tflops = work["flops"] / dec_s / 1e12
    t_hbm = work["cache_bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = work["flops"] / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    roof = {
        "kernel": "mla_decode (k_decode + k_combine)",
        "bound": bound,
        "achieved": cache_gbs if bound == "hbm" else tflops,
        "peak": peaks["hbm_gbs"] if bound == "hbm" else peaks["bf16_tflops"],
        "unit": "GB/s" if bound == "hbm" else "TFLOP/s",
        "frac": (t_hbm if bound == "hbm" else t_tc) / dec_s,
        "traffic": decode_traffic(w.name),
        "traffic_kernel": "k_decode (ncu dram__bytes_read.sum + dram__bytes_write.sum, one launch)",
        "peak_source": peak_kind,
        "algorithmic_bytes": work["cache_bytes"], "algorithmic_flops": work["flops"],
        "decode_us": r["dec_ms"] * 1e3,
        "roofline_us": max(t_hbm, t_tc) * 1e6,
    }
    line = {
        "metric": METRIC, "value": us, "unit": "µs/step", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["step_ms"], "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(w, world, x, r["n_copies"], args),
        "decode_us": r["dec_ms"] * 1e3, "decode_us_p10_p50_p90": r["dec_pct"], "decode_timed_on": r["timed_calls"],
        "cache_gbs": cache_gbs,
        "tflops": tflops,
        "tokens_per_s": world * w.T / (r["step_ms"] * 1e-3),
        "roofline": roof,
        "e2e": {"value": r["e2e_ms"] * 1e3, "unit": "µs/step", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
        **({"o_proj": o_proj_line(w, r["op_ms"], peaks, args.o_proj_absorbed)} if r["op_ms"] is not None else {}),
        **({"breakdown": r["breakdown"]} if r.get("breakdown") else {}),
        "tensor_core_decode": r["tc"],
        "clocks": r["clocks"],
    }
    if not args.no_cpu_baseline and world == 1:
        s, sample, cores = oracle_sample(w, x, args.cpu_sample_s)
        line["cpu_baseline"] = {"value": s * 1e6, "unit": "µs/step", "cores": cores, "kind": "oracle",
                                "sample": sample}
    line["launch"] = (
        ("eager C-ABI calls" if r["launch_mode"].startswith("eager") else
         "the step's four C-ABI calls captured once into a CUDA graph, replayed (timed: one graph of K steps; "
         "e2e: a one-step graph between the host copies)")
        + ("; launch overlap on (programmatic dependent launch)" if r["launch_mode"].endswith("+overlap") else ""))
    print(json.dumps(line))


if __name__ == "__main__":
    main()
