"""Benchmark of the TurboQuant hot path on B200 (one JSON line on rank 0).

Workload (default): one layer of a Llama-3.1-8B-shaped KV cache at 32768 tokens --
batch 1, 32 query heads / 8 KV heads (GQA 4), head_dim 128, bf16 K/V N(0,1) with 4
outlier channels per head scaled x8.  One step = quantize the whole cache (keys:
3-bit MSE + 1-bit QJL, values: 4-bit MSE), then fused logits -> softmax -> V for one new
token.  value = keys scored per second over whole steps (all ranks).

Timing: W warm-up steps, then K timed steps; before every step a 256 MiB buffer is
written to flush the 126 MB L2; each step is bracketed by CUDA events on the stream the
kernels run on; ranks are synchronised by a barrier and the max over ranks is taken.
Multi-GPU (torchrun): every rank runs its own independent copy of the workload (the
path shards over independent caches with no data-path collective): weak scaling.

--impl reference runs the float64 CPU oracle (the method's plain definition) on a
bounded sample of the same workload and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "keys scored/s and decode-attn HBM GB/s (% of 8 TB/s); quantize vectors/s"
NOMINAL_HBM_GBS = 8000.0


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sus=p["bf16_tflops_sustained"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x, ws, device=None):
    """The largest value of a per-rank float over all ranks (a job takes as long as its
    slowest rank).  Every rank must call it, in the same order as the other collectives."""
    if ws <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, ws, seconds):
    """Units processed by all ranks per second of the slowest rank's time."""
    return units_per_rank * ws / seconds


# ------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = [l.strip().split(",") for l in open(self.path) if l.strip()]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except (ValueError, IndexError):
                continue
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------- GPU workload
class DecodeBench:
    """Device-resident state of one decode workload (quantize cache + one decode step)."""

    def __init__(self, w: W.DecodeWorkload, device, seed: int = 0):
        import torch
        import kv_cache_vector_08_b200 as tq
        self.tq, self.torch, self.w, self.dev = tq, torch, w, device
        B, Hkv, Hq, D, T = w.batch, w.kv_heads, w.q_heads, w.head_dim, w.context
        self.B, self.Hkv, self.Hq, self.D, self.T = B, Hkv, Hq, D, T
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        # K/V bf16 [B, Hkv, T, D] generated on the device (same distribution as workloads.decode_kv)
        k = torch.randn((B, Hkv, T, D), generator=g, device=device, dtype=torch.float32)
        v = torch.randn((B, Hkv, T, D), generator=g, device=device, dtype=torch.float32)
        if w.outliers:
            for x, stream in ((k, W.STREAM_KEY_OUTLIERS), (v, W.STREAM_VALUE_OUTLIERS)):
                ch = W.outlier_channels(Hkv, D, w.outliers, seed, stream)
                for h in range(Hkv):
                    x[:, h, :, torch.tensor(ch[h], device=device)] *= w.outlier_factor
        if w.lognormal_sigma:
            k *= torch.exp(torch.randn((B, 1, T, 1), generator=g, device=device) * w.lognormal_sigma)
            v *= torch.exp(torch.randn((B, 1, T, 1), generator=g, device=device) * w.lognormal_sigma)
        self.K = k.to(torch.bfloat16).reshape(-1, D)
        self.V = v.to(torch.bfloat16).reshape(-1, D)
        del k, v
        self.q = torch.randn((B, Hq, D), generator=g, device=device).to(torch.bfloat16)
        self.kctx, self.vctx, self.kc, self.vc, self.off = [], [], [], [], []
        for gi, (off, wd, kb, vb) in enumerate(w.groups):
            kx = tq.Context(wd, kb, 1000 + 2 * gi, tq.MODE_PROD)
            vx = tq.Context(wd, vb, 1001 + 2 * gi, tq.MODE_MSE)
            self.kctx.append(kx)
            self.vctx.append(vx)
            self.kc.append(tq.alloc_packed(kx, B * Hkv * T, device))
            self.vc.append(tq.alloc_packed(vx, B * Hkv * T, device))
            self.off.append(off)
        self.off.append(D)
        self.seq = torch.full((B,), T, dtype=torch.int32, device=device)
        self.out = torch.empty((B, Hq, D), dtype=torch.float32, device=device)
        self.plan = tq.DecodePlan(self.kctx, self.vctx, self.off, self.kc, self.vc, B, Hq, Hkv, D, T, device=device)
        self.scale = 1.0 / math.sqrt(D)
        self.flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
        self.vectors = B * Hkv * T            # per K (and per V) quantize
        self.keys = B * Hkv * T               # token-heads scored per decode step

    # algorithmic bytes
    def quantize_bytes(self):
        kb = vb = 0
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            kb += wd * 2 + self.kctx[gi].code_bytes * wd // self.kctx[gi].d_pad + 4
            vb += wd * 2 + self.vctx[gi].code_bytes * wd // self.vctx[gi].d_pad + 2
        return kb * self.vectors, vb * self.vectors

    def quantize_flops(self):
        """Algorithmic flops of the fp32-accurate projections: keys 2d^2 (Pi x) + 2d^2 (S r)
        per vector and group, values 2d^2."""
        kf = vf = 0
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            kf += 4 * wd * wd
            vf += 2 * wd * wd
        return kf * self.vectors, vf * self.vectors

    def decode_bytes(self):
        per = 0
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            per += (self.kctx[gi].code_bytes * wd // self.kctx[gi].d_pad + 4)
            per += (self.vctx[gi].code_bytes * wd // self.vctx[gi].d_pad + 2)
        return per * self.keys

    def quantize_keys(self, stream=None):
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            self.tq.quantize_kv(self.kctx[gi], self.K[:, off:off + wd], self.kc[gi], stream=stream)

    def quantize_values(self, stream=None):
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            self.tq.quantize_kv(self.vctx[gi], self.V[:, off:off + wd], self.vc[gi], stream=stream)

    def quantize(self, stream=None):
        self.quantize_keys(stream)
        self.quantize_values(stream)

    def decode(self, stream=None):
        self.plan(self.q, self.seq, self.scale, self.out, stream=stream)

    def flush_l2(self, stream):
        with self.torch.cuda.stream(stream):
            self.flush.fill_(1.0)

    def capture(self, fn):
        """CUDA graph of one library call sequence (replayed in the timed loop, so the
        timing sees device time rather than Python/ctypes launch overhead)."""
        torch = self.torch
        s = torch.cuda.Stream(device=self.dev)
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(2):
                fn()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g


def run_gpu(args):
    import torch
    ws, rank, local = _dist()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import kv_cache_vector_08_b200 as tq
    w = W.LLAMA_DECODE
    bench = DecodeBench(w, dev)
    st = torch.cuda.current_stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    gK = bench.capture(bench.quantize_keys)
    gV = bench.capture(bench.quantize_values)
    gD = bench.capture(bench.decode)
    per_step_launches = 0
    n0 = tq.launch_count()
    bench.quantize()
    bench.decode()
    torch.cuda.synchronize()
    per_step_launches = tq.launch_count() - n0

    def step(record):
        bench.flush_l2(st)
        e0, e1, e2, e3 = ev(), ev(), ev(), ev()
        e0.record(st)
        gK.replay()
        e1.record(st)
        gV.replay()
        e2.record(st)
        gD.replay()
        e3.record(st)
        record.append((e0, e1, e2, e3))

    for _ in range(args.warmup):
        step([])
    torch.cuda.synchronize()
    recs = []
    barrier = (lambda: torch.distributed.barrier()) if ws > 1 else (lambda: None)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        for _ in range(args.steps):
            step(recs)
        torch.cuda.synchronize()
        barrier()
    launches = per_step_launches * args.steps
    clocks = clk.summary()
    t_step = np.array([a.elapsed_time(d) for a, b, c, d in recs]) / 1e3
    t_qk = np.array([a.elapsed_time(b) for a, b, c, d in recs]) / 1e3
    t_qv = np.array([b.elapsed_time(c) for a, b, c, d in recs]) / 1e3
    t_dec = np.array([c.elapsed_time(d) for a, b, c, d in recs]) / 1e3
    ms_step = max_over_ranks(float(t_step.mean() * 1e3), ws, dev)

    # decode alone, L2 flushed before every launch (the HBM GB/s figure)
    dec = []
    for _ in range(max(args.steps, 20)):
        bench.flush_l2(st)
        a, b = ev(), ev()
        a.record(st)
        gD.replay()
        b.record(st)
        dec.append((a, b))
    torch.cuda.synchronize()
    t_dec_alone = float(np.median([a.elapsed_time(b) for a, b in dec]) / 1e3)

    # end to end through the public API from pinned host buffers (whole job: all ranks'
    # keys over the slowest rank's time)
    e2e = run_e2e(bench, st, args.steps, args.warmup)
    e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], ws, dev)
    e2e["value"] = whole_job_rate(bench.keys, ws, e2e["ms_per_step"] / 1e3)

    if rank != 0:
        if ws > 1:
            torch.distributed.destroy_process_group()
        return
    peaks = _peaks()
    qk_bytes, qv_bytes = bench.quantize_bytes()
    dec_bytes = bench.decode_bytes()
    value = whole_job_rate(bench.keys, ws, ms_step / 1e3)
    kernels = {"quantize_keys": float(t_qk.mean()), "quantize_values": float(t_qv.mean()),
               "decode_attention": float(t_dec.mean())}
    dominant = max(kernels, key=kernels.get)
    # roofline of each kernel: HBM (algorithmic bytes at the measured copy bandwidth) and,
    # for the quantizer, the tensor pipe: an fp32-accurate product costs three bf16 passes
    # (Pi in three bf16 splits; the QJL product as three fp16 hi/lo products), so its peak
    # is the measured bf16 GEMM peak / 3.  The binding roofline is the slower floor.
    qk_flops, qv_flops = bench.quantize_flops()
    fp32acc_peak = peaks["bf16"] / 3.0
    bytes_of = {"quantize_keys": qk_bytes, "quantize_values": qv_bytes, "decode_attention": dec_bytes}
    flops_of = {"quantize_keys": qk_flops, "quantize_values": qv_flops, "decode_attention": 0}

    def roof(kname):
        t = kernels[kname]
        hbm_floor = bytes_of[kname] / (peaks["hbm"] * 1e9)
        ten_floor = flops_of[kname] / (fp32acc_peak * 1e12)
        if ten_floor > hbm_floor:
            a = flops_of[kname] / t / 1e12
            return {"kernel": kname, "bound": "tensor", "achieved": a, "peak": fp32acc_peak, "unit": "TFLOP/s",
                    "frac": a / fp32acc_peak, "floor_us": ten_floor * 1e6, "hbm_floor_us": hbm_floor * 1e6,
                    "peak_source": "measured bf16 dense burst %.0f TFLOP/s / 3 (three split passes per "
                                   "fp32-accurate product)" % peaks["bf16"]}
        a = bytes_of[kname] / t / 1e9
        return {"kernel": kname, "bound": "hbm", "achieved": a, "peak": peaks["hbm"], "unit": "GB/s",
                "frac": a / peaks["hbm"], "floor_us": hbm_floor * 1e6,
                "peak_source": "measured hbm_gbs" if peaks["src"] == "measured" else "fallback 6650 GB/s"}
    line = {
        "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
                   "head_dim": w.head_dim, "context": w.context, "key_bits": 4, "value_bits": 4,
                   "step": "quantize K+V cache, then decode attention for 1 token",
                   "l2": "flushed (256 MiB write) before every step", "parallelism": "replicas%d" % ws},
        "components": {
            "quantize_vectors_per_s": 2 * bench.vectors / (kernels["quantize_keys"] + kernels["quantize_values"]),
            "quantize_keys_us": kernels["quantize_keys"] * 1e6,
            "quantize_values_us": kernels["quantize_values"] * 1e6,
            "decode_us_in_step": kernels["decode_attention"] * 1e6,
            "decode_us_l2_flushed": t_dec_alone * 1e6,
            "decode_keys_scored_per_s": bench.keys / t_dec_alone,
            "decode_hbm_gbs": dec_bytes / t_dec_alone / 1e9,
            "decode_frac_of_8tbs": dec_bytes / t_dec_alone / 1e9 / NOMINAL_HBM_GBS,
        },
        "timing": "device time of CUDA-graph replays of the library calls (captured once), L2 flushed before each step",
        "roofline": dict(roof(dominant), traffic=recorded_traffic(dominant)),
        "roofline_quantize_values": roof("quantize_values"),
        "roofline_decode": {"bound": "hbm", "achieved": dec_bytes / t_dec_alone / 1e9, "peak": peaks["hbm"],
                            "unit": "GB/s", "frac": dec_bytes / t_dec_alone / 1e9 / peaks["hbm"],
                            "bytes_per_launch": dec_bytes, "traffic": recorded_traffic("decode_attention")},
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    line["rows"] = measure_rows(bench, peaks)
    line["cpu_baseline"] = cpu_baseline(w, w.kv_heads)
    print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------- the other path rows
def _time_device(fn, flush, reps):
    """Median device time (s) of fn() over reps, L2 flushed before every rep."""
    import torch
    st = torch.cuda.current_stream()
    fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush(st)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        fn()
        b.record(st)
        b.synchronize()
        ts.append(a.elapsed_time(b) / 1e3)
    return float(np.median(ts))


def recorded_traffic(kernel):
    """DRAM bytes per launch from the committed ncu record (profiles/), or None when the
    kernel's source has changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic_llama_32k.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(kernel)
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != rec["sha256"]:
        return None
    return rec["bytes_per_launch"]


def fp32_fma_peak_tflops():
    """CUDA-core fp32 peak from unit counts and clocks: 148 SMs x 128 FMA lanes x 2 flop x
    the maximum SM clock (1965 MHz)."""
    return 148 * 128 * 2 * 1.965e9 / 1e12


def measure_rows(bench, peaks, reps=5):
    """Time the hot-path rows that the decode step does not call (standalone logits,
    dequantize, index + search) on bounded synthetic workloads, each against its roofline.
    Runs after the timed step; not part of the step time."""
    import torch
    tq, dev = bench.tq, bench.dev
    out = {}
    flush = bench.flush_l2

    def entry(t, bound, work, peak, unit, extra):
        a = work / t / (1e9 if unit == "GB/s" else 1e12)
        return dict(extra, us=t * 1e6, bound=bound, achieved=a, peak=peak, unit=unit, frac=a / peak)

    # standalone logits of 4 queries against all 262,144 cached keys of the layer
    kctx, kc = bench.kctx[0], bench.kc[0]
    n = bench.vectors
    q4 = torch.randn((4, bench.D), device=dev, generator=torch.Generator(device=dev).manual_seed(11))
    lg = torch.empty((4, n), dtype=torch.float32, device=dev)
    ws = torch.empty(max(int(tq.lib().tq_attn_logits_workspace_size(kctx.handle, 4)), 1), dtype=torch.uint8,
                     device=dev)
    t = _time_device(lambda: tq.attn_logits(kctx, q4, kc, n, out=lg, workspace=ws), flush, reps)
    nbytes = n * (kctx.code_bytes + 4) + 4 * n * 4
    out["logits"] = entry(t, "hbm", nbytes, peaks["hbm"], "GB/s",
                          {"work": "4 queries x 262144 keys (d=128, 4-bit prod)", "bytes": nbytes})
    # dequantize the 262,144 value vectors of the layer (x = ||x|| Pi^T c[idx])
    vctx, vc = bench.vctx[0], bench.vc[0]
    xo = torch.empty((n, bench.D), dtype=torch.float32, device=dev)
    t = _time_device(lambda: tq.dequantize(vctx, vc, n, out=xo), flush, reps)
    flops = 2.0 * bench.D * bench.D * n
    out["dequantize"] = entry(t, "alu", flops, fp32_fma_peak_tflops(), "TFLOP/s",
                              {"work": "262144 value vectors (d=128, 4-bit MSE)", "flops": flops,
                               "hbm_floor_us": (n * (vctx.code_bytes + 2) + n * bench.D * 4) / peaks["hbm"] / 1e3,
                               "peak_source": "fp32 FMA lanes x clock (148 x 128 x 2 x 1.965 GHz)"})
    # index + top-10 search at d = 1536 (200,000 database rows, 1000 queries) and
    # d = 200 (1,000,000 rows, 1000 queries); unit-norm Gaussian vectors
    for d, ndb in ((1536, 200_000), (200, 1_000_000)):
        g = torch.Generator(device=dev).manual_seed(7)
        db = torch.nn.functional.normalize(torch.randn((ndb, d), generator=g, device=dev), dim=1)
        qs = torch.nn.functional.normalize(torch.randn((1000, d), generator=g, device=dev), dim=1)
        ctx = tq.Context(d, 4, 12, tq.MODE_PROD)
        pk = tq.alloc_packed(ctx, ndb, dev)
        t_idx = _time_device(lambda: tq.quantize_kv(ctx, db, pk), flush, 2)
        t_s = _time_device(lambda: tq.search_topk(ctx, qs, pk, ndb, 10), flush, 2)
        fl = 4.0 * d * 1000 * ndb
        out["search_d%d" % d] = entry(t_s, "tensor", fl, peaks["bf16"], "TFLOP/s",
                                      {"work": "1000 queries x %d rows, top-10" % ndb, "flops": fl,
                                       "index_us": t_idx * 1e6,
                                       "index_vectors_per_s": ndb / t_idx,
                                       "peak_source": "measured bf16 dense burst"})
        del db, qs, pk, ctx
    return out


def run_e2e(bench, st, steps, warmup):
    """Same step through the public API with host (pinned) inputs: H2D of K, V and q,
    quantize + decode, D2H of the attention output, all inside the timed region."""
    import torch
    Kh = torch.empty(bench.K.shape, dtype=bench.K.dtype, pin_memory=True)
    Vh = torch.empty(bench.V.shape, dtype=bench.V.dtype, pin_memory=True)
    qh = torch.empty(bench.q.shape, dtype=bench.q.dtype, pin_memory=True)
    Kh.copy_(bench.K)
    Vh.copy_(bench.V)
    qh.copy_(bench.q)
    oh = torch.empty(bench.out.shape, dtype=bench.out.dtype, pin_memory=True)
    times = []
    for i in range(warmup + steps):
        bench.flush_l2(st)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        bench.K.copy_(Kh, non_blocking=True)
        bench.V.copy_(Vh, non_blocking=True)
        bench.q.copy_(qh, non_blocking=True)
        bench.quantize()
        bench.decode()
        oh.copy_(bench.out, non_blocking=True)
        b.record(st)
        if i >= warmup:
            times.append((a, b))
    torch.cuda.synchronize()
    t = float(np.mean([a.elapsed_time(b) for a, b in times]) / 1e3)
    h2d = Kh.numel() * Kh.element_size() + Vh.numel() * Vh.element_size() + qh.numel() * qh.element_size()
    return {"value": bench.keys / t, "unit": "keys/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(oh.numel() * oh.element_size()), "ms_per_step": t * 1e3}


# -------------------------------------------------------------------- CPU oracle
def oracle_sample_step(w: W.DecodeWorkload, heads: int, seed: int = 0):
    """The oracle on a bounded sample of the workload: `heads` KV heads of sequence 0 at
    the full context (quantize their K and V rows, then decode their query heads).
    Returns the number of keys scored."""
    import oracle
    D, T = w.head_dim, w.context
    rep = w.q_heads // w.kv_heads
    kp = [oracle.make_params(wd, kb, 1000 + 2 * gi, 0) for gi, (off, wd, kb, vb) in enumerate(w.groups)] \
        if not hasattr(oracle_sample_step, "params") else oracle_sample_step.params[0]
    vp = [oracle.make_params(wd, vb, 1001 + 2 * gi, 1) for gi, (off, wd, kb, vb) in enumerate(w.groups)] \
        if not hasattr(oracle_sample_step, "params") else oracle_sample_step.params[1]
    oracle_sample_step.params = (kp, vp)
    if not hasattr(oracle_sample_step, "data"):
        g = W.generator(seed, 99)
        K = W.round_bf16(g.standard_normal((1, heads, T, D)))
        V = W.round_bf16(g.standard_normal((1, heads, T, D)))
        q = W.round_bf16(g.standard_normal((1, heads * rep, D)))
        oracle_sample_step.data = (K, V, q)
    K, V, q = oracle_sample_step.data
    offs = [g[0] for g in w.groups] + [D]
    kcodes, vcodes = [], []
    for gi, (off, wd, kb, vb) in enumerate(w.groups):
        ko = oracle.quantize(kp[gi], K[..., off:off + wd].reshape(-1, wd).astype(np.float64))
        vo = oracle.quantize(vp[gi], V[..., off:off + wd].reshape(-1, wd).astype(np.float64))
        kcodes.append(dict(idx=ko["idx"].reshape(1, heads, T, wd), signs=ko["signs"].reshape(1, heads, T, wd),
                           norm=ko["norm"].reshape(1, heads, T), rnorm=ko["rnorm"].reshape(1, heads, T)))
        vcodes.append(dict(idx=vo["idx"].reshape(1, heads, T, wd), norm=vo["norm"].reshape(1, heads, T)))
    oracle.decode_attention(kp, vp, offs, q.astype(np.float64), kcodes, vcodes, [T], 1.0 / math.sqrt(D))
    return heads * T


def cpu_baseline(w, heads: int):
    import oracle  # noqa: F401  (the baseline times the oracle as it stands)
    oracle_sample_step(w, heads)     # parameters and data outside the timing
    t0 = time.perf_counter()
    keys = oracle_sample_step(w, heads)
    dt = time.perf_counter() - t0
    return {"value": keys / dt, "unit": "keys/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": "%d of %d KV heads at the full %d-token context: quantize their K and V rows "
                      "(float64) and decode their %d query heads; %.1f s" % (
                          heads, w.kv_heads, w.context, heads * (w.q_heads // w.kv_heads), dt)}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    w = W.LLAMA_DECODE
    oracle_sample_step(w, args.cpu_sample_heads)
    for _ in range(args.warmup):
        oracle_sample_step(w, args.cpu_sample_heads)
    ts = []
    keys = 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        keys = oracle_sample_step(w, args.cpu_sample_heads)
        ts.append(time.perf_counter() - t0)
    t = float(np.mean(ts))
    value = keys / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
                   "head_dim": w.head_dim, "context": w.context, "key_bits": 4, "value_bits": 4,
                   "step": "quantize K+V cache, then decode attention for 1 token",
                   "sample": "%d of %d KV heads" % (args.cpu_sample_heads, w.kv_heads)},
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": "%d of %d KV heads at the full context per step" % (args.cpu_sample_heads, w.kv_heads)},
        "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--cpu-sample-heads", type=int, default=2,
                    help="KV heads per oracle step in --impl reference")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
