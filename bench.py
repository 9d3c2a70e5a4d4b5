"""Benchmark of the TurboQuant hot path on B200 (one JSON line on rank 0).

Headline workload (default, ``--config serving``): serving decode at 3.5 bits per channel
-- batch 64, 32 query heads / 8 KV heads (GQA 4), head_dim 128, 8192-token contexts, bf16
K/V Gaussian with per-token log-normal(0, 0.5) norms; channels [0, 64) at 4 bits and
[64, 128) at 3 bits, each group with its own Pi, S and codebook.  One step = append-
quantize one new token per sequence (64 x 8 = 512 key and 512 value vectors per group)
and decode attention for one new query token over the 4,194,304 cached token-heads.
value = keys scored per second over whole steps (all ranks).

``--config llama`` (one Llama-3.1-8B-shaped layer at 32K: quantize the whole K/V cache,
then decode) and ``--config long`` (131072-token context at 2.5 bits: one append + decode
per step) select the other decode workloads as the headline.  Unless ``--no-configs`` is
given, the run also measures every other workload after the timed region (not part of the
step time) and reports it under "configs": the other decode workloads, the long-context
prefill quantize, the toy parity workload, vector search (index + top-10 search + 1@10
recall at d = 1536 and d = 200 over 10^6 rows), standalone logits and dequantize.

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
import hashlib
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
DECODE_CONFIGS = {"serving": W.SERVING_3P5, "llama": W.LLAMA_DECODE, "long": W.LONG_2P5}


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


# ----------------------------------------------------------------- roofline helpers
def hbm_roof(nbytes, seconds, peaks, kernel, **extra):
    a = nbytes / seconds / 1e9
    return dict(kernel=kernel, bound="hbm", achieved=a, peak=peaks["hbm"], unit="GB/s", frac=a / peaks["hbm"],
                bytes_per_launch=int(nbytes), us=seconds * 1e6,
                peak_source="measured copy bandwidth (MEASURED_PEAKS.json hbm_gbs)" if peaks["src"] == "measured"
                else "fallback 6650 GB/s", **extra)


def tensor_roof(flops, seconds, peak_tflops, kernel, peak_source, **extra):
    a = flops / seconds / 1e12
    return dict(kernel=kernel, bound="tensor", achieved=a, peak=peak_tflops, unit="TFLOP/s", frac=a / peak_tflops,
                flops_per_launch=float(flops), us=seconds * 1e6, peak_source=peak_source, **extra)


def recorded_traffic(workload, kernel):
    """DRAM bytes per launch from the committed ncu record (profiles/dram_traffic.json), or
    None when the record is missing or the kernel's source has changed since the counters
    were taken."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get("%s/%s" % (workload, kernel))
    if not rec:
        return None
    for src_rel, sha in rec["sources"].items():
        src = os.path.join(ROOT, src_rel)
        if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != sha:
            return None
    return rec["bytes_per_launch"]


# ------------------------------------------------------------------- GPU workload
class DecodeBench:
    """Device-resident state of one decode workload: the bf16 K/V rows, the packed caches
    (one key and one value context per channel group) and the decode plan."""

    def __init__(self, w: W.DecodeWorkload, device, seed: int = 0, extra_tokens: int = 0):
        import torch
        import kv_cache_vector_08_b200 as tq
        self.tq, self.torch, self.w, self.dev = tq, torch, w, device
        B, Hkv, Hq, D, T = w.batch, w.kv_heads, w.q_heads, w.head_dim, w.context
        self.B, self.Hkv, self.Hq, self.D, self.T = B, Hkv, Hq, D, T
        self.max_len = T + extra_tokens
        L = self.max_len
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        # K/V bf16 [B, Hkv, L, D] generated on the device (same distribution as workloads.decode_kv)
        K = torch.empty((B, Hkv, L, D), dtype=torch.bfloat16, device=device)
        V = torch.empty((B, Hkv, L, D), dtype=torch.bfloat16, device=device)
        for dst, stream, sstream in ((K, W.STREAM_KEY_OUTLIERS, 0), (V, W.STREAM_VALUE_OUTLIERS, 1)):
            for b in range(B):
                x = torch.randn((Hkv, L, D), generator=g, device=device)
                if w.outliers:
                    ch = W.outlier_channels(Hkv, D, w.outliers, seed, stream)
                    for h in range(Hkv):
                        x[h, :, torch.tensor(ch[h], device=device)] *= w.outlier_factor
                if w.lognormal_sigma:
                    x *= torch.exp(torch.randn((1, L, 1), generator=g, device=device) * w.lognormal_sigma)
                dst[b] = x.to(torch.bfloat16)
                del x
        self.K, self.V = K, V
        self.Kf, self.Vf = K.reshape(-1, D), V.reshape(-1, D)
        self.q = torch.randn((B, Hq, D), generator=g, device=device).to(torch.bfloat16)
        self.kctx, self.vctx, self.kc, self.vc, self.off = [], [], [], [], []
        for gi, (off, wd, kb, vb) in enumerate(w.groups):
            kx = tq.Context(wd, kb, 1000 + 2 * gi, tq.MODE_PROD)
            vx = tq.Context(wd, vb, 1001 + 2 * gi, tq.MODE_MSE)
            self.kctx.append(kx)
            self.vctx.append(vx)
            self.kc.append(tq.alloc_packed(kx, B * Hkv * L, device))
            self.vc.append(tq.alloc_packed(vx, B * Hkv * L, device))
            self.off.append(off)
        self.off.append(D)
        self.out = torch.empty((B, Hq, D), dtype=torch.float32, device=device)
        self.plan = tq.DecodePlan(self.kctx, self.vctx, self.off, self.kc, self.vc, B, Hq, Hkv, D, L, device=device)
        self.scale = 1.0 / math.sqrt(D)
        self.flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
        # append state: per position t, the slots of token t of every (sequence, kv head),
        # the rows of K/V holding it, and the sequence lengths after the append
        bh = torch.arange(B * Hkv, device=device, dtype=torch.int64)
        self.app_slots, self.app_rows, self.app_seq = {}, {}, {}
        for t in range(T - 1, L):
            self.app_slots[t] = (bh * L + t).contiguous()
            self.app_rows[t] = (bh * L + t).contiguous()
            self.app_seq[t] = torch.full((B,), t + 1, dtype=torch.int32, device=device)
        self.app_k = {t: self.Kf[self.app_rows[t]].contiguous() for t in self.app_rows}
        self.app_v = {t: self.Vf[self.app_rows[t]].contiguous() for t in self.app_rows}

    # ----- algorithmic bytes / flops (SURVEY-style counts: input + codes, or codes read)
    def rec_bytes(self, gi, keys):
        ctx = self.kctx[gi] if keys else self.vctx[gi]
        wd = self.w.groups[gi][1]
        return ctx.code_bytes * wd // ctx.d_pad + (4 if keys else 2)

    def quantize_bytes(self, n):
        kb = sum(wd * 2 + self.rec_bytes(gi, True) for gi, (_, wd, _, _) in enumerate(self.w.groups))
        vb = sum(wd * 2 + self.rec_bytes(gi, False) for gi, (_, wd, _, _) in enumerate(self.w.groups))
        return kb * n, vb * n

    def quantize_flops(self, n):
        """Algorithmic flops: keys 2d^2 (Pi x) + 2d^2 (S r) per vector and group, values 2d^2."""
        kf = sum(4 * wd * wd for (_, wd, _, _) in self.w.groups)
        vf = sum(2 * wd * wd for (_, wd, _, _) in self.w.groups)
        return kf * n, vf * n

    def token_head_bytes(self):
        return sum(self.rec_bytes(gi, True) + self.rec_bytes(gi, False) for gi in range(len(self.w.groups)))

    # ----- library calls
    def prefill(self, T, stream=None):
        """Quantize tokens [0, T) of every (sequence, kv head) into the caches."""
        L = self.max_len
        if T == L:
            for gi, (off, wd, _, _) in enumerate(self.w.groups):
                self.tq.quantize_kv(self.kctx[gi], self.Kf[:, off:off + wd], self.kc[gi], stream=stream)
                self.tq.quantize_kv(self.vctx[gi], self.Vf[:, off:off + wd], self.vc[gi], stream=stream)
            return
        torch = self.torch
        rows = (torch.arange(self.B * self.Hkv, device=self.dev).view(-1, 1) * L
                + torch.arange(T, device=self.dev).view(1, -1)).reshape(-1)
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            self.tq.quantize_kv(self.kctx[gi], self.Kf[rows, off:off + wd], self.kc[gi], slots=rows, stream=stream)
            self.tq.quantize_kv(self.vctx[gi], self.Vf[rows, off:off + wd], self.vc[gi], slots=rows, stream=stream)

    def quantize_all_keys(self, stream=None):
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            self.tq.quantize_kv(self.kctx[gi], self.Kf[:, off:off + wd], self.kc[gi], stream=stream)

    def quantize_all_values(self, stream=None):
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            self.tq.quantize_kv(self.vctx[gi], self.Vf[:, off:off + wd], self.vc[gi], stream=stream)

    def append(self, t, stream=None, k=None, v=None):
        """Quantize token t of every (sequence, kv head) into its cache slot.  The key and
        value calls of every group are independent, so they run on parallel streams (forked
        from and joined back into the calling stream; parallel branches inside a graph)."""
        torch = self.torch
        k = self.app_k[t] if k is None else k
        v = self.app_v[t] if v is None else v
        jobs = []
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            jobs.append((self.kctx[gi], k[:, off:off + wd], self.kc[gi]))
            jobs.append((self.vctx[gi], v[:, off:off + wd], self.vc[gi]))
        cur = torch.cuda.current_stream(self.dev) if stream is None else stream
        if not hasattr(self, "side"):
            self.side = [torch.cuda.Stream(device=self.dev) for _ in range(3)]
        streams = [cur] + self.side[:len(jobs) - 1]
        for s in streams[1:]:
            s.wait_stream(cur)
        for s, (ctx, x, dst) in zip(streams, jobs):
            self.tq.quantize_kv(ctx, x, dst, slots=self.app_slots[t], stream=s)
        for s in streams[1:]:
            cur.wait_stream(s)

    def decode(self, seq, stream=None):
        self.plan(self.q, seq, self.scale, self.out, stream=stream)

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

    def free(self):
        for name in ("K", "V", "Kf", "Vf", "kc", "vc", "plan", "flush", "app_k", "app_v"):
            if hasattr(self, name):
                delattr(self, name)


class StepRunner:
    """A decode workload's step as a list of named CUDA-graph phases; each timed step
    flushes L2, then replays the phases with an event between every two."""

    def __init__(self, bench, phases):
        self.bench = bench
        self.names = [n for n, _ in phases]
        self.graphs = [bench.capture(fn) for _, fn in phases]

    def run(self, st, record):
        torch = self.bench.torch
        self.bench.flush_l2(st)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(self.graphs) + 1)]
        evs[0].record(st)
        for g, e in zip(self.graphs, evs[1:]):
            g.replay()
            e.record(st)
        record.append(evs)

    @staticmethod
    def times(records):
        """-> (step seconds [n], phase seconds [n, phases])"""
        step = np.array([r[0].elapsed_time(r[-1]) for r in records]) / 1e3
        ph = np.array([[r[i].elapsed_time(r[i + 1]) for i in range(len(r) - 1)] for r in records]) / 1e3
        return step, ph


def decode_phases(bench, kind):
    """The phases of one step of a decode workload and the token-heads it scores."""
    T = bench.T
    if kind == "llama":
        return [("quantize_keys", bench.quantize_all_keys), ("quantize_values", bench.quantize_all_values),
                ("decode_attention", lambda: bench.decode(bench.app_seq[T - 1]))]
    # serving / long: append the token at position T-1 (its slot is rewritten every step),
    # then decode over the T tokens
    return [("append_quantize", lambda: bench.append(T - 1)),
            ("decode_attention", lambda: bench.decode(bench.app_seq[T - 1]))]


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
    kind = args.config
    w = DECODE_CONFIGS[kind]
    bench = DecodeBench(w, dev)
    if kind == "llama":
        bench.prefill(bench.max_len)
    else:
        bench.prefill(w.context - 1)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream(dev)
    runner = StepRunner(bench, decode_phases(bench, kind))
    n0 = tq.launch_count()
    for name, fn in decode_phases(bench, kind):
        fn()
    torch.cuda.synchronize()
    per_step_launches = tq.launch_count() - n0
    keys = bench.B * bench.Hkv * bench.T          # token-heads scored per step

    for _ in range(args.warmup):
        runner.run(st, [])
    torch.cuda.synchronize()
    recs = []
    barrier = (lambda: torch.distributed.barrier()) if ws > 1 else (lambda: None)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        for _ in range(args.steps):
            runner.run(st, recs)
        torch.cuda.synchronize()
        barrier()
    clocks = clk.summary()
    t_step, t_ph = StepRunner.times(recs)
    ms_step = max_over_ranks(float(t_step.mean() * 1e3), ws, dev)
    phase_s = {n: float(t_ph[:, i].mean()) for i, n in enumerate(runner.names)}

    # end to end through the public API from pinned host buffers
    e2e = run_e2e(bench, kind, st, args.steps, args.warmup)
    e2e["ms_per_step"] = max_over_ranks(e2e["ms_per_step"], ws, dev)
    e2e["value"] = whole_job_rate(keys, ws, e2e["ms_per_step"] / 1e3)

    if rank != 0:
        if ws > 1:
            torch.distributed.destroy_process_group()
        return
    peaks = _peaks()
    value = whole_job_rate(keys, ws, ms_step / 1e3)
    dec_bytes = bench.token_head_bytes() * keys
    t_dec = phase_s["decode_attention"]
    dominant = max(phase_s, key=phase_s.get)
    rooflines = {"decode_attention": hbm_roof(dec_bytes, t_dec, peaks, "decode_attention",
                                              traffic=recorded_traffic(w.name, "decode_attention"))}
    if kind == "llama":
        n = bench.B * bench.Hkv * bench.max_len
        qkb, qvb = bench.quantize_bytes(n)
        qkf, qvf = bench.quantize_flops(n)
        for name, nb, fl, split in (("quantize_keys", qkb, qkf, 3), ("quantize_values", qvb, qvf, 3)):
            rooflines[name] = hbm_roof(nb, phase_s[name], peaks, name, traffic=recorded_traffic(w.name, name),
                                       algorithmic_tflops=fl / phase_s[name] / 1e12,
                                       executed_split_tflops=split * fl / phase_s[name] / 1e12)
    else:
        n = bench.B * bench.Hkv
        qkb, qvb = bench.quantize_bytes(n)
        rooflines["append_quantize"] = hbm_roof(qkb + qvb, phase_s["append_quantize"], peaks, "append_quantize",
                                                note="512 key + 512 value vectors per group: launch-bound")
    line = {
        "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, kind, ws),
        "components": dict({n + "_us": s * 1e6 for n, s in phase_s.items()},
                           decode_keys_scored_per_s=keys / t_dec,
                           decode_hbm_gbs=dec_bytes / t_dec / 1e9,
                           decode_frac_of_8tbs=dec_bytes / t_dec / 1e9 / NOMINAL_HBM_GBS),
        "timing": "device time of CUDA-graph replays of the library calls (captured once), CUDA events on the "
                  "launching stream, L2 flushed (256 MiB write) before every step",
        "roofline": rooflines[dominant],
        "rooflines": rooflines,
        "e2e": e2e,
        "gpu_launches": int(per_step_launches * args.steps),
        "clocks": clocks,
    }
    if kind == "llama" and args.configs:
        line["rows"] = measure_rows(bench, peaks)
    del runner
    bench.free()
    del bench
    torch.cuda.empty_cache()
    if args.configs:
        line["stream_peaks"] = guarded(measure_stream, dev)
        line["configs"] = measure_configs(kind, dev, peaks, args)
    line["cpu_baseline"] = cpu_baseline(w, kind)
    print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


def workload_config(w, kind, ws):
    step = {"llama": "quantize the whole K/V cache, then decode attention for 1 token",
            "serving": "append-quantize 1 token per sequence (all kv heads, both groups), then decode attention "
                       "for 1 query token per sequence over the full context",
            "long": "append-quantize 1 token, then decode attention over the full context"}[kind]
    return {"workload": w.name, "batch": w.batch, "q_heads": w.q_heads, "kv_heads": w.kv_heads,
            "head_dim": w.head_dim, "context": w.context,
            "groups": [{"channels": [o, o + wd], "key_bits": kb, "value_bits": vb} for o, wd, kb, vb in w.groups],
            "outlier_channels_per_head": w.outliers, "lognormal_sigma": w.lognormal_sigma, "step": step,
            "l2": "flushed (256 MiB write) before every step", "parallelism": "replicas%d" % ws}


# ---------------------------------------------------------------- other workloads
def _time_device(fn, flush, reps, warm=1, graph=False):
    """Mean device time (s) of fn() over reps, L2 flushed before every rep.  graph=True
    captures fn once in a CUDA graph and times its replays, so that the host's launch
    latency (Python, ctypes) of a short call is not counted as device time."""
    import torch
    st = torch.cuda.current_stream()
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    run = fn
    if graph:
        side = torch.cuda.Stream()
        side.wait_stream(st)
        with torch.cuda.stream(side):
            fn()
        st.wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        run = g.replay
    ts = []
    for _ in range(reps):
        flush(st)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        run()
        b.record(st)
        ts.append((a, b))
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in ts]) / 1e3)


def measure_stream(dev):
    """Copy (read + write) and read-only streaming bandwidth of this GPU over 4 GiB,
    measured with torch kernels in the same run (context for the HBM fractions)."""
    import torch
    a = torch.empty(1 << 30, dtype=torch.float32, device=dev)
    b = torch.empty_like(a)
    a.fill_(1.0)
    torch.cuda.synchronize()
    nofl = lambda st: None
    t_copy = min(_time_device(lambda: b.copy_(a), nofl, 5) for _ in range(2))
    t_read = min(_time_device(lambda: torch.sum(a), nofl, 5) for _ in range(2))
    nb = a.numel() * 4
    del a, b
    torch.cuda.empty_cache()
    return {"copy_gbs": 2 * nb / t_copy / 1e9, "read_only_gbs": nb / t_read / 1e9,
            "how": "torch copy_ and sum over 4 GiB fp32, best of 2 x mean of 5, CUDA events"}


def guarded(fn, *a):
    """fn(*a), or {"error": ...} if it raises (a secondary measurement never costs the
    headline line)."""
    import torch
    try:
        return fn(*a)
    except Exception as e:  # noqa: BLE001
        torch.cuda.synchronize()
        return {"error": "%s: %s" % (type(e).__name__, e)}
    finally:
        torch.cuda.empty_cache()


def measure_configs(headline, dev, peaks, args):
    out = {}
    for kind in ("serving", "llama", "long"):
        if kind == headline:
            continue
        out[DECODE_CONFIGS[kind].name] = guarded(measure_decode_config, kind, dev, peaks)
    out[W.TOY["name"]] = guarded(measure_toy, dev)
    for spec in (W.SEARCH_1536, W.SEARCH_200, W.SEARCH_3072):
        out[spec["name"]] = guarded(measure_search, spec, dev, peaks)
    return out


def measure_decode_config(kind, dev, peaks, steps=10):
    """Step time of another decode workload (CUDA-graph phases, L2 flushed before each
    step); the long-context workload also reports its full prefill quantize and the mean
    of its 32 appending decode steps."""
    import torch
    w = DECODE_CONFIGS[kind]
    extra = w.decode_steps if kind == "long" else 0
    bench = DecodeBench(w, dev, extra_tokens=extra)
    st = torch.cuda.current_stream(dev)
    res = {"config": workload_config(w, kind, 1)}
    if kind == "long":
        # the prefill quantize of all 131072 tokens (K and V, both groups), L2 flushed
        T = w.context
        n = bench.B * bench.Hkv * T
        rows = (torch.arange(bench.B * bench.Hkv, device=dev).view(-1, 1) * bench.max_len
                + torch.arange(T, device=dev).view(1, -1)).reshape(-1)
        Kp = bench.Kf[rows].contiguous()
        Vp = bench.Vf[rows].contiguous()

        def pre():
            for gi, (off, wd, _, _) in enumerate(w.groups):
                tq_q(bench.kctx[gi], Kp[:, off:off + wd], bench.kc[gi], rows)
                tq_q(bench.vctx[gi], Vp[:, off:off + wd], bench.vc[gi], rows)
        tq_q = lambda c, x, p, r: bench.tq.quantize_kv(c, x, p, slots=r)
        g = bench.capture(pre)
        t_pre = _time_device(g.replay, bench.flush_l2, 5)
        del Kp, Vp
        qkb, qvb = bench.quantize_bytes(n)
        qkf, qvf = bench.quantize_flops(n)
        res["prefill_quantize"] = hbm_roof(qkb + qvb, t_pre, peaks, "quantize (K+V, 2 groups)",
                                           vectors=2 * n, vectors_per_s=2 * n / t_pre,
                                           algorithmic_tflops=(qkf + qvf) / t_pre / 1e12)
        # 32 decode steps, each appending one token at T + s and attending over T + s + 1
        graphs = []
        for s in range(w.decode_steps):
            t = T - 1 + s
            if t not in bench.app_slots:
                continue
            graphs.append((bench.capture(lambda t=t: bench.append(t)),
                           bench.capture(lambda t=t: bench.decode(bench.app_seq[t])), t))
        ts, td = [], []
        for ga, gd, t in graphs:
            bench.flush_l2(st)
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(st)
            ga.replay()
            e1.record(st)
            gd.replay()
            e2.record(st)
            ts.append((e0, e1, e2))
        torch.cuda.synchronize()
        t_step = float(np.mean([a.elapsed_time(c) for a, b, c in ts]) / 1e3)
        t_dec = float(np.mean([b.elapsed_time(c) for a, b, c in ts]) / 1e3)
        keys = float(np.mean([bench.B * bench.Hkv * (t + 1) for _, _, t in graphs]))
        res["decode_steps"] = len(graphs)
        res["ms_per_step"] = t_step * 1e3
        res["keys_scored_per_s"] = keys / t_step
        res["decode_attention"] = hbm_roof(bench.token_head_bytes() * keys, t_dec, peaks, "decode_attention",
                                           keys_scored_per_s=keys / t_dec)
    else:
        if kind == "llama":
            bench.prefill(bench.max_len)
        else:
            bench.prefill(w.context - 1)
        runner = StepRunner(bench, decode_phases(bench, kind))
        for _ in range(3):
            runner.run(st, [])
        recs = []
        for _ in range(steps):
            runner.run(st, recs)
        torch.cuda.synchronize()
        t_step, t_ph = StepRunner.times(recs)
        keys = bench.B * bench.Hkv * bench.T
        ph = {n: float(t_ph[:, i].mean()) for i, n in enumerate(runner.names)}
        res["ms_per_step"] = float(t_step.mean() * 1e3)
        res["keys_scored_per_s"] = keys / float(t_step.mean())
        res["phases_us"] = {n: s * 1e6 for n, s in ph.items()}
        res["decode_attention"] = hbm_roof(bench.token_head_bytes() * keys, ph["decode_attention"], peaks,
                                           "decode_attention", keys_scored_per_s=keys / ph["decode_attention"],
                                           traffic=recorded_traffic(w.name, "decode_attention"))
        if kind == "llama":
            n = bench.B * bench.Hkv * bench.max_len
            qkb, qvb = bench.quantize_bytes(n)
            qkf, qvf = bench.quantize_flops(n)
            res["quantize_keys"] = hbm_roof(qkb, ph["quantize_keys"], peaks, "quantize_keys",
                                            algorithmic_tflops=qkf / ph["quantize_keys"] / 1e12,
                                            traffic=recorded_traffic(w.name, "quantize_keys"))
            res["quantize_values"] = hbm_roof(qvb, ph["quantize_values"], peaks, "quantize_values",
                                              algorithmic_tflops=qvf / ph["quantize_values"] / 1e12,
                                              traffic=recorded_traffic(w.name, "quantize_values"))
            res["rows"] = measure_rows(bench, peaks)
        del runner
    bench.free()
    return res


def measure_rows(bench, peaks, reps=5):
    """Standalone logits (4 queries x every cached key of group 0) and dequantize (every
    cached value vector of group 0) on a decode workload's caches; device time of CUDA-graph
    replays of the library call."""
    import torch
    tq, dev = bench.tq, bench.dev
    out = {}
    kctx, kc = bench.kctx[0], bench.kc[0]
    n = kc.cap
    q4 = torch.randn((4, kctx.d), device=dev, generator=torch.Generator(device=dev).manual_seed(11))
    lg = torch.empty((4, n), dtype=torch.float32, device=dev)
    ws = torch.empty(max(int(tq.lib().tq_attn_logits_workspace_size(kctx.handle, 4)), 1), dtype=torch.uint8,
                     device=dev)
    t = _time_device(lambda: tq.attn_logits(kctx, q4, kc, n, out=lg, workspace=ws), bench.flush_l2, reps, graph=True)
    nbytes = n * (kctx.code_bytes + 4) + 4 * n * 4
    out["logits"] = hbm_roof(nbytes, t, peaks, "attn_logits",
                             work="4 queries x %d keys (d=%d, %d-bit prod)" % (n, kctx.d, kctx.bits))
    vctx, vc = bench.vctx[0], bench.vc[0]
    xo = torch.empty((n, vctx.d), dtype=torch.float32, device=dev)
    t = _time_device(lambda: tq.dequantize(vctx, vc, n, out=xo), bench.flush_l2, reps, graph=True)
    nbytes = n * (vctx.code_bytes + 2) + n * vctx.d * 4
    out["dequantize"] = hbm_roof(nbytes, t, peaks, "dequantize",
                                 work="%d value vectors (d=%d, %d-bit MSE) -> fp32" % (n, vctx.d, vctx.bits),
                                 algorithmic_tflops=2.0 * vctx.d * vctx.d * n / t / 1e12)
    kq = torch.empty((n, kctx.d), dtype=torch.float32, device=dev)
    t = _time_device(lambda: tq.dequantize(kctx, kc, n, out=kq, qjl=True), bench.flush_l2, reps, graph=True)
    nbytes = n * (kctx.code_bytes + 4) + n * kctx.d * 4
    out["dequantize_qjl"] = hbm_roof(nbytes, t, peaks, "dequantize_qjl",
                                     work="%d key vectors (d=%d, %d-bit prod) -> fp32, QJL-augmented" % (
                                         n, kctx.d, kctx.bits),
                                     algorithmic_tflops=4.0 * kctx.d * kctx.d * n / t / 1e12)
    return out


def measure_toy(dev, reps=10):
    """The toy parity workload: 4096 fp32 keys at d = 128, 3-bit prod; quantize, 16 x 4096
    logits, dequantize.  Launch-bound: times only."""
    import torch
    import kv_cache_vector_08_b200 as tq
    keys, qs = W.toy_inputs()
    x = torch.tensor(keys, device=dev)
    q = torch.tensor(qs, device=dev)
    ctx = tq.Context(W.TOY["d"], W.TOY["bits"], 1000, tq.MODE_PROD)
    pk = tq.alloc_packed(ctx, x.shape[0], dev)
    nofl = lambda st: None
    t_q = _time_device(lambda: tq.quantize_kv(ctx, x, pk), nofl, reps)
    lg = torch.empty((q.shape[0], x.shape[0]), dtype=torch.float32, device=dev)
    t_l = _time_device(lambda: tq.attn_logits(ctx, q, pk, x.shape[0], out=lg), nofl, reps)
    xo = torch.empty_like(x)
    t_d = _time_device(lambda: tq.dequantize(ctx, pk, x.shape[0], out=xo), nofl, reps)
    return {"quantize_us": t_q * 1e6, "logits_us": t_l * 1e6, "dequantize_us": t_d * 1e6,
            "note": "launch-bound parity workload; times include the ctypes call"}


def measure_search(spec, dev, peaks):
    """Index (quantize the 10^6-row fp32 database), top-10 search of 1000 queries, and
    1@10 recall against the exact fp32 maximum inner product (torch matmul, fp32)."""
    import torch
    import kv_cache_vector_08_b200 as tq
    d, N, nq, k = spec["d"], spec["n_db"], spec["n_queries"], spec["k"]
    g = torch.Generator(device=dev).manual_seed(7)
    db = torch.nn.functional.normalize(torch.randn((N, d), generator=g, device=dev), dim=1)
    qs = torch.nn.functional.normalize(torch.randn((nq, d), generator=g, device=dev), dim=1)
    ctx = tq.Context(d, spec["bits"], 12, tq.MODE_PROD)
    pk = tq.alloc_packed(ctx, N, dev)
    fl = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def flush(st):
        with torch.cuda.stream(st):
            fl.fill_(1.0)
    t_idx = _time_device(lambda: tq.quantize_kv(ctx, db, pk), flush, 3)
    scores = ids = None

    def srch():
        nonlocal scores, ids
        scores, ids = tq.search_topk(ctx, qs, pk, N, k)
    t_s = _time_device(srch, flush, 3)
    # exact fp32 nearest neighbour of every query
    old = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    best = torch.full((nq,), -float("inf"), device=dev)
    arg = torch.zeros((nq,), dtype=torch.int64, device=dev)
    for c0 in range(0, N, 100_000):
        ip = qs @ db[c0:c0 + 100_000].T
        m, a = ip.max(dim=1)
        upd = m > best
        best = torch.where(upd, m, best)
        arg = torch.where(upd, a + c0, arg)
    torch.backends.cuda.matmul.allow_tf32 = old
    recall = float((ids == arg[:, None]).any(dim=1).float().mean().item())
    idx_bytes = N * (d * 4 + ctx.code_bytes + 4)
    idx_flops = 4.0 * d * d * N
    s_flops = 4.0 * d * nq * N
    res = {"index": dict(hbm_roof(idx_bytes, t_idx, peaks, "quantize (index)"),
                         vectors_per_s=N / t_idx, algorithmic_tflops=idx_flops / t_idx / 1e12,
                         tensor_frac_sustained=idx_flops / t_idx / 1e12 / peaks["bf16_sus"]),
           "search": tensor_roof(s_flops, t_s, peaks["bf16"], "search_topk",
                                 "measured bf16 dense burst (MEASURED_PEAKS.json bf16_tflops)",
                                 queries_per_s=nq / t_s, work="%d queries x %d rows, top-%d" % (nq, N, k)),
           "recall_at_10": recall, "recall_ground_truth": "exact fp32 argmax inner product, all %d queries" % nq}
    del db, qs, pk, fl
    return res


def run_e2e(bench, kind, st, steps, warmup):
    """The step through the public API with pinned host inputs and outputs: per step the
    host-to-device copy of the step's inputs (llama: the whole bf16 K/V cache and the
    query; serving / long: the appended token's K/V rows and the queries), the library
    calls, and the device-to-host copy of the attention output, all inside the timed
    region."""
    import torch
    T = bench.T
    if kind == "llama":
        srcs = [bench.K, bench.V, bench.q]
    else:
        srcs = [bench.app_k[T - 1], bench.app_v[T - 1], bench.q]
    hosts = [torch.empty(s.shape, dtype=s.dtype, pin_memory=True) for s in srcs]
    for h, s in zip(hosts, srcs):
        h.copy_(s)
    dsts = [torch.empty_like(s) for s in srcs]
    oh = torch.empty(bench.out.shape, dtype=bench.out.dtype, pin_memory=True)
    seq = bench.app_seq[T - 1]
    times = []
    for i in range(warmup + steps):
        bench.flush_l2(st)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        for d_, h in zip(dsts, hosts):
            d_.copy_(h, non_blocking=True)
        if kind == "llama":
            K, V, q = dsts
            Kf, Vf = K.reshape(-1, bench.D), V.reshape(-1, bench.D)
            for gi, (off, wd, _, _) in enumerate(bench.w.groups):
                bench.tq.quantize_kv(bench.kctx[gi], Kf[:, off:off + wd], bench.kc[gi])
                bench.tq.quantize_kv(bench.vctx[gi], Vf[:, off:off + wd], bench.vc[gi])
        else:
            k, v, q = dsts
            bench.append(T - 1, k=k, v=v)
        bench.plan(q, seq, bench.scale, bench.out)
        oh.copy_(bench.out, non_blocking=True)
        b.record(st)
        if i >= warmup:
            times.append((a, b))
    torch.cuda.synchronize()
    t = float(np.mean([a.elapsed_time(b) for a, b in times]) / 1e3)
    h2d = sum(h.numel() * h.element_size() for h in hosts)
    keys = bench.B * bench.Hkv * bench.T
    return {"value": keys / t, "unit": "keys/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(oh.numel() * oh.element_size()), "ms_per_step": t * 1e3,
            "how": "eager library calls (no graph; the append's key and value calls on parallel streams), pinned host buffers"}


# -------------------------------------------------------------------- CPU oracle
class OracleSample:
    """The float64 oracle on a bounded sample of a decode workload: sequence 0's first
    `heads` KV heads at the full context.  Set-up (parameters, the sample's prefill cache
    quantized by the oracle) happens once; a step quantizes the appended token (serving /
    long) or the whole sampled cache (llama) and decodes the sampled query heads."""

    def __init__(self, w, kind, heads, seed=0):
        import oracle
        self.oracle, self.w, self.kind, self.heads = oracle, w, kind, heads
        D, T = w.head_dim, w.context
        self.rep = w.q_heads // w.kv_heads
        self.kp = [oracle.make_params(wd, kb, 1000 + 2 * gi, 0) for gi, (_, wd, kb, _) in enumerate(w.groups)]
        self.vp = [oracle.make_params(wd, vb, 1001 + 2 * gi, 1) for gi, (_, wd, _, vb) in enumerate(w.groups)]
        K, V = W.decode_kv(w, seed, context=T, batch=1)
        self.K, self.V = K[:, :heads], V[:, :heads]
        self.q = W.decode_queries(w, seed, batch=1)[:, :heads * self.rep]
        self.offs = [g[0] for g in w.groups] + [D]
        self.kcodes, self.vcodes = self._quantize(self.K, self.V)

    def _quantize(self, K, V):
        o = self.oracle
        Tn, D = K.shape[2], self.w.head_dim
        kcodes, vcodes = [], []
        for gi, (off, wd, _, _) in enumerate(self.w.groups):
            ko = o.quantize(self.kp[gi], K[..., off:off + wd].reshape(-1, wd).astype(np.float64))
            vo = o.quantize(self.vp[gi], V[..., off:off + wd].reshape(-1, wd).astype(np.float64))
            sh = (1, self.heads, Tn)
            kcodes.append(dict(idx=ko["idx"].reshape(sh + (wd,)), signs=ko["signs"].reshape(sh + (wd,)),
                               norm=ko["norm"].reshape(sh), rnorm=ko["rnorm"].reshape(sh)))
            vcodes.append(dict(idx=vo["idx"].reshape(sh + (wd,)), norm=vo["norm"].reshape(sh)))
        return kcodes, vcodes

    def step(self):
        T = self.w.context
        if self.kind == "llama":
            kcodes, vcodes = self._quantize(self.K, self.V)
        else:
            nk, nv = self._quantize(self.K[:, :, T - 1:], self.V[:, :, T - 1:])
            for c, n in zip(self.kcodes + self.vcodes, nk + nv):
                for key in c:
                    c[key][:, :, T - 1:] = n[key]
            kcodes, vcodes = self.kcodes, self.vcodes
        self.oracle.decode_attention(self.kp, self.vp, self.offs, self.q.astype(np.float64), kcodes, vcodes, [T],
                                     1.0 / math.sqrt(self.w.head_dim))
        return self.heads * T

    def describe(self, dt):
        w = self.w
        what = "quantize the sampled K/V cache" if self.kind == "llama" else "append-quantize 1 token per kv head"
        return ("sequence 0, %d of %d KV heads at the full %d-token context (%d of %d token-heads of a step): %s "
                "(float64), decode its %d query heads; %.2f s per step" % (
                    self.heads, w.kv_heads, w.context, self.heads * w.context, w.batch * w.kv_heads * w.context,
                    what, self.heads * self.rep, dt))


def _oracle_heads(kind):
    return {"serving": 8, "llama": 2, "long": 1}[kind]


def cpu_baseline(w, kind):
    s = OracleSample(w, kind, _oracle_heads(kind))
    s.step()
    t0 = time.perf_counter()
    keys = s.step()
    dt = time.perf_counter() - t0
    return {"value": keys / dt, "unit": "keys/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": s.describe(dt)}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return
    kind = args.config
    w = DECODE_CONFIGS[kind]
    s = OracleSample(w, kind, _oracle_heads(kind))
    for _ in range(args.warmup):
        s.step()
    ts = []
    keys = 0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        keys = s.step()
        ts.append(time.perf_counter() - t0)
    t = float(np.mean(ts))
    value = keys / t
    cfg = workload_config(w, kind, ws)
    cfg["sample"] = "%d of %d KV heads of sequence 0" % (s.heads, w.kv_heads * w.batch)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "keys/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": "keys/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": s.describe(t)},
        "e2e": {"value": value, "unit": "keys/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------- small cases for profilers
KERNEL_CASES = ("decode-serving-b16", "search-d1536-200k", "search-d200-1m", "dequant-d128", "quantize-fp32-d1536", "logits-d128")


def run_kernel_case(args):
    """One small case of a kernel family, run `reps` times, for ncu captures (inputs larger
    than L2, a few GB on the device at most).  Prints the median device time of the call;
    this is a profiling aid, not a bench line."""
    import dataclasses
    import torch
    import kv_cache_vector_08_b200 as tq
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    case = args.kernel_case

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        return sorted(a.elapsed_time(b) for a, b in ts)[len(ts) // 2] * 1e3

    if case == "decode-serving-b16":
        w = dataclasses.replace(W.SERVING_3P5, batch=16, name="serving-decode-3.5bit-b16")
        bench = DecodeBench(w, dev)
        bench.prefill(bench.max_len)
        seq = torch.full((bench.B,), bench.T, dtype=torch.int32, device=dev)
        us = timed(lambda: bench.decode(seq))
        note = "%d token-heads" % (bench.B * bench.Hkv * bench.T)
    elif case in ("search-d1536-200k", "search-d200-1m"):
        d, N, nq = (1536, 200000, 1000) if case == "search-d1536-200k" else (200, 1000000, 1000)
        db = torch.nn.functional.normalize(torch.randn((N, d), generator=g, device=dev), dim=1)
        qs = torch.nn.functional.normalize(torch.randn((nq, d), generator=g, device=dev), dim=1)
        ctx = tq.Context(d, 4, 12, tq.MODE_PROD)
        pk = tq.alloc_packed(ctx, N)
        tq.quantize_kv(ctx, db, pk)
        del db
        us = timed(lambda: tq.search_topk(ctx, qs, pk, N, 10))
        note = "%.0f TFLOP/s (4 d flops per pair)" % (4.0 * d * N * nq / us / 1e6)
    elif case == "dequant-d128":
        d, n = 128, 262144
        x = torch.randn((n, d), generator=g, device=dev).to(torch.bfloat16)
        ctx = tq.Context(d, 4, 5, tq.MODE_MSE)
        pk = tq.alloc_packed(ctx, n)
        tq.quantize_kv(ctx, x, pk)
        out = torch.empty((n, d), device=dev)
        us = timed(lambda: tq.dequantize(ctx, pk, n, out=out))
        note = "%.0f GB/s (66 + 512 B per vector)" % (n * (66 + 512) / us / 1e3)
    elif case == "logits-d128":
        d, n, nq = 128, 262144, 4
        x = torch.randn((n, d), generator=g, device=dev).to(torch.bfloat16)
        ctx = tq.Context(d, 4, 1000, tq.MODE_PROD)
        pk = tq.alloc_packed(ctx, n)
        tq.quantize_kv(ctx, x, pk)
        q4 = torch.randn((nq, d), generator=g, device=dev)
        lg = torch.empty((nq, n), dtype=torch.float32, device=dev)
        ws = torch.empty(max(int(tq.lib().tq_attn_logits_workspace_size(ctx.handle, nq)), 1), dtype=torch.uint8,
                         device=dev)
        us = timed(lambda: tq.attn_logits(ctx, q4, pk, n, out=lg, workspace=ws))
        note = "%.0f GB/s (68 B of codes and norms + 16 B of logits per key)" % (n * 84 / us / 1e3)
    else:   # quantize-fp32-d1536
        d, n = 1536, 32768
        x = torch.nn.functional.normalize(torch.randn((n, d), generator=g, device=dev), dim=1)
        ctx = tq.Context(d, 4, 12, tq.MODE_PROD)
        pk = tq.alloc_packed(ctx, n)
        ws = torch.empty(tq.quantize_workspace_size(ctx, 0, n, d), dtype=torch.uint8, device=dev)
        us = timed(lambda: tq.quantize_kv(ctx, x, pk, workspace=ws))
        note = "%.0f TFLOP/s algorithmic (4 d^2 per vector)" % (4.0 * d * d * n / us / 1e6)
    print("%s: %.1f us per call (median of %d), %s" % (case, us, args.reps, note), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--config", default="serving", choices=sorted(DECODE_CONFIGS),
                    help="headline decode workload")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the measurements of the other workloads")
    ap.add_argument("--kernel-case", choices=KERNEL_CASES,
                    help="run one small case of a kernel family for a profiler instead of the bench")
    ap.add_argument("--reps", type=int, default=3, help="calls of --kernel-case")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.kernel_case:
        run_kernel_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
