"""Benchmark of the VAR-Q packed-KV hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--bits B] [--impl ours|reference]

One step = plan the cache (host), quantize+pack K and V of the whole cache
(varq_quantize_pack, two launches), then fused packed-KV attention of the
query block over every cached token (varq_packed_attention).  Default
workload: the Infinity-8B-like next-scale 1024px layer (B=2 CFG pair, 32 heads,
D=128, 13 scales / 10,521 tokens, 4096-token query block), INT4, with INT2
measured the same way and reported under "also".

Printed (rank 0, one JSON line): the metric, whole-job value (attention
TFLOP/s over the full step time), per-kernel CUDA-event times, the roofline
of the dominant kernel (attention, tensor-bound) and of quantize+pack
(HBM-bound) against the measured peaks in MEASURED_PEAKS.json, the CPU
oracle timed on a bounded sample (cpu_baseline), the end-to-end number
through the C ABI with host buffers (e2e), SM clocks sampled during the timed
region, and the number of library kernel launches.

Multi-GPU (torchrun, one process per GPU): every rank runs its own copy of
the workload (the path shards by (batch, head) with no exchange), so scaling
is weak; the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from packed_kv_attention_b200 import synth  # noqa: E402

METRIC = "fused packed-KV attention TFLOP/s and quant+pack GB/s at INT4/INT2 (% of roofline)"

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the
# dominant kernel (attn_tc_kernel<4,128,2,false> on the Infinity-8B-like INT4
# layer), from one ncu capture of this bench run with `--steps 2 --warmup 3
# --also-bits 0 --no-e2e --no-cpu-baseline --no-rows`, the fourth launch of the
# kernel.  Reported as the roofline "traffic" only while the kernel's sources
# hash to the value they had when the counters were taken; otherwise null.
MEASURED_TRAFFIC = {"workload": "infinity_8b", "bits": 4, "lq": 4096, "rope": False,
                    "bytes": 154.583552e6 + 40.038144e6, "sources_sha256_16": "7cfc2c2543c454d0"}
TRAFFIC_SOURCES = ("packed_kv_attention_b200/csrc/attn_tc.cu", "packed_kv_attention_b200/csrc/attn_tc_common.cuh",
                   "packed_kv_attention_b200/csrc/common.cuh")


def measured_traffic(w, bits, lq, rope):
    """ncu DRAM bytes per attention launch when they still describe this kernel and workload."""
    import hashlib
    m = MEASURED_TRAFFIC
    if (w.name, bits, lq, rope) != (m["workload"], m["bits"], m["lq"], m["rope"]):
        return None
    h = hashlib.sha256()
    try:
        for f in TRAFFIC_SOURCES:
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return m["bytes"] if h.hexdigest()[:16] == m["sources_sha256_16"] else None
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def attention_flops(w, lq):
    return 4.0 * w.batch * w.heads * lq * w.n_tokens * w.head_dim


def quant_bytes(L, w):
    """Algorithmic bytes of one quantize+pack of K and V: bf16 read once,
    packed words and metadata written once."""
    bf16 = w.batch * w.heads * w.n_tokens * w.head_dim * 2
    return 2 * (bf16 + L.packed_bytes + L.meta_bytes)


def attention_bytes(L, w, lq, rope):
    qo = 2 * w.batch * w.heads * lq * w.head_dim * 2
    kv = 2 * (L.packed_bytes + L.meta_bytes)
    tables = (w.n_tokens * w.head_dim // 2 * 4 * 2) if rope else 0
    return qo + kv + tables


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        busy = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# --------------------------------------------------------------- our arm

class Pipeline:
    """Device buffers and the step of one workload at one bit width."""

    def __init__(self, w, bits, lq, device, seed=0):
        from packed_kv_attention_b200 import varq as V
        self.V = V
        self.w, self.bits, self.lq = w, bits, lq
        data = synth.make_inputs(w, lq=lq, seed=seed, device=device)
        self.k, self.v, self.q = data["k"], data["v"], data["q"]
        self.cos, self.sin = data.get("rope_cos"), data.get("rope_sin")
        self.bs = data["block_start"]
        self.L = V.varq_cache_alloc(w.batch, w.heads, w.head_dim, bits, self.bs)
        self.kp, self.km = V.alloc_cache(self.L, device)
        self.vp, self.vm = V.alloc_cache(self.L, device)
        self.out = torch.empty_like(self.q)
        ws = V.varq_packed_attention_workspace(self.L, lq, w.n_blocks)
        self.ws = torch.empty(max(ws // 4, 1), dtype=torch.float32, device=device)
        # quantize+pack of K and V plus the attention (split-KV: split + combine)
        self.launches_per_step = 2 * V.varq_quantize_pack_launches(self.L) + (1 if ws == 0 else 2)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        # made on the default stream; the library's launches go to another one
        torch.cuda.synchronize(device)

    def step(self, stream, ev=None):
        V = self.V
        self.L = V.varq_cache_alloc(self.w.batch, self.w.heads, self.w.head_dim, self.bits, self.bs)
        if ev is not None:
            ev[0].record(stream)
        V.varq_quantize_pack(self.L, self.k, self.kp, self.km, dev_status=self.status, stream=stream)
        V.varq_quantize_pack(self.L, self.v, self.vp, self.vm, dev_status=self.status, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        V.varq_packed_attention(self.L, self.q, self.kp, self.km, self.vp, self.vm, self.out,
                                rope_cos=self.cos, rope_sin=self.sin, workspace=self.ws,
                                dev_status=self.status, stream=stream)
        if ev is not None:
            ev[2].record(stream)


def max_over_ranks(x, device, dist_ok):
    """The largest value of x over all ranks (x itself on one rank)."""
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    if dist_ok:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world, flops_per_rank_step, steps, total_ms):
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (total_ms * 1e-3) / 1e12


def time_ours(pipe, steps, warmup, stream, dist_ok):
    for _ in range(warmup):
        pipe.step(stream)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist_ok:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(steps):
        pipe.step(stream, evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    if dist_ok:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(end)
    qp = [e[0].elapsed_time(e[1]) for e in evs]
    at = [e[1].elapsed_time(e[2]) for e in evs]
    return total_ms, qp, at


def time_e2e(pipe, steps, warmup, stream):
    """The same step through the C ABI with host buffers: every step copies its
    K, V and Q in from pinned host memory and its output back out, inside the
    timed region.  As a serving loop would, the copies run on their own streams
    (host->device and device->host use the two directions of the link) and
    overlap the neighbouring steps' kernels: two device buffer sets alternate,
    and events order each copy after the kernels that last used its buffers."""
    V = pipe.V
    hk = pipe.k.cpu().pin_memory()
    hv = pipe.v.cpu().pin_memory()
    hq = pipe.q.cpu().pin_memory()
    ho = torch.empty(pipe.out.shape, dtype=pipe.out.dtype).pin_memory()
    dev = pipe.k.device
    bufs = [(pipe.k, pipe.v, pipe.q, pipe.out),
            (torch.empty_like(pipe.k), torch.empty_like(pipe.v), torch.empty_like(pipe.q), torch.empty_like(pipe.out))]
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, computed, out_read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    torch.cuda.synchronize(dev)
    for e in computed + out_read:  # nothing pending on either buffer set yet
        e.record(stream)

    def one(i):
        k, v, q, out = bufs[i & 1]
        with torch.cuda.stream(h2d):
            h2d.wait_event(computed[i & 1])      # the kernels of step i - 2 are done with this set
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            q.copy_(hq, non_blocking=True)
            in_ready[i & 1].record(h2d)
        stream.wait_event(in_ready[i & 1])
        stream.wait_event(out_read[i & 1])        # step i - 2's output has left the device
        V.varq_quantize_pack(pipe.L, k, pipe.kp, pipe.km, dev_status=pipe.status, stream=stream)
        V.varq_quantize_pack(pipe.L, v, pipe.vp, pipe.vm, dev_status=pipe.status, stream=stream)
        V.varq_packed_attention(pipe.L, q, pipe.kp, pipe.km, pipe.vp, pipe.vm, out, rope_cos=pipe.cos,
                                rope_sin=pipe.sin, workspace=pipe.ws, dev_status=pipe.status, stream=stream)
        computed[i & 1].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(computed[i & 1])
            ho.copy_(out, non_blocking=True)
            out_read[i & 1].record(d2h)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize(dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(h2d)
    for i in range(steps):
        one(warmup + i)
    d2h.wait_event(computed[(warmup + steps - 1) & 1])
    e.record(d2h)
    torch.cuda.synchronize(dev)
    h2d_bytes = (hk.numel() + hv.numel() + hq.numel()) * 2
    d2h_bytes = ho.numel() * 2
    # the host copy of the last step equals the device output of the same inputs
    same = bool(torch.equal(ho, pipe.out.cpu()))
    del bufs
    return s.elapsed_time(e) / steps, h2d_bytes, d2h_bytes, same


# ------------------------------------------------------------- CPU oracle

def oracle_sample(w, bits, lq, rows, seed=0):
    """Bounded CPU sample of one step: quantize+pack+dequantize K and V of one
    (batch, head) slice, then fp64 attention of `rows` query rows over it.
    Returns (seconds, attention flops of the sample, description)."""
    from oracle import varq_oracle as O
    data = synth.make_inputs(w, lq=lq, seed=seed, device="cpu", batch=1, heads=1)
    bs = data["block_start"]
    kb = data["k"].view(torch.int16).numpy().view(np.uint16)
    vb = data["v"].view(torch.int16).numpy().view(np.uint16)
    qb = data["q"][0, 0].view(torch.int16).numpy().view(np.uint16)
    rsel = np.arange(min(rows, lq))
    cos = data.get("rope_cos")
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=cpu_cores()):  # numpy's BLAS on every core this process may use
        t0 = time.perf_counter()
        hats = []
        for xb in (kb, vb):
            codes, s, mn = O.quantize(xb, bs, bits)
            words = O.pack(codes, bits)
            meta = O.meta_words(s, mn)
            hats.append(O.dequantize(O.unpack(words, bits, bs[-1]), meta, bs)[0, 0])
        O.attention(qb, hats[0], hats[1], rope_cos=None if cos is None else cos.numpy(),
                    rope_sin=None if cos is None else data["rope_sin"].numpy(), rows=rsel)
        dt = time.perf_counter() - t0
    flops = 4.0 * len(rsel) * w.n_tokens * w.head_dim
    desc = (f"one (batch, head) slice of {w.name}: quantize+pack+unpack+dequant of K and V "
            f"({w.n_tokens} tokens x {w.head_dim} channels), fp64 attention of {len(rsel)} query rows")
    return dt, flops, desc


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, w, rank, world):
    if rank != 0:
        return 0
    rows = args.oracle_rows
    times, flops = [], 0.0
    desc = ""
    for _ in range(args.warmup):
        oracle_sample(w, args.bits, args.lq, rows)
    for _ in range(args.steps):
        dt, flops, desc = oracle_sample(w, args.bits, args.lq, rows)
        times.append(dt)
    tot = sum(times)
    val = flops * len(times) / tot / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, args),
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle", "sample": desc},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _event_times(fn, stream, iters):
    """Per-iteration device times (ms) of fn() on stream, each bracketed by
    CUDA events (every input below exceeds the 126 MB L2)."""
    torch.cuda.synchronize()
    times = []
    for _ in range(iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    return times


def measure_rows(dev, stream, peaks, iters=5):
    """The hot-path steps bench's main step does not time, each on the
    workload made for it and against its own roofline:
      a2-a5 quantize+pack and a6 unpack+dequant on the 1 GiB kernel-sweep
            cache (bits 2, 3, 4, 8; inputs and outputs exceed L2);
      a9    split-KV attention (Lq = 1, 4 and 16) over the sweep cache (INT4);
      a8    pre-RoPE keys: tensor-path attention of the Self-Forcing-like
            next-frame layer (INT4, 4680 queries over 32,760 tokens)."""
    from packed_kv_attention_b200 import varq as V
    hbm = peaks["hbm_gbs"]
    # kernels here are timed over regions well under a second at full clocks:
    # the burst peak applies; the sustained (power-capped) one is reported beside
    tflops_peak = peaks["bf16_tflops"]
    tflops_sus = peaks["bf16_tflops_sustained"]
    rows = {}
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    w = synth.WORKLOADS["sweep"]
    data = synth.make_inputs(w, lq=16, seed=3, device=dev)
    k, v = data["k"], data["v"]
    bs = data["block_start"]
    out = torch.empty_like(k)
    qp, ud = {}, {}
    for bits in (2, 3, 4, 8):
        L = V.varq_cache_alloc(w.batch, w.heads, w.head_dim, bits, bs)
        kp, km = V.alloc_cache(L, dev)
        torch.cuda.synchronize()  # made on the default stream, used on `stream`
        for _ in range(3):
            V.varq_quantize_pack(L, k, kp, km, dev_status=st, stream=stream)
        tq = statistics.median(_event_times(
            lambda: V.varq_quantize_pack(L, k, kp, km, dev_status=st, stream=stream), stream, iters))
        for _ in range(3):
            V.varq_unpack_dequant(L, kp, km, out, stream=stream)
        tu = statistics.median(_event_times(lambda: V.varq_unpack_dequant(L, kp, km, out, stream=stream), stream, iters))
        nbytes = k.numel() * 2 + L.packed_bytes + L.meta_bytes
        qp[f"int{bits}"] = {"us": 1e3 * tq, "GB/s": nbytes / (tq * 1e-3) / 1e9, "frac_hbm": nbytes / (tq * 1e-3) / 1e9 / hbm}
        ud[f"int{bits}"] = {"us": 1e3 * tu, "GB/s": nbytes / (tu * 1e-3) / 1e9, "frac_hbm": nbytes / (tu * 1e-3) / 1e9 / hbm}
        if bits == 4:
            kp4, km4, L4 = kp, km, L
    desc = f"sweep: B={w.batch} H={w.heads} D={w.head_dim} T={w.n_tokens} blocks={w.n_blocks}"
    rows["a2_a5_quant_pack"] = {"workload": desc, "bytes": "bf16 read + packed + metadata written", **qp}
    rows["a6_unpack_dequant"] = {"workload": desc, "bytes": "packed + metadata read + bf16 written", **ud}

    # a9: split-KV attention over the INT4 sweep cache (K and V share the packed words here)
    vp4, vm4 = V.alloc_cache(L4, dev)
    torch.cuda.synchronize()
    V.varq_quantize_pack(L4, v, vp4, vm4, dev_status=st, stream=stream)
    split = {}
    for lq in (1, 4, 16):
        q = data["q"][:, :, :lq].contiguous()
        o = torch.empty_like(q)
        ws_bytes = V.varq_packed_attention_workspace(L4, lq, w.n_blocks, V.PATH_SPLIT)
        ws = torch.empty(max(ws_bytes // 4, 1), dtype=torch.float32, device=dev)

        def run():
            V.varq_packed_attention(L4, q, kp4, km4, vp4, vm4, o, workspace=ws, path=V.PATH_SPLIT,
                                    dev_status=st, stream=stream)
        torch.cuda.synchronize()
        for _ in range(3):
            run()
        t = statistics.median(_event_times(run, stream, iters))
        nbytes = attention_bytes(L4, w, lq, False)
        split[f"lq{lq}"] = {"us": 1e3 * t, "GB/s": nbytes / (t * 1e-3) / 1e9,
                            "frac_hbm": nbytes / (t * 1e-3) / 1e9 / hbm}
    rows["a9_split_kv"] = {"workload": desc + " INT4", "bound": "hbm",
                           "bytes": "Q + O + packed K, V + metadata", **split}
    del data, k, v, out, kp4, km4, vp4, vm4
    torch.cuda.empty_cache()

    # a8: pre-RoPE keys on the tensor path (Self-Forcing-like layer)
    w = synth.WORKLOADS["self_forcing"]
    pipe = Pipeline(w, 4, w.lq[-1], dev, seed=4)
    torch.cuda.synchronize()
    pipe.step(stream)
    torch.cuda.synchronize()

    def attn():
        V.varq_packed_attention(pipe.L, pipe.q, pipe.kp, pipe.km, pipe.vp, pipe.vm, pipe.out,
                                rope_cos=pipe.cos, rope_sin=pipe.sin, workspace=pipe.ws,
                                dev_status=st, stream=stream)
    torch.cuda.synchronize()
    for _ in range(2):
        attn()
    t = statistics.median(_event_times(attn, stream, 3))
    fl = attention_flops(w, w.lq[-1])

    # the same layer with keys rotated before quantization (post-RoPE cache):
    # no tables, the plain tensor path; the cost comparison of the two modes
    def attn_post():
        V.varq_packed_attention(pipe.L, pipe.q, pipe.kp, pipe.km, pipe.vp, pipe.vm, pipe.out,
                                workspace=pipe.ws, dev_status=st, stream=stream)
    for _ in range(2):
        attn_post()
    t_post = statistics.median(_event_times(attn_post, stream, 3))

    # the same pre-RoPE layer with the angles computed in the kernel from the
    # (frame, row, column) schedule the tables describe
    rope3d = V.Rope3d.make(1560, 52, synth.rope_axis_pairs(w.head_dim))

    def attn_sched():
        V.varq_packed_attention_rope3d(pipe.L, pipe.q, pipe.kp, pipe.km, pipe.vp, pipe.vm, pipe.out, rope3d,
                                       workspace=pipe.ws, dev_status=st, stream=stream)
    for _ in range(2):
        attn_sched()
    t_sched = statistics.median(_event_times(attn_sched, stream, 3))
    rows["a8_pre_rope_attention"] = {
        "workload": f"self_forcing: B={w.batch} H={w.heads} D={w.head_dim} T={w.n_tokens} Lq={w.lq[-1]} INT4 pre-RoPE "
                    "keys, 3D rotary schedule (1560-token frames, 52-wide rows) computed in the kernel; tables_* = "
                    "the same angles read from [T, D/2] fp32 tables; post_rope_* = keys rotated before quantization",
        "bound": "tensor", "ms": t_sched, "TFLOP/s": fl / (t_sched * 1e-3) / 1e12,
        "frac_tensor": fl / (t_sched * 1e-3) / 1e12 / tflops_peak,
        "frac_tensor_sustained": fl / (t_sched * 1e-3) / 1e12 / tflops_sus,
        "tables_ms": t, "tables_TFLOP/s": fl / (t * 1e-3) / 1e12,
        "post_rope_ms": t_post, "post_rope_TFLOP/s": fl / (t_post * 1e-3) / 1e12}
    del pipe
    torch.cuda.empty_cache()

    # generation loop (a step beyond the path's single call): per generation
    # block, quantize+pack its K and V into the preallocated caches, then its
    # queries attend to all blocks so far; whole loop timed, INT4
    from packed_kv_attention_b200.generation import PackedKVLoop
    loops = {}
    for name in ("var_d16", "infinity_8b"):
        w = synth.WORKLOADS[name]
        data = synth.make_inputs(w, lq=1, seed=5, device=dev)
        k, v, bs = data["k"], data["v"], data["block_start"]
        g = torch.Generator(device=dev)
        g.manual_seed(5)
        qs = [torch.randn(w.batch, w.heads, n, w.head_dim, generator=g, device=dev).to(torch.bfloat16)
              for n in w.block_sizes]
        outs = [torch.empty_like(q) for q in qs]
        loop = PackedKVLoop(w.batch, w.heads, w.head_dim, 4, w.block_sizes, device=dev)
        torch.cuda.synchronize()  # inputs and buffers were made on the default stream

        def run_loop():
            for i in range(len(w.block_sizes)):
                loop.step(i, k[:, :, bs[i]:bs[i + 1]], v[:, :, bs[i]:bs[i + 1]], qs[i], out=outs[i], stream=stream)
        run_loop()
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > L2, written between timed loops
        times = []
        for _ in range(3):
            with torch.cuda.stream(stream):
                flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            run_loop()
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        t = statistics.median(times)
        # the same loop captured once in a CUDA graph and replayed (launch costs
        # leave the host); the library makes no allocation or synchronisation
        graph_ms, graph_note = None, None
        try:
            ref = [o.clone() for o in outs]
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                run_loop()
            with torch.cuda.stream(stream):  # replay() runs on the current stream
                for o in outs:
                    o.zero_()
                graph.replay()
            torch.cuda.synchronize()
            if not all(torch.equal(o, r) for o, r in zip(outs, ref)):
                raise RuntimeError("graph replay did not reproduce the loop's outputs")
            gtimes = []
            for _ in range(3):
                with torch.cuda.stream(stream):
                    flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                with torch.cuda.stream(stream):
                    graph.replay()
                b.record(stream)
                torch.cuda.synchronize()
                gtimes.append(a.elapsed_time(b))
            graph_ms = statistics.median(gtimes)
            del graph, ref
        except Exception as e:  # capture not possible here: keep the stream-launched time only
            graph_note = f"{type(e).__name__}: {str(e)[:160]}"
            torch.cuda.synchronize()
        del flush
        fl = sum(4.0 * w.batch * w.heads * n * bs[i + 1] * w.head_dim for i, n in enumerate(w.block_sizes))
        loops[name] = {"steps": len(w.block_sizes), "ms": t, "ms_per_step": t / len(w.block_sizes),
                       "attention_TFLOP": fl / 1e12, "TFLOP/s": fl / (t * 1e-3) / 1e12,
                       "graph_ms": graph_ms, "device_status": loop.device_status()}
        if graph_note:
            loops[name]["graph_note"] = graph_note
        del data, k, v, qs, outs, loop
        torch.cuda.empty_cache()
    rows["next_generation_loop"] = {
        "workload": "VAR-d16-like (B1 H16 D64, 10 blocks, T=680) and Infinity-8B-like (B2 H32 D128, 13 blocks, "
                    "T=10521); each step: quantize+pack K, V of block k, then its queries over blocks 0..k; INT4; "
                    "L2 flushed before each timed loop",
        **loops}
    rows["device_status"] = int(st.item())
    return rows


def _median_ms(fn, stream, iters, warm=2):
    # the inputs and buffers were made on the default stream, the library runs
    # on `stream`: finish the former before the first launch
    torch.cuda.synchronize()
    for _ in range(warm):
        fn()
    return statistics.median(_event_times(fn, stream, iters))


def roofline_frac(flops, nbytes, ms, peaks):
    """Binding roofline time (tensor at the burst bf16 peak, or HBM) over the
    measured time, and which one binds."""
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    return max(t_tc, t_hbm) / (ms * 1e-3), ("tensor" if t_tc >= t_hbm else "hbm")


def measure_fused_vs_unfused(dev, stream, peaks, bits=4, iters=3):
    """Kernel-sweep cache (B8 H32 T16384 D128, 16 blocks of 1,024), query
    blocks of 1 to 4,096 tokens: the fused packed-KV attention against the
    unfused baseline (unpack+dequant of K and V into dense bf16, then dense
    tensor-core attention over them), each against its binding roofline."""
    from packed_kv_attention_b200 import varq as V
    w = synth.WORKLOADS["sweep"]
    data = synth.make_inputs(w, lq=max(w.lq), seed=6, device=dev)
    bs = data["block_start"]
    L = V.varq_cache_alloc(w.batch, w.heads, w.head_dim, bits, bs)
    kp, km = V.alloc_cache(L, dev)
    vp, vm = V.alloc_cache(L, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()  # inputs and buffers come from the default stream
    V.varq_quantize_pack(L, data["k"], kp, km, dev_status=st, stream=stream)
    V.varq_quantize_pack(L, data["v"], vp, vm, dev_status=st, stream=stream)
    kd, vd = data["k"], data["v"]  # reused as the dense workspaces (overwritten by unpack+dequant)
    torch.cuda.synchronize()
    T, B, H, D = w.n_tokens, w.batch, w.heads, w.head_dim
    dense_bytes = B * H * T * D * 2
    out = {}
    for lq in w.lq:
        q = data["q"][:, :, :lq].contiguous()
        o = torch.empty_like(q)
        ws_f = V.varq_packed_attention_workspace(L, lq, w.n_blocks)
        wsf = torch.empty(max(ws_f // 4, 1), dtype=torch.float32, device=dev)
        ws_d = V.varq_dense_attention_workspace(B, H, D, lq, T)
        wsd = torch.empty(max(ws_d // 4, 1), dtype=torch.float32, device=dev)

        def fused():
            V.varq_packed_attention(L, q, kp, km, vp, vm, o, workspace=wsf, dev_status=st, stream=stream)

        def unpack():
            V.varq_unpack_dequant(L, kp, km, kd, stream=stream)
            V.varq_unpack_dequant(L, vp, vm, vd, stream=stream)

        def dense():
            V.varq_dense_attention(q, kd, vd, o, workspace=wsd, dev_status=st, stream=stream)

        def unfused():
            unpack()
            dense()
        t_f = _median_ms(fused, stream, iters)
        t_u = _median_ms(unfused, stream, iters)
        t_up = _median_ms(unpack, stream, iters)
        t_d = _median_ms(dense, stream, iters)
        fl = attention_flops(w, lq)
        b_f = attention_bytes(L, w, lq, False)
        # unfused bytes: unpack reads the packed cache and writes dense K, V;
        # the dense attention reads them back (plus Q, O)
        b_up = 2 * (L.packed_bytes + L.meta_bytes + dense_bytes)
        b_d = 2 * B * H * lq * D * 2 + 2 * dense_bytes
        fr_f, bound_f = roofline_frac(fl, b_f, t_f, peaks)
        fr_u, bound_u = roofline_frac(fl, b_up + b_d, t_u, peaks)
        fr_d, bound_d = roofline_frac(fl, b_d, t_d, peaks)
        out[f"lq{lq}"] = {
            "fused_us": 1e3 * t_f, "fused_TFLOP/s": fl / (t_f * 1e-3) / 1e12, "fused_bound": bound_f,
            "fused_frac": fr_f,
            "unfused_us": 1e3 * t_u, "unfused_unpack_us": 1e3 * t_up, "unfused_dense_attention_us": 1e3 * t_d,
            "unfused_frac": fr_u, "unfused_bound": bound_u, "dense_attention_frac": fr_d,
            "dense_attention_bound": bound_d, "fused_speedup": t_u / t_f}
        del q, o, wsf, wsd
    res = {"workload": f"sweep: B={B} H={H} D={D} T={T} blocks={w.n_blocks} INT{bits}; fused = "
                       "varq_packed_attention (AUTO path), unfused = varq_unpack_dequant of K and V into dense bf16 + "
                       "varq_dense_attention; fractions of the binding roofline (burst bf16 peak or HBM) over each "
                       "path's own algorithmic bytes", **out, "device_status": int(st.item())}
    del data, kp, km, vp, vm, kd, vd
    torch.cuda.empty_cache()
    return res


def measure_longlive(dev, stream, peaks, iters=3):
    """LongLive-like long-horizon layer (B4 H12 D128, 40 chunks of 4,680
    tokens = 187,200 cached, pre-RoPE keys rotated after dequantization, one
    4,680-token query block) at INT2, INT3 and INT4: quantize+pack of K and V
    and the fused attention, each against its roofline."""
    from packed_kv_attention_b200 import varq as V
    w = synth.WORKLOADS["longlive"]
    data = synth.make_inputs(w, lq=w.lq[-1], seed=7, device=dev)
    bs = data["block_start"]
    cos, sin = data["rope_cos"], data["rope_sin"]
    rope3d = V.Rope3d.make(1560, 52, synth.rope_axis_pairs(w.head_dim))
    tables = 2 * cos.numel() * cos.element_size()
    lq = w.lq[-1]
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    o = torch.empty_like(data["q"])
    res = {}
    for bits in w.bits:
        L = V.varq_cache_alloc(w.batch, w.heads, w.head_dim, bits, bs)
        kp, km = V.alloc_cache(L, dev)
        vp, vm = V.alloc_cache(L, dev)

        def quant():
            V.varq_quantize_pack(L, data["k"], kp, km, dev_status=st, stream=stream)
            V.varq_quantize_pack(L, data["v"], vp, vm, dev_status=st, stream=stream)

        def attn():
            V.varq_packed_attention(L, data["q"], kp, km, vp, vm, o, rope_cos=cos, rope_sin=sin, dev_status=st,
                                    stream=stream)

        def attn_sched():
            V.varq_packed_attention_rope3d(L, data["q"], kp, km, vp, vm, o, rope3d, dev_status=st, stream=stream)
        t_q = _median_ms(quant, stream, iters)
        t_a = _median_ms(attn, stream, iters)
        t_s = _median_ms(attn_sched, stream, iters)
        fl = attention_flops(w, lq)
        qb = quant_bytes(L, w)
        ab = attention_bytes(L, w, lq, True)
        fr_a, bound = roofline_frac(fl, ab, t_a, peaks)
        res[f"int{bits}"] = {"quant_pack_us": 1e3 * t_q, "quant_pack_GB/s": qb / (t_q * 1e-3) / 1e9,
                             "quant_pack_frac_hbm": qb / (t_q * 1e-3) / 1e9 / peaks["hbm_gbs"],
                             "attention_ms": t_s, "attention_TFLOP/s": fl / (t_s * 1e-3) / 1e12,
                             "attention_bound": bound, "attention_frac": roofline_frac(fl, ab - tables, t_s, peaks)[0],
                             "attention_frac_sustained": fl / (t_s * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"],
                             "tables_attention_ms": t_a, "tables_attention_TFLOP/s": fl / (t_a * 1e-3) / 1e12,
                             "tables_attention_frac": fr_a}
        del kp, km, vp, vm
    res = {"workload": f"longlive: B={w.batch} H={w.heads} D={w.head_dim} T={w.n_tokens} blocks={w.n_blocks} "
                       f"Lq={lq} pre-RoPE keys, 3D rotary schedule computed in the kernel (tables_* = the same "
                       f"angles from [T, D/2] fp32 tables)", **res, "device_status": int(st.item())}
    del data, o
    torch.cuda.empty_cache()
    return res


def measure_var_d16(dev, stream, peaks, iters=20):
    """VAR-d16-like layer as one call each (B1 H16 D64, 10 scales = 680 tokens,
    INT4, the last 256-token block attending to all 680): quantize+pack of K
    and V and the attention, captured once in a CUDA graph and replayed (at
    these sizes the launch costs dominate; the roofline time is below a
    microsecond)."""
    from packed_kv_attention_b200 import varq as V
    w = synth.WORKLOADS["var_d16"]
    pipe = Pipeline(w, 4, w.lq[-1], dev, seed=8)
    torch.cuda.synchronize()

    def step():
        pipe.step(stream)

    def attn():
        V.varq_packed_attention(pipe.L, pipe.q, pipe.kp, pipe.km, pipe.vp, pipe.vm, pipe.out, workspace=pipe.ws,
                                dev_status=pipe.status, stream=stream)
    res = {}
    for name, fn in (("step", step), ("attention", attn)):
        with torch.cuda.stream(stream):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()

        def replay():
            with torch.cuda.stream(stream):
                g.replay()
        t_graph = _median_ms(replay, stream, iters, warm=3)
        t_launch = _median_ms(fn, stream, iters, warm=3)
        res[name] = {"graph_replay_us": 1e3 * t_graph, "stream_launched_us": 1e3 * t_launch}
        del g
    fl = attention_flops(w, w.lq[-1])
    fr, bound = roofline_frac(fl, attention_bytes(pipe.L, w, w.lq[-1], False), res["attention"]["graph_replay_us"] * 1e-3,
                              peaks)
    res["attention"].update({"TFLOP/s": fl / (res["attention"]["graph_replay_us"] * 1e-6) / 1e12, "bound": bound,
                             "frac": fr})
    res["step"]["launches"] = pipe.launches_per_step
    out = {"workload": f"var_d16: B={w.batch} H={w.heads} D={w.head_dim} T={w.n_tokens} blocks={w.n_blocks} "
                       f"Lq={w.lq[-1]} INT4; one step = quantize+pack K, V + attention", **res,
           "device_status": int(pipe.status.item())}
    del pipe
    torch.cuda.empty_cache()
    return out


def config_of(w, args):
    return {"workload": f"{w.name}: B={w.batch} H={w.heads} D={w.head_dim} T={w.n_tokens} "
                        f"blocks={w.n_blocks} Lq={args.lq} INT{args.bits}",
            "global_batch": w.batch, "seq_len": w.n_tokens, "lq": args.lq, "bits": args.bits,
            "parallelism": f"replica x{args.gpus}",
            "l2": "inputs larger than L2 (bf16 K+V of the step exceed 126 MB)"}


def profile_case(name):
    """One small case of one kernel, for an ncu capture (`-k` the kernel,
    `-s` the warm-up launches): inputs above the 126 MB L2 but a few hundred
    MB on the device, three launches of the kernel, then exit."""
    from packed_kv_attention_b200 import varq as V
    dev = torch.device("cuda:0")
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    if name == "attn_sk_sweep_int4_lq16":
        # swap-AB split-KV kernel: a quarter of the sweep cache (B2 H32 T16384 D128), INT4, Lq 16
        w = synth.WORKLOADS["sweep"]
        data = synth.make_inputs(w, lq=16, seed=3, device=dev, batch=2)
        L = V.varq_cache_alloc(2, w.heads, w.head_dim, 4, data["block_start"])
        kp, km = V.alloc_cache(L, dev)
        vp, vm = V.alloc_cache(L, dev)
        V.varq_quantize_pack(L, data["k"], kp, km)
        V.varq_quantize_pack(L, data["v"], vp, vm)
        q = data["q"].contiguous()
        o = torch.empty_like(q)
        ws = torch.empty(max(V.varq_packed_attention_workspace(L, 16, w.n_blocks) // 4, 1), dtype=torch.float32,
                         device=dev)
        torch.cuda.synchronize()
        for _ in range(3):
            V.varq_packed_attention(L, q, kp, km, vp, vm, o, workspace=ws, dev_status=st)
    elif name == "quant_pack_sweep_b1_int4":
        # quantize+pack of one tensor [1, 32, 16384, 128] (128 MiB) in 16 blocks of 1,024 tokens, INT4
        sizes = (1024,) * 16
        g = torch.Generator(device=dev)
        g.manual_seed(0)
        x = synth.kv_cache(g, 1, 32, sizes, 128, 8, 10.0, 80.0, device=dev)
        L = V.varq_cache_alloc(1, 32, 128, 4, synth.block_starts(sizes))
        kp, km = V.alloc_cache(L, dev)
        torch.cuda.synchronize()
        for _ in range(3):
            V.varq_quantize_pack(L, x, kp, km, dev_status=st)
    elif name == "attn_tc2_self_forcing_b2_schedule":
        # paired-CTA kernel, pre-RoPE keys rotated from the 3D schedule: two of the twelve
        # sequences of the Self-Forcing-like layer (B2 H12 T32760 D128, Lq 4680), INT4
        w = synth.WORKLOADS["self_forcing"]
        data = synth.make_inputs(w, lq=w.lq[-1], seed=4, device=dev, batch=2)
        L = V.varq_cache_alloc(2, w.heads, w.head_dim, 4, data["block_start"])
        kp, km = V.alloc_cache(L, dev)
        vp, vm = V.alloc_cache(L, dev)
        V.varq_quantize_pack(L, data["k"], kp, km)
        V.varq_quantize_pack(L, data["v"], vp, vm)
        o = torch.empty_like(data["q"])
        rope = V.Rope3d.make(1560, 52, synth.rope_axis_pairs(w.head_dim))
        torch.cuda.synchronize()
        for _ in range(3):
            V.varq_packed_attention_rope3d(L, data["q"], kp, km, vp, vm, o, rope, dev_status=st)
    elif name == "unpack_dequant_sweep_b1_int4":
        # standalone unpack+dequant of one packed tensor [1, 32, 16384, 128] to bf16, INT4
        sizes = (1024,) * 16
        g = torch.Generator(device=dev)
        g.manual_seed(0)
        x = synth.kv_cache(g, 1, 32, sizes, 128, 8, 10.0, 80.0, device=dev)
        L = V.varq_cache_alloc(1, 32, 128, 4, synth.block_starts(sizes))
        kp, km = V.alloc_cache(L, dev)
        V.varq_quantize_pack(L, x, kp, km, dev_status=st)
        out = torch.empty_like(x)
        torch.cuda.synchronize()
        for _ in range(3):
            V.varq_unpack_dequant(L, kp, km, out)
    elif name in ("attn_decode_sweep_int4_lq1", "attn_decode_sweep_int4_lq4"):
        # CUDA-core split-KV decode (one row, or four rows per CTA): a quarter of the
        # sweep cache (B2 H32 T16384 D128), INT4, Lq 1 or 4
        lq = int(name[-1])
        w = synth.WORKLOADS["sweep"]
        data = synth.make_inputs(w, lq=lq, seed=3, device=dev, batch=2)
        L = V.varq_cache_alloc(2, w.heads, w.head_dim, 4, data["block_start"])
        kp, km = V.alloc_cache(L, dev)
        vp, vm = V.alloc_cache(L, dev)
        V.varq_quantize_pack(L, data["k"], kp, km)
        V.varq_quantize_pack(L, data["v"], vp, vm)
        q = data["q"].contiguous()
        o = torch.empty_like(q)
        ws = torch.empty(max(V.varq_packed_attention_workspace(L, lq, w.n_blocks) // 4, 1), dtype=torch.float32,
                         device=dev)
        torch.cuda.synchronize()
        for _ in range(3):
            V.varq_packed_attention(L, q, kp, km, vp, vm, o, workspace=ws, dev_status=st)
    else:
        raise SystemExit(f"unknown profile case {name}")
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": name, "device_status": int(st.item())}))


PROFILE_CASES = ("attn_sk_sweep_int4_lq16", "quant_pack_sweep_b1_int4", "attn_tc2_self_forcing_b2_schedule",
                 "unpack_dequant_sweep_b1_int4", "attn_decode_sweep_int4_lq1", "attn_decode_sweep_int4_lq4")


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="infinity_8b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--bits", type=int, default=4)
    ap.add_argument("--also-bits", type=int, default=2, help="second bit width reported under 'also' (0: none)")
    ap.add_argument("--lq", type=int, default=0, help="query block length (default: the workload's)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--oracle-rows", type=int, default=256)
    ap.add_argument("--oracle-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row measurements (unpack, split-KV, pre-RoPE)")
    ap.add_argument("--profile-case", choices=PROFILE_CASES,
                    help="run one small case of one kernel for an ncu capture, then exit (no JSON line)")
    args = ap.parse_args(argv)
    if args.profile_case:
        profile_case(args.profile_case)
        return
    w = synth.WORKLOADS[args.workload]
    if args.lq <= 0:
        args.lq = w.lq[-1]
    args.warmup = max(args.warmup, 3) if args.impl == "ours" else args.warmup

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, w, rank, world)

    dist_ok = world > 1
    if dist_ok:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    peaks = load_peaks()

    def measure(bits):
        pipe = Pipeline(w, bits, args.lq, dev)
        torch.cuda.synchronize()
        sampler = ClockSampler(local)
        sampler.start()
        total_ms, qp, at = time_ours(pipe, args.steps, args.warmup, stream, dist_ok)
        clocks = sampler.stop()
        total_ms = max_over_ranks(total_ms, dev, dist_ok)
        st = int(pipe.status.item())
        return pipe, total_ms, qp, at, clocks, st

    pipe, total_ms, qp, at, clocks, st = measure(args.bits)
    flops = attention_flops(w, args.lq)
    ms = total_ms / args.steps
    value = job_tflops(world, flops, args.steps, total_ms)
    at_avg = statistics.mean(at)
    qp_avg = statistics.mean(qp)
    att_tflops = flops / (at_avg * 1e-3) / 1e12
    qbytes = quant_bytes(pipe.L, w)
    qp_gbs = qbytes / (qp_avg * 1e-3) / 1e9
    abytes = attention_bytes(pipe.L, w, args.lq, pipe.cos is not None)
    # the timed region lasts tens of milliseconds at full clocks: the burst bf16
    # peak is the denominator, the sustained one is reported beside it
    tensor_peak = peaks["bf16_tflops"]
    tensor_peak_sus = peaks["bf16_tflops_sustained"]
    hbm_peak = peaks["hbm_gbs"]
    roof_time = max(flops / (tensor_peak * 1e12), abytes / (hbm_peak * 1e9))
    bound = "tensor" if flops / (tensor_peak * 1e12) >= abytes / (hbm_peak * 1e9) else "hbm"
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 MMA / fp32 accumulate; int codes", "data": "synthetic",
        "config": config_of(w, args),
        "gpu_launches": pipe.launches_per_step * args.steps,
        "device_status": st,
        "components": {
            "quant_pack": {"us": 1e3 * qp_avg, "GB/s": qp_gbs, "algorithmic_bytes": qbytes,
                           "frac_hbm": qp_gbs / hbm_peak, "peak_GB/s": hbm_peak},
            "attention": {"us": 1e3 * at_avg, "TFLOP/s": att_tflops, "flops": flops,
                          "algorithmic_bytes": abytes, "bound": bound,
                          "frac_of_binding_roofline": roof_time / (at_avg * 1e-3)},
        },
        "roofline": {"kernel": "attn_tc_kernel (fused packed-KV attention)", "bound": bound,
                     "achieved": att_tflops if bound == "tensor" else abytes / (at_avg * 1e-3) / 1e9,
                     "peak": tensor_peak if bound == "tensor" else hbm_peak,
                     "unit": "TFLOP/s" if bound == "tensor" else "GB/s",
                     "frac": (att_tflops / tensor_peak) if bound == "tensor" else
                     (abytes / (at_avg * 1e-3) / 1e9) / hbm_peak,
                     "peak_source": f"{peaks['source']} ({'bf16_tflops (burst)' if bound == 'tensor' else 'hbm_gbs'})",
                     "frac_of_sustained_peak": (att_tflops / tensor_peak_sus) if bound == "tensor" else None,
                     "traffic": measured_traffic(w, args.bits, args.lq, pipe.cos is not None),
                     "traffic_unit": "bytes per launch (ncu dram read + write)"},
        "clocks": clocks,
    }
    if args.also_bits and args.also_bits != args.bits:
        del pipe
        torch.cuda.empty_cache()
        p2, tot2, qp2, at2, clk2, st2 = measure(args.also_bits)
        line["also"] = {
            "bits": args.also_bits, "value": job_tflops(world, flops, args.steps, tot2),
            "ms_per_step": tot2 / args.steps, "device_status": st2,
            "quant_pack_GB/s": quant_bytes(p2.L, w) / (statistics.mean(qp2) * 1e-3) / 1e9,
            "attention_TFLOP/s": flops / (statistics.mean(at2) * 1e-3) / 1e12,
            "clocks": clk2}
        line["also"]["quant_pack_frac_hbm"] = line["also"]["quant_pack_GB/s"] / hbm_peak
        line["also"]["attention_frac_tensor"] = line["also"]["attention_TFLOP/s"] / tensor_peak
        del p2
        torch.cuda.empty_cache()
        pipe = Pipeline(w, args.bits, args.lq, dev)
    if not args.no_rows and world == 1:
        del pipe
        torch.cuda.empty_cache()
        line["rows"] = measure_rows(dev, stream, peaks)
        line["rows"]["c5_fused_vs_unfused"] = measure_fused_vs_unfused(dev, stream, peaks)
        line["rows"]["c4_longlive"] = measure_longlive(dev, stream, peaks)
        line["rows"]["c1_var_d16"] = measure_var_d16(dev, stream, peaks)
        pipe = Pipeline(w, args.bits, args.lq, dev)
    if not args.no_e2e:
        e2e_ms, h2d, d2h, same = time_e2e(pipe, max(4, args.steps), 2, stream)
        e2e_ms = max_over_ranks(e2e_ms, dev, dist_ok)  # every rank runs this section
        line["e2e"] = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                       "copies": "own streams, overlapping the neighbouring steps' kernels (two buffer sets)",
                       "output_equals_device_step": same}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # repeat the bounded sample (fresh seeds) for about ten seconds of CPU work
        dt_tot, fl_tot, reps, desc = 0.0, 0.0, 0, ""
        while dt_tot < args.oracle_seconds and reps < 256:
            dt, sflops, desc = oracle_sample(w, args.bits, args.lq, args.oracle_rows, seed=reps)
            dt_tot += dt
            fl_tot += sflops
            reps += 1
        line["cpu_baseline"] = {"value": fl_tot / dt_tot / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(),
                                "kind": "oracle", "sample": f"{reps} x [{desc}]", "seconds": dt_tot,
                                "threads": "numpy BLAS (the fp64 attention products) on every core of the "
                                           "process's affinity set; the quantize/pack/dequant steps are "
                                           "single-threaded numpy"}
    if dist_ok:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
