"""Benchmark: quantized-KV decode attention on the long-context workload.

One *step* = one serving decode step of the hot path on one request's cache:
rq_decode_step = rq_append_token (the new token enters the bf16 window) +
rq_decode_attention (split-K over the packed tiles plus the bf16 window,
fused combine), one kernel launch per step; the launch of the step before a
tile flush also quantizes and packs that tile (every 32nd step).  The
per-head bit allocation (host) and the bulk prefill quantize run before the
timed loop and are reported separately (alloc_ms, quantize_gbs).

Workload: long_128k -- batch 1, 32 query / 8 kv heads, head_dim 128, 131072
tokens, K outlier channels lognormal(1.5), 2-bit average over {2,3,4}.  Four
independent caches (405 MB of packed data) are decoded round-robin so that a
step never finds its cache in the 126 MB L2.

value = algorithmic bytes of the K steps / device time of the K steps (GB/s),
summed over ranks and divided by the slowest rank's time.  Algorithmic bytes
per decode: packed codes + scale/zero of every tile, bf16 sink + recent
window, q and the fp32 output; per append: the new bf16 K/V rows (and the
flushed tile: 32 bf16 rows read, one record written).

--impl reference runs the CPU oracle (numpy, fp64 attention) on a bounded
sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantized-KV decode attention: effective HBM GB/s & µs/step; quantize GB/s"
WORKLOAD = "long_128k"
L2_BYTES = 126_000_000


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# --------------------------------------------------------------- byte counts
def split_lengths(T, n_sink, n_recent):
    """(sink, quantized, recent) token counts of a stream of T tokens: tiles of
    32 are quantized once more than n_recent tokens follow the sink."""
    s = min(T, n_sink)
    tq = ((T - n_sink - n_recent) // 32) * 32 if T >= n_sink + n_recent else 0
    return s, tq, T - s - tq


def decode_bytes(wl, rec, T):
    """Algorithmic bytes of one decode over a cache of T tokens (all streams);
    rec[l][h] = bytes of one packed 32-token tile record of (layer, kv-head)."""
    s, tq, r = split_lengths(T, wl.n_sink, wl.n_recent)
    n_tiles = tq // 32
    D, G = wl.head_dim, wl.group
    total = 0
    for l in range(wl.n_layers):
        for h in range(wl.n_kv_heads):
            per_stream = n_tiles * int(rec[l][h])
            per_stream += (s + r) * D * 2 * 2 + G * D * 2 + G * D * 4
            total += per_stream * wl.batch
    return total


def arm_config(wl, nc, splits, world):
    """The workload description both arms print (same keys and values)."""
    cpw = 16  # 2-bit codes per 32-bit word (every long-context head is at 2 bits)
    rec = 2 * (-(-wl.head_dim // cpw) * 128) + 8 * wl.head_dim
    per_cache = decode_bytes(wl, [[rec] * wl.n_kv_heads] * wl.n_layers, wl.context)
    return {"workload": WORKLOAD, "batch": wl.batch, "q_heads": wl.n_q_heads, "kv_heads": wl.n_kv_heads,
            "head_dim": wl.head_dim, "context": wl.context, "bits": "K=V=2 on every head (avg 2 over {2,3,4})",
            "splits": splits or "auto",
            "l2": f"{nc} caches decoded round-robin ({nc * per_cache / 1e6:.0f} MB > 126 MB L2)",
            "parallelism": f"replicas x{world}"}


def append_bytes(wl, rec, T_old):
    D = wl.head_dim
    s, tq, r = split_lengths(T_old, wl.n_sink, wl.n_recent)
    flush = T_old >= wl.n_sink and r + 1 == wl.n_recent + 32
    total = 0
    for l in range(wl.n_layers):
        for h in range(wl.n_kv_heads):
            b = 2 * D * 2 * 2  # read new rows, write them to the ring
            if flush:
                b += 32 * D * 2 * 2 + int(rec[l][h])
            total += b * wl.batch
    return total


# ------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"rq_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, _, flags in rows:
            for n, fl in zip(names, flags):
                if fl.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# ----------------------------------------------------------------- oracle arm
def oracle_sample(wl, seconds=12.0):
    """Time the CPU oracle on a bounded sample: one kv-head stream of the
    workload (its full context), one decode step.  Returns a dict."""
    import torch

    from oracle import attention as at
    from oracle import cache as ca
    from oracle import quantize as qz
    from quantized_decode_attention_head_b200 import workloads

    try:
        from threadpoolctl import threadpool_info, threadpool_limits

        threadpool_limits(os.cpu_count())
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = 1
    one = wl.with_(n_layers=1, batch=1, n_kv_heads=1, n_q_heads=wl.group)
    k, v, f = workloads.kv_inputs(one, "cpu")
    q, _, _ = workloads.step_inputs(one, 1, f, "cpu")
    to32 = lambda t: qz.bf16_bits_to_f32(t.contiguous().view(torch.int16).numpy().view(np.uint16))
    kn, vn, qn = to32(k)[0, 0, 0], to32(v)[0, 0, 0], to32(q)[0, 0, 0].astype(np.float64)
    st = ca.StreamCache(wl.head_dim, 2, 2, wl.n_sink, wl.n_recent)
    t0 = time.perf_counter()
    st.prefill(kn, vn)
    t_quant = time.perf_counter() - t0
    runs, t0 = 0, time.perf_counter()
    while True:
        kh, vh = st.dequantized()
        at.attend(qn, kh, vh)
        runs += 1
        if time.perf_counter() - t0 >= seconds:
            break
    t_dec = (time.perf_counter() - t0) / runs
    rec = [[qz.record_bytes(2, 2, wl.head_dim)]]
    bytes_dec = decode_bytes(one, rec, wl.context)
    bytes_q = wl.context * wl.head_dim * 2 * 2 + bytes_dec
    return {
        "decode_gbs": bytes_dec / t_dec / 1e9,
        "decode_s": t_dec,
        "quantize_gbs": bytes_q / t_quant / 1e9,
        "threads": threads,
        "sample": f"one of {wl.n_kv_heads} kv-head streams of {WORKLOAD} ({wl.context} tokens, {wl.group} query "
                  f"heads, 2-bit K/V), one decode step (dequantize + fp64 attention), {runs} runs",
    }


def host_cpu():
    """CPU model name (lscpu), logical cores and the BLAS thread count the
    oracle runs with (pinned to every host core)."""
    model = None
    try:
        out = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for line in out.splitlines():
            if line.lower().startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except Exception:
        pass
    threads = 1
    try:
        from threadpoolctl import threadpool_info, threadpool_limits

        threadpool_limits(os.cpu_count())
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        pass
    return {"model": model, "cores": os.cpu_count(), "blas_threads": threads}


# streams of each workload the oracle runs (None: every stream of the cache)
ORACLE_STREAMS = {"tiny": None, "llama3_8b": None, "long_128k": 2, "qwen3_8b": 8, "mistral_7b_b64": 2}


def oracle_configs():
    """The CPU oracle on every benchmark workload: quantize + pack of the
    prefill (the cache's bytes) and one decode step (dequantize + fp64
    attention), per stream, summed over the streams run.  Workloads whose
    stream count is given in ORACLE_STREAMS run that many streams (the first
    ones) and are extrapolated linearly to the whole cache, labelled so."""
    import torch

    from oracle import attention as at
    from oracle import cache as ca
    from oracle import quantize as qz
    from quantized_decode_attention_head_b200 import workloads

    to32 = lambda t: qz.bf16_bits_to_f32(t.contiguous().view(torch.int16).numpy().view(np.uint16))
    res = {}
    for name, n_run in ORACLE_STREAMS.items():
        wl = workloads.CONFIGS[name]
        kb, vb = workload_bits_oracle(wl)
        n_all = wl.n_layers * wl.batch * wl.n_kv_heads
        keys = [(l, b, h) for l in range(wl.n_layers) for b in range(wl.batch) for h in range(wl.n_kv_heads)]
        keys = keys[: (n_all if n_run is None else n_run)]
        t_q = t_d = 0.0
        q_bytes = d_bytes = 0
        for (l, b, h) in keys:
            one = wl.with_(n_layers=1, batch=1, n_kv_heads=1, n_q_heads=wl.group)
            k, v, f = workloads.kv_inputs(one, "cpu", seed=wl.seed + 7919 * (1 + l * 977 + b * 31 + h))
            q, _, _ = workloads.step_inputs(one, 1, f, "cpu", seed=wl.seed + 7919 * (1 + l * 977 + b * 31 + h))
            kn, vn, qn = to32(k)[0, 0, 0], to32(v)[0, 0, 0], to32(q)[0, 0, 0].astype(np.float64)
            st = ca.StreamCache(wl.head_dim, int(kb[l, h]), int(vb[l, h]), wl.n_sink, wl.n_recent)
            t0 = time.perf_counter()
            st.prefill(kn, vn)
            st.records()
            t1 = time.perf_counter()
            kh, vh = st.dequantized()
            at.attend(qn, kh, vh)
            t2 = time.perf_counter()
            t_q += t1 - t0
            t_d += t2 - t1
            rec = [[qz.record_bytes(int(kb[l, h]), int(vb[l, h]), wl.head_dim)]]
            db = decode_bytes(one, rec, wl.context)
            d_bytes += db
            q_bytes += wl.context * wl.head_dim * 2 * 2 + db
        scale = n_all / len(keys)
        res[name] = {
            "streams_run": len(keys), "streams": n_all,
            "extrapolated": len(keys) < n_all,
            "quantize_s": t_q * scale, "quantize_gbs": q_bytes / t_q / 1e9,
            "decode_s": t_d * scale, "decode_gbs": d_bytes / t_d / 1e9,
        }
    return res


def workload_bits_oracle(wl):
    """Per-(layer, kv-head) K and V bit widths from the oracle's allocator."""
    from oracle import allocation as al
    from quantized_decode_attention_head_b200 import workloads

    inp = workloads.allocation_inputs(wl)
    shape = (wl.n_layers, wl.n_kv_heads)
    if "kv" in inp:
        b = al.allocate(*inp["kv"], wl.allowed)["b_int"].reshape(shape)
        return b, b
    return tuple(al.allocate(*inp[key], wl.allowed)["b_int"].reshape(shape) for key in ("k", "v"))


def run_reference(args):
    from quantized_decode_attention_head_b200 import workloads

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = workloads.CONFIGS[WORKLOAD]
    res = oracle_sample(wl, seconds=args.cpu_seconds)
    cb = {"value": res["decode_gbs"], "unit": "GB/s", "cores": res["threads"], "kind": "oracle",
          "sample": res["sample"]}
    line = {
        "impl": "reference", "metric": METRIC, "value": res["decode_gbs"], "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["decode_s"] * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(wl, args.copies, args.splits, args.gpus),
        "cpu_baseline": cb,
        "e2e": {"value": res["decode_gbs"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def allocator_timings(repeats=5):
    """Host allocator (rq_allocate_bits) at the pages' scale: the Qwen3-8B
    workload's 288 (layer, kv-head) units for its K and V budgets (allowed set
    {2, 3, 4, 8}: exact DP), the same 288 units over the contiguous set
    {2, 3, 4} (greedy max-heap), and the long-context workload's 8 heads.
    Best of `repeats` calls, milliseconds."""
    from quantized_decode_attention_head_b200 import rq_allocate_bits, workloads

    def best(*a):
        t = []
        for _ in range(repeats):
            t0 = time.perf_counter()
            rq_allocate_bits(*a)
            t.append(time.perf_counter() - t0)
        return min(t) * 1e3

    qw = workloads.CONFIGS["qwen3_8b"]
    inp = workloads.allocation_inputs(qw)
    wk, ak, bk, avk = inp["k"]
    wv, av, bv, avv = inp["v"]
    lw = workloads.CONFIGS[WORKLOAD]
    return {
        "qwen3_8b_k_288_units_dp_ms": best(wk, ak, bk, avk, qw.allowed),
        "qwen3_8b_v_288_units_dp_ms": best(wv, av, bv, avv, qw.allowed),
        "qwen3_8b_k_288_units_greedy_234_ms": best(wk, ak, bk, avk, (2, 3, 4)),
        "long_128k_8_heads_ms": best(*workloads.allocation_inputs(lw)["kv"], lw.allowed),
        "context": "RateQuant §3.3 quotes under 10 ms for Qwen3-8B's 288 KV heads (hardware not stated)",
    }


# ------------------------------------------------------ secondary measurements
def workload_bits(wl):
    """Per-(layer, kv-head) K and V bit widths of a workload from the host
    allocation (one shared budget, or separate K and V budgets)."""
    from quantized_decode_attention_head_b200 import rq_allocate_bits, workloads

    inp = workloads.allocation_inputs(wl)
    shape = (wl.n_layers, wl.n_kv_heads)
    if "kv" in inp:
        w, a, b, avg = inp["kv"]
        kb = rq_allocate_bits(w, a, b, avg, wl.allowed)["b_int"].reshape(shape)
        return kb, kb
    return tuple(rq_allocate_bits(*inp[key], wl.allowed)["b_int"].reshape(shape) for key in ("k", "v"))


def _bits_text(kb, vb):
    cnt = lambda x: ",".join(f"{b}:{int((x == b).sum())}" for b in sorted(set(x.ravel().tolist())))
    return f"K {{{cnt(kb)}}} V {{{cnt(vb)}}} heads per bit width"


def sweep_workloads(names, peak, launches=20):
    """Prefill quantize and one decode of every layer in one launch
    (rq_decode_attention, layer -1) on other benchmark caches.  A cache
    smaller than twice the 126 MB L2 is decoded round-robin over enough
    copies to span twice the L2.  Device time by CUDA events around `launches`
    back-to-back launches after 3 warm-up launches."""
    import torch

    from quantized_decode_attention_head_b200 import QuantizedKVCache, workloads

    res = {}
    stream = torch.cuda.current_stream()
    for name in names:
        try:
            wl = workloads.CONFIGS[name]
            kb, vb = workload_bits(wl)
            caches, qs, qtime, qbytes = [], [], None, 0
            ncopy = 1
            c = 0
            while c < ncopy:
                k, v, f = workloads.kv_inputs(wl, "cuda", seed=wl.seed + 100 * c)
                cache = QuantizedKVCache(wl.n_layers, wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                                         wl.n_sink, wl.n_recent, wl.context + 64, kb, vb)
                cache.rq_quantize_kv(k, v)  # first call pays one-time set-up
                torch.cuda.synchronize()
                if c == 0:
                    rec = [[cache.stream_layout(l, 0, h)["record_bytes"] for h in range(wl.n_kv_heads)]
                           for l in range(wl.n_layers)]
                    dbytes = decode_bytes(wl, rec, wl.context)
                    ncopy = max(1, -(-2 * L2_BYTES // dbytes))  # the copies span twice the L2
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    cache.rq_quantize_kv(k, v)
                    e1.record(stream)
                    torch.cuda.synchronize()
                    qtime = e0.elapsed_time(e1) / 1e3
                    qbytes = k.numel() * 2 * 2 + dbytes
                del k, v
                q = workloads.step_inputs(wl, 1, f, "cuda", seed=wl.seed + 100 * c)[0][0].contiguous()
                caches.append(cache)
                qs.append(q)
                c += 1
            ws = caches[0].make_workspace()
            out = torch.empty(qs[0].shape, dtype=torch.float32, device="cuda")
            for i in range(3):
                caches[i % ncopy].rq_decode_attention(-1, qs[i % ncopy], out=out, workspace=ws)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(launches):
                caches[i % ncopy].rq_decode_attention(-1, qs[i % ncopy], out=out, workspace=ws)
            e1.record(stream)
            torch.cuda.synchronize()
            if QuantizedKVCache.rq_decode_read_status(ws) != 0:
                raise RuntimeError("device status")
            t = e0.elapsed_time(e1) / 1e3 / launches
            # frac: of the copy peak (a read-mostly stream can exceed a copy's
            # bandwidth, so a value a little above 1 is possible); also of the
            # nominal 8 TB/s
            res[name] = {"decode_us": t * 1e6, "decode_gbs": dbytes / t / 1e9, "frac": dbytes / t / 1e9 / peak,
                         "frac_of_nominal_8000_gbs": dbytes / t / 1e9 / 8000.0,
                         "bytes_per_launch": dbytes, "streams": wl.n_layers * wl.batch * wl.n_kv_heads,
                         "context": wl.context, "copies": ncopy, "bits": _bits_text(kb, vb),
                         "quantize_gbs": qbytes / qtime / 1e9}
            del caches, qs, ws, out
            torch.cuda.empty_cache()
        except Exception as exc:  # a secondary figure never hides the main line
            res[name] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    return res


def step_loop_graph(steps=64, copies=4, replays=20):
    """The Llama-3-8B-shaped workload's decode loop -- `steps` serving steps
    (rq_decode_step: append + decode) over `copies` caches round-robin --
    timed per step as eager launches and as one CUDA graph of the whole loop.
    The graph is captured on a second, identical set of caches; its first
    replay performs the same steps on the same data, so its outputs must equal
    the eager loop's bit for bit.  Later replays repeat the captured steps
    (same lengths, same slots) and time the loop."""
    import torch

    from quantized_decode_attention_head_b200 import QuantizedKVCache, workloads

    wl = workloads.CONFIGS["llama3_8b"]
    kb, vb = workload_bits(wl)
    per = -(-steps // copies)
    stream = torch.cuda.current_stream()

    def make_set():
        cs, ins = [], []
        for c in range(copies):
            k, v, f = workloads.kv_inputs(wl, "cuda", seed=wl.seed + 100 * c)
            cache = QuantizedKVCache(wl.n_layers, wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n_sink,
                                     wl.n_recent, wl.context + per + 32, kb, vb)
            cache.rq_quantize_kv(k, v)
            del k, v
            cs.append(cache)
            ins.append(workloads.step_inputs(wl, per, f, "cuda", seed=wl.seed + 100 * c))
        return cs, ins

    shape = (wl.batch, wl.n_q_heads, wl.head_dim)
    eager_set, ins = make_set()
    graph_set, _ = make_set()
    ws_e, ws_g = eager_set[0].make_workspace(), graph_set[0].make_workspace()
    out_e = torch.empty((steps,) + shape, dtype=torch.float32, device="cuda")
    out_g = torch.empty_like(out_e)
    # one decode without append on every cache: one-time host set-up outside the loops
    for cs, ws in ((eager_set, ws_e), (graph_set, ws_g)):
        for c in range(copies):
            cs[c].rq_decode_attention(0, ins[c][0][0, 0], out=out_e[0], workspace=ws)
    torch.cuda.synchronize()

    def loop(cs, ws, out):
        for i in range(steps):
            c, j = i % copies, i // copies
            q, kn, vn = ins[c]
            cs[c].rq_decode_step(0, q[j, 0], kn[j, 0], vn[j, 0], out=out[i], workspace=ws)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    loop(eager_set, ws_e, out_e)
    e1.record(stream)
    torch.cuda.synchronize()
    eager_us = e0.elapsed_time(e1) * 1e3 / steps
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        loop(graph_set, ws_g, out_g)
    g.replay()
    torch.cuda.synchronize()
    same = bool(torch.equal(out_e, out_g))
    g.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(replays):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    graph_us = e0.elapsed_time(e1) * 1e3 / (steps * replays)
    st = (QuantizedKVCache.rq_decode_read_status(ws_e), QuantizedKVCache.rq_decode_read_status(ws_g))
    del g
    return {"steps": steps, "copies": copies, "eager_us_per_step": eager_us, "graph_us_per_step": graph_us,
            "graph_equals_eager": same, "device_status": list(st), "bits": _bits_text(kb, vb),
            "note": "eager: one timed pass of the loop (first use of each length); graph: mean of "
                    f"{replays} replays"}


# ------------------------------------------------------------------ GPU arm
def aggregate_ranks(elapsed, step_bytes, e2e_elapsed, e2e_bytes, world, device):
    """Whole-job figures of the replicas: bytes summed over ranks, time of the
    slowest rank (both the device-timed loop and the end-to-end loop)."""
    if world <= 1:
        return elapsed, step_bytes, e2e_elapsed, e2e_bytes
    import torch
    import torch.distributed as dist

    vals = torch.tensor([elapsed, step_bytes, e2e_elapsed, e2e_bytes], dtype=torch.float64, device=device)
    mx = vals.clone()
    dist.all_reduce(mx, op=dist.ReduceOp.MAX)
    sm = vals.clone()
    dist.all_reduce(sm, op=dist.ReduceOp.SUM)
    return mx[0].item(), sm[1].item(), mx[2].item(), sm[3].item()


def upload_graph(graph, stream):
    """Uploads an instantiated CUDA graph to the device (cuGraphUpload) ahead
    of its first replay, which would otherwise carry the upload inside the
    timed region; no node of the graph runs.  Returns whether it succeeded."""
    import ctypes

    try:
        drv = ctypes.CDLL("libcuda.so.1")
        rc = drv.cuGraphUpload(ctypes.c_void_p(graph.raw_cuda_graph_exec()), ctypes.c_void_p(stream.cuda_stream))
    except (OSError, AttributeError, RuntimeError):
        return False
    return rc == 0


def traffic_record():
    """ncu DRAM traffic of the decode kernel recorded for the current sources."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path))
    h = hashlib.sha256()
    for name in ("rq_decode.cuh", "rq_device.cuh", "rq_internal.h", "rq_pack.cuh"):
        h.update(open(os.path.join(ROOT, "quantized_decode_attention_head_b200", "csrc", name), "rb").read())
    if rec.get("source_sha256") != h.hexdigest():
        return None
    return rec


def run_gpu(args):
    import torch
    import torch.distributed as dist

    from quantized_decode_attention_head_b200 import QuantizedKVCache, rq_allocate_bits, workloads

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    wl = workloads.CONFIGS[WORKLOAD]
    NC = args.copies

    # a1: allocation (host)
    w, a, b, avg = workloads.allocation_inputs(wl)["kv"]
    t0 = time.perf_counter()
    alloc = rq_allocate_bits(w, a, b, avg, wl.allowed)
    alloc_ms = (time.perf_counter() - t0) * 1e3
    kb = alloc["b_int"].reshape(wl.n_layers, wl.n_kv_heads)

    # Step budget per cache copy (steps go round-robin over the copies):
    # warm-up, the K timed steps (one CUDA graph), the same K steps launched
    # eagerly (host submit time), the isolated launches of the per-launch
    # statistics, and the end-to-end loop.
    n_launch_stats = 20 + args.launch_stats
    total_steps = args.warmup + args.steps
    e2e_steps = args.steps
    j_eager = (total_steps + NC - 1) // NC
    j_stats = j_eager + (args.steps + NC - 1) // NC
    j0 = j_stats + (n_launch_stats + NC - 1) // NC  # first per-copy step index of the e2e loop
    steps_per_copy = j0 + (e2e_steps + NC - 1) // NC + 1
    max_tokens = wl.context + steps_per_copy + 32
    caches, step_in = [], []
    qbytes, qtimes = 0, []
    stream = torch.cuda.current_stream()
    for c in range(NC):
        seed = wl.seed + 1000 * rank + c
        k, v, f = workloads.kv_inputs(wl, "cuda", seed=seed)
        cache = QuantizedKVCache(wl.n_layers, wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n_sink,
                                 wl.n_recent, max_tokens, kb, kb)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        cache.rq_quantize_kv(k, v)
        e1.record(stream)
        torch.cuda.synchronize()
        if c > 0:  # the first call pays one-time set-up
            qtimes.append(e0.elapsed_time(e1) / 1e3)
            qbytes = k.numel() * 2 * 2 + decode_bytes(wl, rec, wl.context)
        del k, v
        q, kn, vn = workloads.step_inputs(wl, steps_per_copy, f, "cuda", seed=seed)
        caches.append(cache)
        step_in.append((q, kn, vn))
        if c == 0:  # packed record size of every (layer, kv-head), from the library's own layout
            rec = [[cache.stream_layout(l, 0, h)["record_bytes"] for h in range(wl.n_kv_heads)]
                   for l in range(wl.n_layers)]
    ws = caches[0].make_workspace(n_splits=args.splits)
    outs = [torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=torch.float32, device="cuda") for _ in range(NC)]
    torch.cuda.synchronize()
    step_rows = {}  # (copy, per-copy index) -> the step's q, k_new, v_new views (made once, outside timing)

    def rows(c, j):
        key = (c, j)
        if key not in step_rows:
            q, kn, vn = step_in[c]
            step_rows[key] = (q[j, 0], kn[j, 0], vn[j, 0])
        return step_rows[key]

    def do_step(i, j_base=0):
        c = i % NC
        j = j_base + i // NC
        q, kn, vn = rows(c, j)
        # append + decode: one fused launch, two when the append completes a tile
        caches[c].rq_decode_step(0, q, kn, vn, out=outs[c], n_splits=args.splits, workspace=ws)

    def bytes_of(i_from, n, base_len):
        """Algorithmic bytes of n round-robin steps starting at step i_from,
        from each copy's length base_len[c] before them; also the number of
        two-launch steps (a flush that was not packed ahead: the first step
        of a copy after its prefill)."""
        tot, two_n = 0, 0
        for i in range(i_from, i_from + n):
            c = i % NC
            T_old = base_len[c] + (i - i_from) // NC
            tot += append_bytes(wl, rec, T_old) + decode_bytes(wl, rec, T_old + 1)
            flush = (split_lengths(T_old + 1, wl.n_sink, wl.n_recent)[1] !=
                     split_lengths(T_old, wl.n_sink, wl.n_recent)[1])
            two_n += flush and (T_old == wl.context or wl.n_recent < 2)
        return tot, two_n

    for i in range(args.warmup):
        do_step(i)
    torch.cuda.synchronize()
    base_len = [caches[c].length(0) for c in range(NC)]
    step_bytes, n_flush = bytes_of(args.warmup, args.steps, base_len)
    for i in range(args.warmup, total_steps):  # the step views exist before capture
        rows(i % NC, i // NC)
    # The K timed steps are captured as one CUDA graph and replayed once: the
    # replay performs exactly those K steps (the host-side length bookkeeping
    # advanced during the capture), back to back, with no host gaps between
    # launches.  A short sleep kernel keeps the GPU busy while the host submits
    # the replay, so the start event is not stamped before the work arrives.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(args.warmup, total_steps):
            do_step(i)
    torch.cuda.synchronize()
    uploaded = upload_graph(graph, stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        torch.cuda.synchronize()
        torch.cuda._sleep(2_000_000)
        start.record(stream)
        graph.replay()
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    elapsed = start.elapsed_time(end) / 1e3
    # The same K steps again, five more timed replays: the graph's arguments
    # (lengths, slots) are those of the capture, so each replay rewrites the
    # same appended rows and packed tile and performs identical work; their
    # spread is the run-to-run spread of the timed region.
    rep_us = []
    for _ in range(5):
        torch.cuda._sleep(2_000_000)
        start.record(stream)
        graph.replay()
        end.record(stream)
        torch.cuda.synchronize()
        rep_us.append(start.elapsed_time(end) * 1e3 / args.steps)
    rep_us.sort()
    repeats = {"n": len(rep_us), "median_us_per_step": rep_us[len(rep_us) // 2], "p10_us_per_step": rep_us[0],
               "p90_us_per_step": rep_us[-1], "note": "five more replays of the timed graph (min and max as p10 / p90)"}
    del graph
    status = QuantizedKVCache.rq_decode_read_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status}")

    # the same number of steps launched eagerly through the Python binding:
    # device time and the host's submit time per step
    base_len = [caches[c].length(0) for c in range(NC)]
    eager_bytes, _ = bytes_of(0, args.steps, base_len)
    for i in range(args.steps):
        rows(i % NC, j_eager + i // NC)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h0 = time.perf_counter()
    for i in range(args.steps):
        do_step(i, j_eager)
    h1 = time.perf_counter()
    e1.record(stream)
    torch.cuda.synchronize()
    eager = {"us_per_step": e0.elapsed_time(e1) * 1e3 / args.steps,
             "host_submit_us_per_step": (h1 - h0) * 1e6 / args.steps,
             "gbs": eager_bytes / (e0.elapsed_time(e1) / 1e3) / 1e9}

    # isolated launches: an event pair around each step (no overlap with the
    # neighbours), 20 warm-up then args.launch_stats timed
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n_launch_stats)]
    for i in range(n_launch_stats):
        c = i % NC
        q, kn, vn = rows(c, j_stats + i // NC)
        ev[i][0].record(stream)
        caches[c].rq_decode_step(0, q, kn, vn, out=outs[c], n_splits=args.splits, workspace=ws)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    lt = sorted(a.elapsed_time(b) * 1e3 for a, b in ev[20:])
    pct = lambda p: lt[min(len(lt) - 1, int(round(p * (len(lt) - 1))))]
    launch_stats = {"n": len(lt), "warmup": 20, "median_us": pct(0.5), "p10_us": pct(0.1), "p90_us": pct(0.9),
                    "note": "one fused decode-step launch between two events (no overlap with its neighbours)"}
    status = QuantizedKVCache.rq_decode_read_status(ws)
    if status != 0:
        raise RuntimeError(f"device status {status}")

    # e2e: host buffers, copies inside the timed region.  Each step's q, k_new
    # and v_new sit next to each other in one pinned host row, so a step
    # moves its inputs with one host-to-device copy and reads its output back
    # with one device-to-host copy.  The copies run on a second stream, one
    # step ahead (inputs) and one step behind (output) of the decode launches,
    # as a serving loop would overlap them; events keep each cache's input and
    # output buffers from being reused before the previous use is done.
    nq = step_in[0][0][0, 0].numel()
    nk = step_in[0][1][0, 0].numel()
    pin_in, dev_in = [], []
    for c in range(NC):
        q_c, k_c, v_c = step_in[c]
        S_c = q_c.shape[0]
        packed = torch.cat([q_c[:, 0].reshape(S_c, -1), k_c[:, 0].reshape(S_c, -1), v_c[:, 0].reshape(S_c, -1)],
                           dim=1)
        pin_in.append(packed.cpu().pin_memory())
        dev_in.append(torch.empty(nq + 2 * nk, dtype=torch.bfloat16, device="cuda"))
    dq = [d[:nq].view(step_in[0][0][0, 0].shape) for d in dev_in]
    dk = [d[nq:nq + nk].view(step_in[0][1][0, 0].shape) for d in dev_in]
    dv = [d[nq + nk:].view(step_in[0][2][0, 0].shape) for d in dev_in]
    host_out = torch.empty((wl.batch, wl.n_q_heads, wl.head_dim), dtype=torch.float32).pin_memory()
    base_len = [caches[c].length(0) for c in range(NC)]
    e2e_bytes = 0
    for i in range(e2e_steps):
        c = i % NC
        e2e_bytes += append_bytes(wl, rec, base_len[c] + i // NC) + decode_bytes(wl, rec, base_len[c] + i // NC + 1)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cstream = torch.cuda.Stream()
    h2d_done = [torch.cuda.Event() for _ in range(NC)]
    used = [torch.cuda.Event() for _ in range(NC)]      # decode of a cache's last step has read its inputs
    d2h_done = [torch.cuda.Event() for _ in range(NC)]  # its output has been copied out

    def e2e_loop(main):
        """The e2e steps on stream `main`, copies on cstream (forked from main)."""
        fork = torch.cuda.Event()
        fork.record(main)
        cstream.wait_event(fork)

        def h2d(i):
            c = i % NC
            with torch.cuda.stream(cstream):
                if i >= NC:
                    cstream.wait_event(used[c])
                dev_in[c].copy_(pin_in[c][j0 + i // NC], non_blocking=True)
                h2d_done[c].record(cstream)

        h2d(0)
        for i in range(e2e_steps):
            c = i % NC
            if i + 1 < e2e_steps:
                h2d(i + 1)
            main.wait_event(h2d_done[c])
            if i >= NC:
                main.wait_event(d2h_done[c])
            caches[c].rq_decode_step(0, dq[c], dk[c], dv[c], out=outs[c], n_splits=args.splits, workspace=ws)
            used[c].record(main)
            with torch.cuda.stream(cstream):
                cstream.wait_event(used[c])
                host_out.copy_(outs[c], non_blocking=True)
                d2h_done[c].record(cstream)
        main.wait_event(d2h_done[(e2e_steps - 1) % NC])

    # Captured as one CUDA graph and replayed once, like the device-timed
    # loop, so the figure is the device's and not the Python submission's
    # (the loop issues about ten stream operations per step).
    e2e_timing = "one CUDA-graph replay of the steps with their copies (copies on a second stream)"
    try:
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2):
            e2e_loop(torch.cuda.current_stream())
        torch.cuda.synchronize()
        upload_graph(g2, stream)
        torch.cuda.synchronize()
        torch.cuda._sleep(2_000_000)
        s2.record(stream)
        g2.replay()
        e2.record(stream)
        torch.cuda.synchronize()
        del g2
    except RuntimeError as exc:  # capture unavailable: the same loop launched eagerly
        torch.cuda.synchronize()
        e2e_timing = f"eager launches (graph capture failed: {str(exc)[:80]})"
        if any(caches[c].length(0) != base_len[c] for c in range(NC)):
            raise  # steps advanced during a partial capture: no consistent byte count
        s2.record(stream)
        e2e_loop(stream)
        e2.record(stream)
        torch.cuda.synchronize()
    e2e_elapsed = s2.elapsed_time(e2) / 1e3
    h2d = dev_in[0].numel() * 2
    d2h = host_out.numel() * 4

    elapsed_all, bytes_all, e2e_el_all, e2e_b_all = aggregate_ranks(elapsed, step_bytes, e2e_elapsed, e2e_bytes,
                                                                    world, "cuda")
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peak, peak_kind = _peaks()
    launches = args.steps + n_flush
    per_launch = elapsed / launches
    bytes_per_launch = step_bytes / launches
    achieved = bytes_per_launch / per_launch / 1e9
    tr = traffic_record()
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": (tr["bytes_per_launch_scaled"] if tr else None),
                "kernel": "decode_kernel<128,4> (fused append + split-K decode + combine; on the step before a tile "
                          "flush also the pack-ahead of that tile)",
                "peak_source": f"{peak_kind} hbm_gbs (burst)", "algorithmic_bytes_per_launch": bytes_per_launch,
                "avg_launch_us": per_launch * 1e6,
                "frac_of_nominal_8000_gbs": achieved / 8000.0,
                "timing": "CUDA events around one replay of a CUDA graph of the K timed steps (launches back to "
                          "back; each may overlap its predecessor's tail through programmatic dependent launch)",
                "graph_uploaded_before_timing": uploaded}
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        res = oracle_sample(wl, seconds=args.cpu_seconds)
        hc = host_cpu()
        cpu = {"value": res["decode_gbs"], "unit": "GB/s", "cores": res["threads"], "kind": "oracle",
               "sample": res["sample"], "cpu_model": hc["model"], "logical_cores": hc["cores"],
               "blas_threads": hc["blas_threads"], "quantize_gbs": res["quantize_gbs"]}
        if not args.no_sweep:
            cpu["workloads"] = oracle_configs()
    clk = clocks.summary()
    extra = {"eager": eager, "launch_stats": launch_stats, "repeats": repeats}
    if world == 1 and not args.no_sweep:
        try:
            extra["llama3_8b_step_loop"] = step_loop_graph()
        except Exception as exc:  # a secondary figure never hides the main line
            extra["llama3_8b_step_loop"] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        extra["workloads"] = sweep_workloads(["llama3_8b", "mistral_7b_b64", "qwen3_8b"], peak)
        extra["allocator"] = allocator_timings()
    line = {
        "metric": METRIC,
        "value": bytes_all / elapsed_all / 1e9,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": elapsed_all / args.steps * 1e3,
        "us_per_step": elapsed_all / args.steps * 1e6,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u2 codes; q and P in 16-bit fixed point (two int8 MMA terms); f32 scale/zero epilogue and softmax",
        "data": "synthetic",
        "config": arm_config(wl, NC, args.splits, world),
        "decode_gbs": achieved,
        "decode_us": per_launch * 1e6,
        "quantize_gbs": (qbytes / (sum(qtimes) / len(qtimes)) / 1e9) if qtimes else None,
        "alloc_ms": alloc_ms,
        "e2e": {"value": e2e_b_all / e2e_el_all / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "timing": e2e_timing},
        "gpu_launches": launches,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "clocks": clk,
    }
    line.update(extra)
    print(json.dumps(line))
    return 0


def run_profile_target(args):
    """A short run for profiler captures: one cache of the named workload,
    prefill, then `--steps` all-layer decode launches (rq_decode_attention,
    automatic plan), or fused steps (rq_decode_step) with --fused.  Prints
    the mean launch time (CUDA events) as one JSON line; not a bench line."""
    import torch

    from quantized_decode_attention_head_b200 import QuantizedKVCache, workloads

    wl = workloads.CONFIGS[args.profile]
    kb, vb = workload_bits(wl)
    if args.layers or args.batch:  # a smaller cache of the same workload (same per-layer bit widths)
        nl = args.layers or wl.n_layers
        wl = wl.with_(n_layers=nl, batch=args.batch or wl.batch)
        kb, vb = kb[:nl], vb[:nl]
    k, v, f = workloads.kv_inputs(wl, "cuda")
    cache = QuantizedKVCache(wl.n_layers, wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.n_sink,
                             wl.n_recent, wl.context + args.steps + 8, kb, vb, k_norm=args.k_norm)
    cache.rq_quantize_kv(k, v)
    del k, v
    torch.cuda.empty_cache()
    q, kn, vn = workloads.step_inputs(wl, args.steps, f, "cuda")
    ws = cache.make_workspace()
    out = torch.empty((wl.n_layers, wl.batch, wl.n_q_heads, wl.head_dim), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for t in range(args.steps):
        if args.fused:
            cache.rq_decode_step(-1, q[t].contiguous(), kn[t].contiguous(), vn[t].contiguous(), out=out, workspace=ws)
        else:
            cache.rq_decode_attention(-1, q[t].contiguous(), out=out, workspace=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    status = QuantizedKVCache.rq_decode_read_status(ws)
    print(json.dumps({"profile_target": args.profile, "launches": args.steps, "fused": bool(args.fused),
                      "k_norm": bool(args.k_norm), "mean_us": e0.elapsed_time(e1) * 1e3 / args.steps,
                      "device_status": status}))
    return 0 if status == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--splits", type=int, default=0)
    ap.add_argument("--copies", type=int, default=4)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--launch-stats", type=int, default=100, help="isolated launches timed one by one")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the secondary figures (other workloads, CUDA-graph step loop)")
    ap.add_argument("--profile", default=None, help="profiler target: a workload name (see run_profile_target)")
    ap.add_argument("--fused", action="store_true", help="with --profile: fused decode steps")
    ap.add_argument("--k-norm", action="store_true", help="with --profile: a K-normalized cache")
    ap.add_argument("--layers", type=int, default=0, help="with --profile: first N layers only")
    ap.add_argument("--batch", type=int, default=0, help="with --profile: batch size override")
    args = ap.parse_args()
    if args.profile:
        return run_profile_target(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
