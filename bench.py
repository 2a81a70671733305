"""Benchmark of Loki sparse decode-step attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One timed step = one Loki decode layer-step (rotate q, low-rank scores, top-k,
gather attention, combine) through the C ABI on a cache already resident in
HBM, by default on the largest single-GPU decode workload
(llama3-8b-gqa-decode: B 8, 32 query / 8 KV heads, S 32768, d_f 0.5,
k_f 0.125).  Each step also appends the step's new token first (timed
separately).  The in-library dense decode on the same cache is timed over K
steps of its own.  The same run also times a short-row decode
(llama2-7b-decode) and the pages' generation run (llama2-13b-generation:
prompt 3072, then 512 steps that append their token inside the call), Loki
against dense, and the fp64 oracle on the host (one thread and the BLAS
pool) with its dense attention beside it.
L2 is flushed before every step by writing a buffer twice the L2 size and then
reading another of that size (a write alone left part of a small workload's
inputs in L2, and its dirty lines cost the next kernel write-backs); the flush
is outside the timed events.  Device time from CUDA events on the launching
stream, summed over the K steps, max over ranks.

With N GPUs (torchrun) each rank runs the whole workload on its own batch
shard of an N-times larger global batch: weak scaling, no data-path
collective.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from workloads import get_workload  # noqa: E402
from workloads import generators as gen  # noqa: E402

METRIC = "Loki decode attention µs/layer-step and achieved HBM GB/s vs peak, vs dense"
UNIT = "us/layer-step"
DEFAULT_WORKLOAD = "llama3-8b-gqa-decode"
# timed in the same run beside the main workload: a short-row decode, and the
# generation run the pages quote their speed-up on
EXTRA_DECODE = "llama2-7b-decode"
GENERATION = "llama2-13b-generation"
FALLBACK_HBM_GBS = 6650.0


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(src: str) -> str:
    """The source without comments and blank space, so that a comment edit
    does not count as a kernel change (string literals hold no comment
    markers in these files)."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def source_hash() -> str:
    """Hash of the kernel sources' code (comments and spacing ignored)."""
    h = hashlib.sha1()
    d = os.path.join(ROOT, "sparse_decode_attention_loki_b200", "csrc")
    for f in sorted(os.listdir(d)):
        with open(os.path.join(d, f), encoding="utf-8") as fh:
            h.update(f.encode() + _code_only(fh.read()).encode())
    return h.hexdigest()[:12]


def decode_kernel_name(rot: int, short_kernel: int) -> str:
    """The kernel(s) of a Loki step, from loki_decode_launch_shape."""
    k = "loki_short_kernel" if short_kernel else "loki_decode_kernel"
    if rot == 0:
        return f"{k} (rotates its own queries)"
    return f"loki_rotate_kernel + {k} (programmatic dependent pair)"


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source; else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t[kernel][workload]
        if e.get("source_hash") == source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# Device-timed loops run in chunks of CHUNK steps.  Each chunk starts with a GPU
# sleep long enough for the host to enqueue the whole chunk, so the GPU never
# waits for a launch inside a timed interval: the events then time the kernels,
# not Python's launch rate.  (The e2e loop does not do this.)
CHUNK = 64
HOST_US_PER_STEP = 250.0


def queue_ahead(torch, n_steps):
    torch.cuda._sleep(int(n_steps * HOST_US_PER_STEP * 1e-6 * 2.0e9))


def lowrank_width(d, dtype, D):
    """Width of the low-rank key plane a cache for reduced dimension d keeps:
    d rounded up to whole 16-byte chunks (0 when that reaches D: no plane)."""
    per = 8 if dtype == "bf16" else 4
    d_lr = (d + per - 1) // per * per
    return d_lr if d_lr < D else 0


def workload_config(w, n_gpus):
    return {"workload": w.name, "batch_per_gpu": w.batch, "global_batch": w.batch * n_gpus,
            "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "seq_len": w.seq_len, "d": w.d, "k": w.k, "d_f": w.d_f, "k_f": w.k_f,
            "cache_dtype": w.dtype, "keys": f"{w.generator} spectrum (alpha {w.alpha})",
            "l2": "flushed before every timed step (write of 2x L2, then a read of 2x L2, outside the timed events)",
            "launch_queue": f"every {CHUNK} timed steps are enqueued behind a GPU sleep, so the host's "
                            "launch rate stays outside the events (not in e2e)",
            "parallelism": f"weak: batch shard per GPU, {n_gpus} GPU(s), no collective"}


# ------------------------------------------------------------------------------------ oracle arm
_ROW_CACHE = {}


def _oracle_rows(w, seed, distinct: int = 16):
    """Seeded (batch, KV head) rows of the workload with their oracle inputs,
    widened to fp64: (q64 [1, G, D], K_hat [1, 1, S, D], V [1, 1, S, D],
    P [1, D, D]).  Up to `distinct` rows are drawn (and kept for later calls),
    then they repeat."""
    import oracle
    key = (w.name, seed)
    if key not in _ROW_CACHE:
        P32 = np.stack([oracle.pca_basis(gen.calibration_keys(w, g))[0]
                        for g in range(w.n_kv_heads)]).astype(np.float32).astype(np.float64)
        _ROW_CACHE[key] = (P32, np.random.default_rng(seed), [])
    P32, rng, rows = _ROW_CACHE[key]
    G = w.group
    i = 0
    while True:
        if i >= len(rows) and len(rows) < distinct:
            b, g = int(rng.integers(0, w.batch)), int(rng.integers(0, w.n_kv_heads))
            _, k64 = gen.to_cache_dtype(gen.row_keys(w, b, g, w.seq_len), w.dtype)
            _, v64 = gen.to_cache_dtype(gen.row_values(w, b, g, w.seq_len), w.dtype)
            _, q64 = gen.to_cache_dtype(gen.queries(w, b)[g * G:(g + 1) * G][None], w.dtype)
            K_hat = oracle.rotate_keys(k64[None, None], P32[g:g + 1], w.dtype)
            rows.append((q64, K_hat, v64[None, None], P32[g:g + 1]))
        yield rows[i % len(rows)]
        i += 1


def oracle_sample_us(w, budget_s: float, seed: int = 0, threads=None, dense: bool = False):
    """Time the fp64 oracle (the Loki decode, or with dense=True its dense
    attention) on whole (batch, KV head) rows of the workload, one row at a
    time, until budget_s of wall time is spent; scale the mean row time to one
    layer-step (all B*Hkv rows).  threads: the BLAS thread limit (None: the
    library's default pool).  Returns (us per layer-step, rows timed, thread
    limit, effective cores = process CPU time / wall time over the timed calls)."""
    import oracle
    from threadpoolctl import threadpool_info, threadpool_limits
    times, cpu = [], []
    t_start = time.perf_counter()
    with threadpool_limits(limits=threads):
        limit = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        for q64, K_hat, v64, P in _oracle_rows(w, seed):
            c0, t0 = time.process_time(), time.perf_counter()
            if dense:
                oracle.dense_decode(q64, K_hat, v64, P, w.seq_len)
            else:
                oracle.loki_decode(q64, K_hat, v64, P, w.seq_len, w.d, w.k)
            times.append(time.perf_counter() - t0)
            cpu.append(time.process_time() - c0)
            if sum(times) >= budget_s or time.perf_counter() - t_start > 3 * budget_s or len(times) >= 4096:
                break
    per_row = float(np.mean(times))
    return per_row * w.rows * 1e6, len(times), limit, float(sum(cpu) / max(sum(times), 1e-12))


def cpu_baseline(w, budget_s: float):
    """The oracle's Loki decode with the default BLAS pool and with one
    thread, and its dense attention beside it (default pool), each on a
    bounded sample of rows."""
    us, rows, limit, eff = oracle_sample_us(w, budget_s)
    us1, rows1, _, eff1 = oracle_sample_us(w, budget_s / 2, threads=1)
    dus, drows, dlimit, deff = oracle_sample_us(w, budget_s / 2, dense=True)
    host = len(os.sched_getaffinity(0))
    return {"value": us, "unit": UNIT, "cores": limit, "kind": "oracle",
            "sample": f"{rows} calls on whole (batch, KV head) rows (up to 16 distinct rows, repeated), fp64 numpy "
                      f"oracle, scaled to all {w.rows} rows of one layer-step; BLAS pool of {limit} threads, "
                      f"{eff:.2f} cores busy on average",
            "effective_cores": eff, "host_cores": host,
            "single_thread": {"value": us1, "unit": UNIT, "cores": 1, "rows": rows1, "effective_cores": eff1},
            "dense_fp64": {"value": dus, "unit": UNIT, "cores": dlimit, "rows": drows, "effective_cores": deff,
                           "what": "the oracle's dense attention over all S tokens of each row"}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = get_workload(args.workload)
    budget = args.cpu_budget
    for _ in range(args.warmup if args.warmup > 0 else 0):
        oracle_sample_us(w, budget_s=0.0, seed=1)
    per_step = []
    rows = 0
    threads = 1
    effs = []
    for s in range(args.steps):
        us, n, threads, eff = oracle_sample_us(w, budget_s=budget / max(1, args.steps), seed=100 + s)
        per_step.append(us)
        effs.append(eff)
        rows += n
    value = float(np.mean(per_step))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": value / 1000.0,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{rows} whole (batch, KV head) rows of the workload, fp64 numpy oracle, "
                                   f"scaled to all {w.rows} rows; BLAS pool of {threads} threads, "
                                   f"{float(np.mean(effs)):.2f} cores busy on average",
                         "effective_cores": float(np.mean(effs))},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------------------------ GPU arm
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.proc = None
        self.gpu_index = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def time_prefill(L, cache, k_pre, v_pre, P, stream, dev, reps: int = 5):
    """Device time of the bulk append of the prompt (rewriting the same cache
    rows), L2 flushed before each repetition; median over reps."""
    import torch
    flush = L2Flush(torch, dev)
    ts = []
    for i in range(reps + 2):
        flush(float(i))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        L.loki_append(cache, 0, k_pre, v_pre, P)
        e1.record(stream)
        e1.synchronize()
        if i >= 2:
            ts.append(e0.elapsed_time(e1) * 1000.0)
    us = float(np.median(ts))
    # keys in, rotated keys out, values in, values out, and the low-rank plane's copy
    nbytes = 4 * k_pre.numel() * k_pre.element_size()
    if cache.k_lr is not None:
        nbytes += k_pre.numel() // k_pre.shape[-1] * cache.d_lr * k_pre.element_size()
    return {"us": us, "vectors_per_kv_head": int(k_pre.shape[0] * k_pre.shape[2]), "bytes": nbytes,
            "lowrank_plane": cache.d_lr,
            "hbm_gbs": nbytes / (us * 1e-6) / 1e9, "reps": reps,
            "kernel": "append_tc_kernel" if (k_pre.dtype == torch.bfloat16
                                             and k_pre.shape[0] * k_pre.shape[2] >= 256) else "append_kernel"}


def calibrate(L, calib, dev, stream, reps: int = 3):
    """P of every KV head from its calibration keys on the GPU
    (loki_pca_calibrate), and the device time of that calibration (median over
    reps)."""
    import torch
    keys = torch.as_tensor(np.stack(calib).astype(np.float32)).to(dev)
    H, N, D = keys.shape
    ws = torch.empty(L.loki_pca_workspace_size(H, D), dtype=torch.uint8, device=dev)
    P, _ = L.loki_pca_calibrate(keys, workspace=ws)
    if reps < 1:
        return P, None
    ts = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        L.loki_pca_calibrate(keys, workspace=ws)
        e1.record(stream)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1) * 1000.0)
    return P, {"us": float(np.median(ts)), "heads": int(H), "keys_per_head": int(N), "reps": reps,
               "kernels": "pca_mean_kernel, pca_cov_kernel, pca_jacobi_kernel",
               "note": "P of every measurement comes from this calibration"}


def fill_cache(L, w, cache, P, n_tokens, g_dev, dev, td):
    """Bulk-append n_tokens synthetic tokens (keys of the workload's generator,
    N(0, 1) values) at positions [0, n_tokens) of every row; returns the
    appended (k, v) tensors."""
    import torch
    B, Hkv, D = w.batch, w.n_kv_heads, w.head_dim
    k_pre = torch.empty((B, Hkv, n_tokens, D), dtype=td, device=dev)
    for h in range(Hkv):
        k_pre[:, h] = gen.device_keys(gen.make_key_model(w, h), B, n_tokens, g_dev, dev, td)
    v_pre = torch.randn((B, Hkv, n_tokens, D), generator=g_dev, device=dev).to(td)
    L.loki_append(cache, 0, k_pre, v_pre, P)
    return k_pre, v_pre


class L2Flush:
    """Evicts the L2 before a timed call: writes a buffer twice the L2 size,
    then reads another of that size.  On B200 a written buffer alone (even 4x
    the L2) left part of a small workload's inputs cached, and its dirty lines
    made the next kernel pay their write-back; the read leaves clean lines of
    a buffer the timed call never touches."""

    def __init__(self, torch, dev):
        n = 2 * torch.cuda.get_device_properties(dev).L2_cache_size // 4
        self.torch = torch
        self.w = torch.empty(n, dtype=torch.float32, device=dev)
        self.r = torch.ones(n, dtype=torch.float32, device=dev)
        self.sink = torch.empty(1, dtype=torch.float32, device=dev)

    def __call__(self, v):
        self.w.fill_(float(v))
        self.torch.sum(self.r, 0, True, out=self.sink)


def time_calls(torch, stream, flush, calls, steps, warmup):
    """Mean device time (us) of each call in `calls`, each in a loop of its own
    over `steps` steps (call(i) for step i), the L2 flushed before every step
    outside the events, every CHUNK steps queued behind a GPU sleep."""
    res = []
    for call in calls:
        for i in range(warmup):
            call(i)
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(min(CHUNK, steps))]
        tot = 0.0
        done = 0
        while done < steps:
            n = min(CHUNK, steps - done)
            queue_ahead(torch, n)
            for i in range(n):
                flush(float(i & 7))
                ev[i][0].record(stream)
                call(done + i)
                ev[i][1].record(stream)
            torch.cuda.synchronize()
            for i in range(n):
                tot += ev[i][0].elapsed_time(ev[i][1])
            done += n
        res.append(tot * 1000.0 / steps)
    return res


def time_decode_workload(L, name, flush, stream, dev, steps, warmup, peak):
    """One more decode workload timed in the same run: the Loki step and the
    dense baseline on its own cache (with the low-rank plane, like the main
    workload), each in a loop of its own, and the Loki step with the dense
    kernel run before it."""
    import torch
    w = get_workload(name)
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    S, B, Hkv, Hq, D = w.seq_len, w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim
    P, _ = calibrate(L, [gen.calibration_keys(w, g) for g in range(Hkv)], dev, stream, reps=0)
    cache = L.LokiCache(B, Hkv, D, S, dtype=td, device=dev, lowrank_dim=lowrank_width(w.d, w.dtype, D))
    g_dev = torch.Generator(device=dev)
    g_dev.manual_seed(w.seed * 131)
    k_pre, v_pre = fill_cache(L, w, cache, P, S, g_dev, dev, td)
    del k_pre, v_pre
    qs = [torch.randn((B, Hq, D), generator=g_dev, device=dev).to(td) for _ in range(4)]
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    dout = torch.empty_like(out)
    idx = torch.empty((B, Hkv, w.k), dtype=torch.int32, device=dev)
    loki = lambda i: L.loki_decode_attention(cache, S, qs[i % 4], P, w.d, w.k, out=out, idx=idx)
    dense = lambda i: L.dense_decode_attention(cache, S, qs[i % 4], P, out=dout)

    def both(i):
        dense(i)
        loki(i)
    loki_us, dense_us = time_calls(torch, stream, flush, [loki, dense], steps, warmup)
    # interleaved: events around the Loki call only, the dense call before it
    for i in range(warmup):
        both(i)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(min(CHUNK, steps))]
    tot, done = 0.0, 0
    while done < steps:
        n = min(CHUNK, steps - done)
        queue_ahead(torch, n)
        for i in range(n):
            flush(float(i & 7))
            dense(done + i)
            ev[i][0].record(stream)
            loki(done + i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        for i in range(n):
            tot += ev[i][0].elapsed_time(ev[i][1])
        done += n
    lb, db = w.loki_bytes(), w.dense_bytes()
    rot, ncta, ctas, short_kernel = L.loki_decode_launch_shape(cache, S, Hq, w.k)
    del cache
    torch.cuda.empty_cache()
    return {"workload": name, "loki_us": loki_us, "dense_us": dense_us,
            "launch": {"kernel": decode_kernel_name(rot, short_kernel), "cluster_ctas": ncta, "ctas": ctas},
            "loki_frac": lb / (loki_us * 1e-6) / 1e9 / peak, "dense_frac": db / (dense_us * 1e-6) / 1e9 / peak,
            "speedup_vs_dense": dense_us / loki_us, "byte_ratio": db / lb,
            "loki_after_dense_us": tot * 1000.0 / steps, "steps": steps,
            "algorithmic_bytes": lb, "dense_bytes": db}


def time_generation(L, name, flush, stream, dev, peak, warmup):
    """The generation run as the pages state it: a prompt cache of prompt_len
    tokens, then gen_steps decode steps, step t appending its token (rotated)
    at position prompt_len + t inside the call and attending over
    prompt_len + t + 1 tokens with k = floor(k_f * length).  The Loki step
    (loki_decode_attention_append) and the dense step
    (dense_decode_attention_append) each run the whole generation in a loop of
    their own; mean device time per step, L2 flushed before every step."""
    import torch
    from workloads.configs import key_budget
    w = get_workload(name)
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    B, Hkv, Hq, D = w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim
    T0, NS = w.prompt_len, w.gen_steps
    cap = T0 + NS
    P, _ = calibrate(L, [gen.calibration_keys(w, g) for g in range(Hkv)], dev, stream, reps=0)
    cache = L.LokiCache(B, Hkv, D, cap, dtype=td, device=dev, lowrank_dim=lowrank_width(w.d, w.dtype, D))
    g_dev = torch.Generator(device=dev)
    g_dev.manual_seed(w.seed * 131)
    k_pre, v_pre = fill_cache(L, w, cache, P, T0, g_dev, dev, td)
    del k_pre, v_pre
    NSET = 8
    qs = [torch.randn((B, Hq, D), generator=g_dev, device=dev).to(td) for _ in range(NSET)]
    kn = [gen.device_keys(gen.make_key_model(w, 0), B * Hkv, 1, g_dev, dev, td).view(B, Hkv, D)
          for _ in range(NSET)]
    vn = [torch.randn((B, Hkv, D), generator=g_dev, device=dev).to(td) for _ in range(NSET)]
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    idxs = {}
    ws = cache.workspace(cap, Hq)

    def loki(t):
        S = T0 + t + 1
        k = key_budget(w.k_f, S)
        if k not in idxs:
            idxs[k] = torch.empty((B, Hkv, k), dtype=torch.int32, device=dev)
        L.loki_decode_attention_append(cache, S, kn[t % NSET], vn[t % NSET], qs[t % NSET], P, w.d, k, out=out,
                                       idx=idxs[k], workspace=ws)

    def dense(t):
        S = T0 + t + 1
        L.dense_decode_attention_append(cache, S, kn[t % NSET], vn[t % NSET], qs[t % NSET], P, out=out)

    for t in range(NS):  # every idx buffer exists before the timed loops
        k = key_budget(w.k_f, T0 + t + 1)
        idxs.setdefault(k, torch.empty((B, Hkv, k), dtype=torch.int32, device=dev))
    loki_us, dense_us = time_calls(torch, stream, flush, [loki, dense], NS, min(warmup, NS))
    e = w.elem_bytes
    lb = sum(w.rows * ((T0 + t + 1) * w.d * e + key_budget(w.k_f, T0 + t + 1) * 2 * D * e)
             for t in range(NS)) / NS
    db = sum(w.rows * (T0 + t + 1) * 2 * D * e for t in range(NS)) / NS
    del cache
    torch.cuda.empty_cache()
    return {"workload": name, "prompt_len": T0, "gen_steps": NS,
            "loki_us_per_step": loki_us, "dense_us_per_step": dense_us, "speedup_vs_dense": dense_us / loki_us,
            "loki_frac": lb / (loki_us * 1e-6) / 1e9 / peak, "dense_frac": db / (dense_us * 1e-6) / 1e9 / peak,
            "mean_algorithmic_bytes_per_step": lb, "mean_dense_bytes_per_step": db,
            "note": "each step appends its token inside the call (rotated key, value, low-rank plane) and "
                    "attends over prompt_len + t + 1 tokens; the bytes exclude the append, as the pages' "
                    "speedup does"}


def time_paged(L, w, cache, qs, P, flush, stream, dev, steps: int, warmup: int, page: int = 16):
    """Device time of loki_paged_decode_attention on a paged copy of the cache
    (pages of `page` tokens in a shuffled order, every sequence at seq_len),
    L2 flushed before each call like the main loop."""
    import torch
    B, Hkv, S, D = w.batch, w.n_kv_heads, w.seq_len, w.head_dim
    pps = (S + page - 1) // page
    gen_t = torch.Generator(device="cpu")
    gen_t.manual_seed(7)
    perm = torch.randperm(B * pps, generator=gen_t).to(dev)
    table = perm.view(B, pps).to(torch.int32).contiguous()
    pcache = L.PagedLokiCache(B * pps, Hkv, D, page, dtype=cache.dtype, device=dev,
                              lowrank_dim=cache.d_lr or None)  # the same low-rank plane, paged
    pad = pps * page - S
    pairs = [(cache.k_hat, pcache.k_hat), (cache.v, pcache.v)]
    if cache.k_lr is not None:
        pairs.append((cache.k_lr, pcache.k_lr))
    for src, dst in pairs:
        W = src.shape[-1]
        x = src[:, :, :S]
        if pad:
            x = torch.cat([x, torch.zeros((B, Hkv, pad, W), dtype=x.dtype, device=dev)], dim=2)
        x = x.view(B, Hkv, pps, page, W).permute(0, 2, 1, 3, 4).reshape(B * pps, Hkv, page, W)
        dst[perm.long()] = x
    seqs = L.SeqTable(table, None, S)
    out = torch.empty((B, w.n_q_heads, D), dtype=torch.float32, device=dev)
    idx = torch.empty((B, Hkv, w.k), dtype=torch.int32, device=dev)
    ws = cache.workspace(S, w.n_q_heads)
    for i in range(max(3, warmup)):
        L.loki_paged_decode_attention(pcache, seqs, qs[i % len(qs)], P, w.d, w.k, out=out, idx=idx, workspace=ws)
    torch.cuda.synchronize()
    tot = 0.0
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        if i % CHUNK == 0:
            queue_ahead(torch, min(CHUNK, steps - i))
        flush(float(i & 7))
        evs[i][0].record(stream)
        L.loki_paged_decode_attention(pcache, seqs, qs[i % len(qs)], P, w.d, w.k, out=out, idx=idx, workspace=ws)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    tot = sum(a.elapsed_time(b) for a, b in evs) * 1000.0
    us = tot / steps
    del pcache
    return {"us": us, "page_size": page, "pages": int(B * pps), "steps": steps,
            "hbm_gbs": w.loki_bytes() / (us * 1e-6) / 1e9, "lowrank_plane": cache.d_lr,
            "layout": "shuffled pages, every sequence at seq_len"}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import sparse_decode_attention_loki_b200 as L

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = get_workload(args.workload)
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    S, B, Hkv, Hq, D = w.seq_len, w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim
    stream = torch.cuda.current_stream(dev)

    # offline calibration (on the GPU, loki_pca_calibrate) and cache prefill:
    # S-1 tokens; each step appends token S-1
    P, pca = calibrate(L, [gen.calibration_keys(w, g) for g in range(Hkv)], dev, stream)
    # the cache keeps a low-rank key plane as wide as d (contiguous score rows)
    d_lr = lowrank_width(w.d, w.dtype, D)
    cache = L.LokiCache(B, Hkv, D, S, dtype=td, device=dev, lowrank_dim=d_lr)
    g_dev = torch.Generator(device=dev)
    g_dev.manual_seed(w.seed * 131 + rank)
    if S > 1:
        k_pre = torch.empty((B, Hkv, S - 1, D), dtype=td, device=dev)
        for h in range(Hkv):
            k_pre[:, h] = gen.device_keys(gen.make_key_model(w, h), B, S - 1, g_dev, dev, td)
        v_pre = torch.randn((B, Hkv, S - 1, D), generator=g_dev, device=dev).to(td)
        L.loki_append(cache, 0, k_pre, v_pre, P)
        prefill = time_prefill(L, cache, k_pre, v_pre, P, stream, dev)
        del k_pre, v_pre
    else:
        prefill = None
    NSET = 4
    qs = [torch.randn((B, Hq, D), generator=g_dev, device=dev).to(td) for _ in range(NSET)]
    kn = [torch.randn((B, Hkv, 1, D), generator=g_dev, device=dev).to(td) for _ in range(NSET)]
    vn = [torch.randn((B, Hkv, 1, D), generator=g_dev, device=dev).to(td) for _ in range(NSET)]
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    idx = torch.empty((B, Hkv, w.k), dtype=torch.int32, device=dev)
    dout = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    flush = L2Flush(torch, dev)
    torch.cuda.synchronize()

    # One Loki step: the one-token append, then the decode.  The dense baseline
    # runs in a loop of its own (dense_step); `with_dense` runs it after the
    # decode of the same step instead, for the interleaved figure.
    def step(i, ev=None, with_dense=False):
        j = i % NSET
        flush(float(i & 7))
        if ev is not None:
            ev[0].record(stream)
        L.loki_append(cache, S - 1, kn[j], vn[j], P)
        if ev is not None:
            ev[1].record(stream)
        L.loki_decode_attention(cache, S, qs[j], P, w.d, w.k, out=out, idx=idx)
        if ev is not None:
            ev[2].record(stream)
        if with_dense:
            L.dense_decode_attention(cache, S, qs[j], P, out=dout)

    def dense_step(i, ev):
        flush(float(i & 7))
        ev[0].record(stream)
        L.dense_decode_attention(cache, S, qs[i % NSET], P, out=dout)
        ev[1].record(stream)

    for i in range(args.warmup):
        step(i)
        L.dense_decode_attention(cache, S, qs[i % NSET], P, out=dout)
    torch.cuda.synchronize()

    # ---------------- device-timed region
    CH = CHUNK
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(min(CH, args.steps))]
    t_app = t_loki = t_dense = 0.0
    per_step_loki = []
    pr = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0")
    time.sleep(0.3)  # let nvidia-smi take its first sample
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    done = 0
    while done < args.steps:
        n = min(CH, args.steps - done)
        queue_ahead(torch, n)
        for i in range(n):
            step(done + i, evs[i])
        torch.cuda.synchronize()
        for i in range(n):
            e = evs[i]
            a, b_ = e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2])
            t_app += a
            t_loki += b_
            per_step_loki.append(b_)
        done += n
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    # the dense baseline, same steps, its own loop
    done = 0
    while done < args.steps:
        n = min(CH, args.steps - done)
        queue_ahead(torch, n)
        for i in range(n):
            dense_step(done + i, evs[i])
        torch.cuda.synchronize()
        for i in range(n):
            t_dense += evs[i][0].elapsed_time(evs[i][1])
        done += n
    clocks = sampler.stop()
    # the Loki step with the dense kernel run after each decode (interleaved)
    il_steps = min(args.steps, 1000)
    t_il = 0.0
    done = 0
    while done < il_steps:
        n = min(CH, il_steps - done)
        queue_ahead(torch, n)
        for i in range(n):
            step(done + i, evs[i], with_dense=True)
        torch.cuda.synchronize()
        for i in range(n):
            t_il += evs[i][1].elapsed_time(evs[i][2])
        done += n

    # ---------------- end to end through host buffers (pinned), copies inside the events
    q_host = [q.cpu().pin_memory() for q in qs]
    out_host = torch.empty((B, Hq, D), dtype=torch.float32).pin_memory()
    idx_host = torch.empty((B, Hkv, w.k), dtype=torch.int32).pin_memory()
    q_dev = torch.empty_like(qs[0])
    e2e_steps = min(args.steps, 2000)
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(min(CH, e2e_steps))]
    t_e2e = 0.0
    for i in range(args.warmup):
        q_dev.copy_(q_host[i % NSET], non_blocking=True)
        L.loki_decode_attention(cache, S, q_dev, P, w.d, w.k, out=out, idx=idx)
        out_host.copy_(out, non_blocking=True)
        idx_host.copy_(idx, non_blocking=True)
    torch.cuda.synchronize()
    done = 0
    while done < e2e_steps:
        n = min(CH, e2e_steps - done)
        for i in range(n):
            flush(float(i & 7))
            e2e_ev[i][0].record(stream)
            q_dev.copy_(q_host[(done + i) % NSET], non_blocking=True)
            L.loki_decode_attention(cache, S, q_dev, P, w.d, w.k, out=out, idx=idx)
            out_host.copy_(out, non_blocking=True)
            idx_host.copy_(idx, non_blocking=True)
            e2e_ev[i][1].record(stream)
        torch.cuda.synchronize()
        for i in range(n):
            t_e2e += e2e_ev[i][0].elapsed_time(e2e_ev[i][1])
        done += n
    # the same step through DecodeGraph (query in, decode, results out: one graph
    # launch per step), one graph per query set
    graphs = [L.DecodeGraph(cache, S, P, w.d, w.k, Hq) for _ in range(NSET)]
    for j, gr in enumerate(graphs):
        gr.q_host.copy_(q_host[j])
    for i in range(args.warmup):
        graphs[i % NSET].replay()
    torch.cuda.synchronize()
    t_e2g = 0.0
    done = 0
    while done < e2e_steps:
        n = min(CH, e2e_steps - done)
        for i in range(n):
            flush(float(i & 7))
            e2e_ev[i][0].record(stream)
            graphs[(done + i) % NSET].replay()
            e2e_ev[i][1].record(stream)
        torch.cuda.synchronize()
        for i in range(n):
            t_e2g += e2e_ev[i][0].elapsed_time(e2e_ev[i][1])
        done += n
    del graphs
    # ---------------- the decode alone, back to back (no other kernel of ours between two
    # decodes), with and without the low-rank plane (same k_hat and v)
    cache_np = L.LokiCache(B, Hkv, D, S, dtype=td, device=dev, k_hat=cache.k_hat, v=cache.v)
    np_steps = min(args.steps, 1000)

    def decode_only(c):
        for i in range(args.warmup):
            L.loki_decode_attention(c, S, qs[i % NSET], P, w.d, w.k, out=out, idx=idx)
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(min(CH, np_steps))]
        tot = 0.0
        done = 0
        while done < np_steps:
            n = min(CH, np_steps - done)
            queue_ahead(torch, n)
            for i in range(n):
                flush(float(i & 7))
                ev[i][0].record(stream)
                L.loki_decode_attention(c, S, qs[(done + i) % NSET], P, w.d, w.k, out=out, idx=idx)
                ev[i][1].record(stream)
            torch.cuda.synchronize()
            for i in range(n):
                tot += ev[i][0].elapsed_time(ev[i][1])
            done += n
        return tot * 1000.0 / np_steps

    t_only = decode_only(cache)
    t_np = decode_only(cache_np) * np_steps / 1000.0
    del cache_np
    # ---------------- Exact-TopK baseline (d = D) and the agreement of the two selections
    idx_exact = torch.empty_like(idx)
    for i in range(args.warmup):
        L.loki_decode_attention(cache, S, qs[i % NSET], P, D, w.k, out=out, idx=idx_exact)
    torch.cuda.synchronize()
    ex_steps = min(args.steps, 500)
    ex_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(min(CH, ex_steps))]
    t_exact = 0.0
    done = 0
    while done < ex_steps:
        n = min(CH, ex_steps - done)
        queue_ahead(torch, n)
        for i in range(n):
            flush(float(i & 7))
            ex_ev[i][0].record(stream)
            L.loki_decode_attention(cache, S, qs[(done + i) % NSET], P, D, w.k, out=out, idx=idx_exact)
            ex_ev[i][1].record(stream)
        torch.cuda.synchronize()
        for i in range(n):
            t_exact += ex_ev[i][0].elapsed_time(ex_ev[i][1])
        done += n
    # ---------------- generation steps that append their token inside the call
    ga_steps = min(args.steps, 1000)
    kn3 = [x.view(B, Hkv, D) for x in kn]
    vn3 = [x.view(B, Hkv, D) for x in vn]
    for i in range(args.warmup):
        L.loki_decode_attention_append(cache, S, kn3[i % NSET], vn3[i % NSET], qs[i % NSET], P, w.d, w.k,
                                       out=out, idx=idx)
        L.dense_decode_attention_append(cache, S, kn3[i % NSET], vn3[i % NSET], qs[i % NSET], P, out=dout)
    torch.cuda.synchronize()
    ga_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(min(CH, ga_steps))]

    def gen_loop(call):
        tot = 0.0
        done = 0
        while done < ga_steps:
            n = min(CH, ga_steps - done)
            queue_ahead(torch, n)
            for i in range(n):
                j = (done + i) % NSET
                flush(float(i & 7))
                ga_ev[i][0].record(stream)
                call(j)
                ga_ev[i][1].record(stream)
            torch.cuda.synchronize()
            for i in range(n):
                tot += ga_ev[i][0].elapsed_time(ga_ev[i][1])
            done += n
        return tot

    # each arm in a loop of its own, like the decode and the dense baseline
    t_ga = gen_loop(lambda j: L.loki_decode_attention_append(cache, S, kn3[j], vn3[j], qs[j], P, w.d, w.k,
                                                             out=out, idx=idx))
    t_gd = gen_loop(lambda j: L.dense_decode_attention_append(cache, S, kn3[j], vn3[j], qs[j], P, out=dout))
    # ---------------- the same step on a paged copy of the cache (16-token pages, shuffled)
    paged = time_paged(L, w, cache, qs, P, flush, stream, dev, steps=min(args.steps, 500), warmup=args.warmup)
    jac = []
    for j in range(NSET):
        L.loki_decode_attention(cache, S, qs[j], P, w.d, w.k, out=out, idx=idx)
        L.loki_decode_attention(cache, S, qs[j], P, D, w.k, out=out, idx=idx_exact)
        jac.append(L.topk_jaccard(idx, idx_exact))
    jaccard = torch.stack(jac)
    rot, ncl, nct, short_kernel = L.loki_decode_launch_shape(cache, S, Hq, w.k)
    _, dcl, dct, _ = L.loki_decode_launch_shape(cache, S, Hq, dense=True)
    # ---------------- the short-row decode and the pages' generation run, same session
    extras = {}
    if world == 1 and not args.no_extras:
        peak_gbs, _ = peaks()
        del cache
        torch.cuda.empty_cache()
        extras["short_decode"] = time_decode_workload(L, EXTRA_DECODE, flush, stream, dev,
                                                      steps=max(args.steps, 200), warmup=args.warmup,
                                                      peak=peak_gbs)
        extras["generation"] = time_generation(L, GENERATION, flush, stream, dev, peak_gbs, args.warmup)
    h2d = q_host[0].numel() * q_host[0].element_size()
    d2h = out_host.numel() * 4 + idx_host.numel() * 4

    # ---------------- max over ranks
    tt = torch.tensor([t_loki, t_dense, t_app, t_e2e, t_e2g], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    t_loki, t_dense, t_app, t_e2e, t_e2g = [float(x) for x in tt.tolist()]

    if rank == 0:
        K = args.steps
        loki_us = t_loki * 1000.0 / K
        dense_us = t_dense * 1000.0 / K
        app_us = t_app * 1000.0 / K
        e2e_us = t_e2g * 1000.0 / e2e_steps
        e2e_eager_us = t_e2e * 1000.0 / e2e_steps
        peak, peak_kind = peaks()
        lb, db = w.loki_bytes(), w.dense_bytes()
        ach = lb / (loki_us * 1e-6) / 1e9
        dach = db / (dense_us * 1e-6) / 1e9
        line = {
            "metric": METRIC, "value": loki_us / world, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": loki_us / 1000.0, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(w, world),
            "us_per_layer_step_per_gpu": loki_us,
            "hbm_gbs": ach,
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                         "traffic": measured_traffic("loki_decode_step", w.name),
                         "kernel": decode_kernel_name(rot, short_kernel),
                         "peak_kind": f"{peak_kind} hbm_gbs (copy, burst)",
                         "algorithmic_bytes_per_launch": lb},
            "dense": {"us": dense_us, "hbm_gbs": dach, "frac": dach / peak, "bytes_per_launch": db,
                      "launch": {"cluster_ctas": dcl, "ctas": dct}},
            "speedup_vs_dense": dense_us / loki_us, "byte_ratio": db / lb,
            "lowrank_plane": {"d_lr": d_lr, "bytes": B * Hkv * S * d_lr * (2 if w.dtype == "bf16" else 4),
                              "no_plane_us": t_np * 1000.0 / np_steps, "no_plane_steps": np_steps,
                              "note": "value streams the scores from the cache's low-rank key plane; "
                                      "no_plane_us reads them from the k_hat rows (same results), "
                                      "timed like decode_only_us"},
            "decode_only_us": t_only,
            "interleaved_with_dense_us": t_il * 1000.0 / il_steps,
            "interleaved_note": "the step loop with the dense kernel run after each decode: a dense kernel "
                                "before a decode slows a short decode (state left on the SMs, most likely "
                                "their instruction caches), even with the L2 flushed in between; value and "
                                "dense are timed in loops of their own",
            "append_us": app_us,
            "step_with_append": {"loki_us": t_ga * 1000.0 / ga_steps, "dense_us": t_gd * 1000.0 / ga_steps,
                                 "loki_separate_us": app_us + loki_us, "steps": ga_steps,
                                 "note": "token appended inside the decode call (loki_decode_attention_append, "
                                         "dense_decode_attention_append) vs loki_append followed by the step"},
            "prefill_append": None if prefill is None else dict(prefill, frac=prefill["hbm_gbs"] / peak),
            "pca_calibrate": pca,
            "paged": dict(paged, frac=paged["hbm_gbs"] / peak),
            "exact_topk": {"us": t_exact * 1000.0 / ex_steps, "d": D, "k": w.k, "steps": ex_steps,
                           "jaccard_vs_loki": {"mean": float(jaccard.mean()), "min": float(jaccard.min()),
                                               "rows": int(jaccard.numel())}},
            "launch": {"rotate_ctas": rot, "decode_cluster_ctas": ncl, "decode_ctas": nct, "threads_per_cta": 256,
                       "decode_kernel": decode_kernel_name(rot, short_kernel)},
            "e2e": {"value": e2e_us / world, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps,
                    "path": "DecodeGraph.replay(): query copied in from pinned host memory, the decode, out "
                            "and idx copied back, captured as one CUDA graph",
                    "eager_value": e2e_eager_us / world,
                    "eager_path": "the same copies and loki_decode_attention issued one by one from Python"},
            "gpu_launches": (2 if rot == 0 else 3) * K,  # timed loop: append, [rotate,] decode
            "clocks": clocks,
            "wall_s_timed_region": wall,
            "per_step_loki_us": {"p50": float(np.percentile(per_step_loki, 50)) * 1000.0,
                                 "p10": float(np.percentile(per_step_loki, 10)) * 1000.0,
                                 "p90": float(np.percentile(per_step_loki, 90)) * 1000.0},
        }
        line.update(extras)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


PHASES = ("query", "stream", "bucket", "select", "attend", "merge")


def phase_summary(st, w, bin_us: float = 1.0):
    """Phase stamps of one decode (loki_phase_stamps: per CTA the global timer
    at kernel entry, queries ready, key stream done, first digit known,
    selection known, attention done, merge done) summarised: the kernel span,
    per phase the CTAs' durations, the achieved HBM rate of the key stream and
    of the gather over the span of each phase across CTAs, and a timeline of
    how many CTAs are in each phase per bin."""
    st = st[st[:, 0] > 0]
    t = st[:, :7].astype(np.float64)
    T0 = t[:, 0].min()
    t = (t - T0) / 1000.0
    span = float(t[:, 6].max())

    def q(x):
        return {"p50": round(float(np.percentile(x, 50)), 2), "p90": round(float(np.percentile(x, 90)), 2),
                "max": round(float(x.max()), 2)}
    phases = {nm: q(t[:, i + 1] - t[:, i]) for i, nm in enumerate(PHASES)}
    e = w.elem_bytes
    key_bytes = w.rows * w.seq_len * w.d * e
    gather_bytes = w.rows * w.k * 2 * w.head_dim * e
    stream_window = float(t[:, 2].max() - t[:, 1].min())
    gather_window = float(t[:, 5].max() - t[:, 4].min())
    nb = int(np.ceil(span / bin_us))
    tl = {nm: np.zeros(nb) for nm in PHASES}
    for i in range(len(t)):
        for p_, nm in enumerate(PHASES):
            a_, b_ = t[i, p_], t[i, p_ + 1]
            if b_ <= a_:
                continue
            for j in range(int(a_ // bin_us), min(nb - 1, int(b_ // bin_us)) + 1):
                lo, hi = max(a_, j * bin_us), min(b_, (j + 1) * bin_us)
                if hi > lo:
                    tl[nm][j] += (hi - lo) / bin_us
    return {"span_us": round(span, 2), "ctas": int(len(t)), "phase_us": phases,
            "phase_ends_us": {nm: q(t[:, i + 1]) for i, nm in enumerate(PHASES)},
            "stream_gbs_over_its_window": key_bytes / (stream_window * 1e-6) / 1e9 if stream_window > 0 else None,
            "gather_gbs_over_its_window": gather_bytes / (gather_window * 1e-6) / 1e9 if gather_window > 0 else None,
            "timeline_bin_us": bin_us,
            "timeline_ctas": {k_: [round(float(x), 1) for x in v] for k_, v in tl.items()}}


def run_phases(args):
    """One Loki decode of the workload on a build with phase stamps
    (-DLOKI_PHASE_STAMPS, built here as libloki_stamps.so): prints the
    stamped build's decode time and the summary of its CTAs' phases
    (phase_summary) as one JSON line."""
    import ctypes
    import torch

    from sparse_decode_attention_loki_b200 import _lib
    from sparse_decode_attention_loki_b200 import build as lbuild
    path = os.path.join(os.path.dirname(lbuild.LIB), "libloki_stamps.so")
    lbuild.build(defines=["-DLOKI_PHASE_STAMPS"], lib=path)
    _lib.load(path)
    import sparse_decode_attention_loki_b200 as L
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    w = get_workload(args.workload)
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    S, B, Hkv, Hq, D = w.seq_len, w.batch, w.n_kv_heads, w.n_q_heads, w.head_dim
    P, _ = calibrate(L, [gen.calibration_keys(w, g) for g in range(Hkv)], dev, stream, reps=0)
    cache = L.LokiCache(B, Hkv, D, S, dtype=td, device=dev, lowrank_dim=lowrank_width(w.d, w.dtype, D))
    g_dev = torch.Generator(device=dev)
    g_dev.manual_seed(w.seed * 131)
    k_pre, v_pre = fill_cache(L, w, cache, P, S, g_dev, dev, td)
    del k_pre, v_pre
    q = torch.randn((B, Hq, D), generator=g_dev, device=dev).to(td)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
    idx = torch.empty((B, Hkv, w.k), dtype=torch.int32, device=dev)
    flush = L2Flush(torch, dev)
    (us,) = time_calls(torch, stream, flush,
                       [lambda i: L.loki_decode_attention(cache, S, q, P, w.d, w.k, out=out, idx=idx)],
                       max(args.steps, 10), max(args.warmup, 3))
    flush(3.0)
    L.loki_decode_attention(cache, S, q, P, w.d, w.k, out=out, idx=idx)
    torch.cuda.synchronize()
    rot, ncta, ctas, _ = L.loki_decode_launch_shape(cache, S, Hq, w.k)
    buf = np.zeros((ctas, 10), dtype=np.uint64)
    n = ctypes.c_int32(0)
    _lib.check(_lib.load().loki_phase_stamps(1 if w.dtype == "bf16" else 0, D, buf.ctypes.data, ctas,
                                             ctypes.byref(n)))
    summ = phase_summary(buf[:n.value], w)
    line = {"phases": w.name, "decode_us_stamped_build": us,
            "launch": {"rotate_ctas": rot, "cluster_ctas": ncta, "ctas": ctas},
            "single_cta_select": bool(int(buf[0, 8]) >> 16 & 1),
            "short_row_kernel": bool(int(buf[0, 8]) >> 17 & 1),
            "algorithmic_bytes": w.loki_bytes(), **summ}
    print(json.dumps(line))
    return 0


def run_sweep(args):
    """Loki against the in-library dense kernel on every point of the
    Mistral-7B-like sweep (S x B x d_f x k_f), one JSON line per point.  The
    cache of one (S, B) serves its nine (d_f, k_f) points; device-timed with
    CUDA events, L2 flushed before every call, median of args.sweep_reps."""
    import torch

    import sparse_decode_attention_loki_b200 as L
    from workloads import mistral_sweep_points

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    flush = L2Flush(torch, dev)
    peak, _ = peaks()
    pts = [w for w in mistral_sweep_points() if args.sweep_filter in w.name]
    groups = {}
    for w in pts:
        groups.setdefault((w.seq_len, w.batch), []).append(w)

    def timed(fn, reps):
        for _ in range(3):
            flush(1.0)
            fn()
        ts = []
        for i in range(reps):
            flush(float(i & 7))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1) * 1000.0)
        return float(np.median(ts))

    for (S, B), ws in groups.items():
        w0 = ws[0]
        Hkv, Hq, D = w0.n_kv_heads, w0.n_q_heads, w0.head_dim
        P, _ = calibrate(L, [gen.calibration_keys(w0, g) for g in range(Hkv)], dev, stream, reps=0)
        cache = L.LokiCache(B, Hkv, D, S, dtype=torch.bfloat16, device=dev)
        g_dev = torch.Generator(device=dev)
        g_dev.manual_seed(w0.seed * 131)
        for h in range(Hkv):  # one KV head at a time: the prompt never holds two full copies
            k_h = gen.device_keys(gen.make_key_model(w0, h), B, S, g_dev, dev, torch.bfloat16)
            v_h = torch.randn((B, S, D), generator=g_dev, device=dev).to(torch.bfloat16)
            kk = torch.zeros((B, Hkv, S, D), dtype=torch.bfloat16, device=dev) if h == 0 else kk
            vv = torch.zeros((B, Hkv, S, D), dtype=torch.bfloat16, device=dev) if h == 0 else vv
            kk[:, h] = k_h
            vv[:, h] = v_h
            del k_h, v_h
        L.loki_append(cache, 0, kk, vv, P)
        del kk, vv
        q = torch.randn((B, Hq, D), generator=g_dev, device=dev).to(torch.bfloat16)
        out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
        # one low-rank plane per reduced dimension, each a view of the same k_hat and v
        planes = {}
        for w in ws:
            d_lr = lowrank_width(w.d, "bf16", D)
            if d_lr and d_lr not in planes:
                c = L.LokiCache(B, Hkv, D, S, dtype=torch.bfloat16, device=dev, k_hat=cache.k_hat, v=cache.v,
                                lowrank_dim=d_lr)
                c.k_lr.copy_(cache.k_hat[..., :d_lr])
                planes[d_lr] = c
        torch.cuda.synchronize()
        dense_us = timed(lambda: L.dense_decode_attention(cache, S, q, P, out=out), args.sweep_reps)
        for w in ws:
            idx = torch.empty((B, Hkv, w.k), dtype=torch.int32, device=dev)
            lc = planes.get(lowrank_width(w.d, "bf16", D), cache)
            loki_us = timed(lambda: L.loki_decode_attention(lc, S, q, P, w.d, w.k, out=out, idx=idx),
                            args.sweep_reps)
            np_us = timed(lambda: L.loki_decode_attention(cache, S, q, P, w.d, w.k, out=out, idx=idx),
                          args.sweep_reps)
            lb, db = w.loki_bytes(), w.dense_bytes()
            print(json.dumps({"sweep": "mistral-7b-gqa", "workload": w.name, "seq_len": S, "batch": B,
                              "d_f": w.d_f, "k_f": w.k_f, "d": w.d, "k": w.k, "loki_us": loki_us,
                              "loki_no_plane_us": np_us, "d_lr": lc.d_lr,
                              "dense_us": dense_us, "speedup_vs_dense": dense_us / loki_us,
                              "byte_ratio": db / lb, "loki_frac": lb / (loki_us * 1e-6) / 1e9 / peak,
                              "dense_frac": db / (dense_us * 1e-6) / 1e9 / peak, "reps": args.sweep_reps,
                              "l2": "flushed before every call"}), flush=True)
        del cache, planes
        torch.cuda.empty_cache()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=8.0, help="seconds of oracle CPU time")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the short-row decode and the generation run timed beside the main workload")
    ap.add_argument("--sweep", choices=["mistral"], default=None,
                    help="time Loki and dense on every Mistral sweep point instead of the bench step")
    ap.add_argument("--sweep-filter", default="", help="only sweep points whose name contains this")
    ap.add_argument("--sweep-reps", type=int, default=20)
    ap.add_argument("--phases", action="store_true",
                    help="build the library with phase stamps and print the unit timeline of one decode")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps; the number is not a valid bench value", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    if args.phases:
        return run_phases(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
