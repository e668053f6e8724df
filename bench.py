#!/usr/bin/env python
"""Benchmark: compressed-KV decode tokens/s at the Qwen2.5-7B layer shape on B200.

One step = one decode pass of the batch (rank-space scores, online softmax,
rank-space value sum and expansion over every compressed block, the
uncompressed suffix, and the split combine) through milo_decode_attn, on
factors produced by milo_compress from a seeded synthetic cache.  Compression
(Gram, Jacobi, entropy allocation, projection) is timed in the same run and
reported as compressions/s.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl milo|reference] [--workload NAME]
  python bench.py --profile decode|compress [--calls N]   (a short run for ncu captures)

Prints one JSON line on rank 0.  For N > 1 launch with torch.distributed.run;
every rank decodes its own batch (independent problems, no collective on the
data path) and the timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "compressed-KV decode tokens/s at Qwen2.5-7B shape; achieved HBM GB/s vs peak"
# DRAM bytes (read + written) of one launch of the main decode kernel, measured with ncu, per workload, keyed by
# the SHA-256 prefix of the kernel's source file at the time of the capture.  A different digest means the
# kernel has changed since the counters were taken, and the line reports traffic as null.
DECODE_TRAFFIC = {("qwen2.5-7b-layer", "e8e6591e8379"): 42518784 + 2560}


def _source_digest() -> str:
    import hashlib
    path = os.path.join(ROOT, "decode_attention_milo_b200", "csrc", "decode_tc.cu")
    with open(path, "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:12]


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="milo", choices=["milo", "reference"])
    p.add_argument("--workload", default="qwen2.5-7b-layer")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="bound of the CPU oracle sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--profile", choices=["decode", "decode8", "rope", "compress"], default=None,
                   help="run only N calls of one phase on the workload (for profiler captures), no JSON contract")
    p.add_argument("--calls", type=int, default=6)
    return p.parse_args()


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            j = json.load(fh)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons every 20 ms while the timed region runs (NVML; nvidia-smi
    when NVML cannot be loaded)."""

    # NVML clocks-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, index: int):
        self.index = index
        self.rows = []  # (sm_mhz, sm_max_mhz, reason bits)
        self._stop = threading.Event()
        self._t = None

    def _sample_nvml(self, nv, h):
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        try:
            bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception:
            bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        return float(sm), float(mx), int(bits)

    def _sample_smi(self):
        fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")
        r = subprocess.run(["nvidia-smi", f"--id={self.index}", f"--query-gpu={fields}",
                            "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5)
        v = [x.strip() for x in r.stdout.strip().split(",")]
        bits = sum(b for b, x in zip((0x8, 0x40, 0x20, 0x4), v[2:]) if x == "Active")
        return float(v[0]), float(v[1]), bits

    def _run(self):
        nv = h = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.index)
        except Exception:
            nv = None
        while True:
            try:
                self.rows.append(self._sample_nvml(nv, h) if nv else self._sample_smi())
            except Exception:
                pass
            if self._stop.wait(0.02 if nv else 0.2):
                break

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        reasons = sorted({name for _, _, bits in self.rows for b, name in self.REASONS.items() if bits & b})
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": max(r[1] for r in self.rows),
                "reasons": reasons, "samples": len(self.rows)}


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _max_over_ranks(x, world):
    """Max of a float over all ranks (the job's time is its slowest rank's); identity on one rank."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _job_value(world, batch, steps, ms):
    """Whole-job decode tokens/s: every rank decodes `batch` tokens per step; `ms` is the max over ranks."""
    return world * batch * steps / (ms / 1e3)


def _config(wl, world, ranks_total=None, **extra):
    """The workload description shared by both arms' JSON lines."""
    c = {"workload": wl.name, "batch": wl.batch, "kv_heads": wl.kv_heads, "q_heads": wl.q_heads,
         "head_dim": wl.head_dim, "context": wl.context, "block_size": wl.block_size, "suffix": wl.suffix,
         "budget": wl.budgets[0], "r_min": wl.r_min, "parallelism": f"replica x{world}"}
    if wl.layers > 1:  # a stack's layers are independent decode calls: one layer is timed
        c["layers_timed"] = f"layer 0 of {wl.layers}"
    if ranks_total is not None:
        c["ranks_total"] = int(ranks_total)
    c.update(extra)
    return c


def _to_dev(a, dt, torch):
    if dt == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def _device_ints(torch, ptr, n):
    """Host copy of n int32 values at a library-owned device address."""
    class _A:
        __cuda_array_interface__ = {"shape": (n,), "typestr": "<i4", "data": (int(ptr), False), "version": 3,
                                    "strides": None}
    return torch.as_tensor(_A(), device="cuda").cpu().numpy()


def _fp32_peak_tflops(torch):
    """FP32 FMA peak from the unit counts: SMs x 128 FP32 lanes x 2 flops x max SM clock."""
    props = torch.cuda.get_device_properties(0)
    mhz = None
    try:
        import pynvml as nv
        nv.nvmlInit()
        mhz = nv.nvmlDeviceGetMaxClockInfo(nv.nvmlDeviceGetHandleByIndex(torch.cuda.current_device()),
                                           nv.NVML_CLOCK_SM)
    except Exception:
        mhz = 1965
    return props.multi_processor_count * 128 * 2 * mhz * 1e6 / 1e12, mhz


def _compress_roofline(torch, wl, esize, ranks, sweeps, kern, peak_gbs):
    """Per-kernel fraction of roofline for one whole-layer compression (median CUDA-event times)."""
    H, T, d, n, nb = wl.kv_heads, wl.context, wl.head_dim, wl.block_size, wl.num_blocks
    nblk = 2 * H * nb
    x_bytes = 2 * H * T * d * esize                          # K and V, read once
    gram_bytes = x_bytes + nblk * d * d * 4                  # + the fp32 Gram matrices written
    rsum = int(ranks.sum())
    proj_bytes = x_bytes + rsum * d * 4 + rsum * (n + d) * esize  # + eigenvectors used, factors written
    pairs = d * (d - 1) // 2
    jac_flops = float(np.sum(sweeps)) * pairs * 18 * d     # per pair: 3 dot products (6d) + 4 column updates (12d)
    fp32_tf, mhz = _fp32_peak_tflops(torch)
    med = {k: statistics.median(v) for k, v in kern.items()}

    def hbm(bytes_, ms):
        gbs = bytes_ / (ms / 1e3) / 1e9
        return {"ms": ms, "bytes": bytes_, "achieved": gbs, "peak": peak_gbs, "unit": "GB/s", "frac": gbs / peak_gbs}
    jt = jac_flops / (med["jacobi"] / 1e3) / 1e12
    return {
        "gram": dict(hbm(gram_bytes, med["gram"]), bound="hbm"),
        "jacobi": {"bound": "alu", "ms": med["jacobi"], "flops": jac_flops, "achieved": jt, "peak": fp32_tf,
                   "unit": "TFLOP/s", "frac": jt / fp32_tf, "sweeps_mean": float(np.mean(sweeps)),
                   "sweeps_max": int(np.max(sweeps)),
                   "peak_note": f"FP32 FMA: SMs x 128 lanes x 2 flops x {mhz} MHz; flops count full sweeps"},
        "alloc": {"ms": med["alloc"]},
        "project": dict(hbm(proj_bytes, med["project"]), bound="hbm"),
    }


def _algorithmic_bytes(ranks, wl, esize):
    """Bytes one decode step must move: factors at their ranks (read once, shared by the batch),
    the per-query suffix K and V, q and out."""
    factors = int(ranks.sum()) * (wl.block_size + wl.head_dim) * esize
    suffix = 2 * wl.batch * wl.kv_heads * wl.suffix * wl.head_dim * esize
    qo = 2 * wl.batch * wl.q_heads * wl.head_dim * esize
    return factors + suffix + qo


def _algorithmic_bytes_8bit(qranks, wl):
    """The same for 8-bit factor objects: one byte per token-factor element, bf16 dimension factors, at the
    8-bit object's ranks (one more component per block below full rank)."""
    factors = int(qranks.sum()) * (wl.block_size * 1 + wl.head_dim * 2)
    suffix = 2 * wl.batch * wl.kv_heads * wl.suffix * wl.head_dim * 2
    qo = 2 * wl.batch * wl.q_heads * wl.head_dim * 2
    return factors + suffix + qo


def _decode_8bit(torch, milo, wl, sets, qs, ks, vs, outs, steps, peak):
    """8-bit factor storage (milo_factors_quantize): quantise time per layer and the decode kernel over the
    8-bit copies, timed like the main kernel (library events around it, eager launches over the copies)."""
    qsets, qms = [], []
    for f in sets:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        qsets.append(milo.quantize(f))
        e1.record()
        torch.cuda.synchronize()
        qms.append(e0.elapsed_time(e1))
    copies = len(qsets)
    for c in range(copies):
        milo.decode_attn(qs[c], qsets[c], ks[c], vs[c], out=outs[c])
    torch.cuda.synchronize()
    n = min(steps, 300)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a_, b_ in evs:
        a_.record()
        b_.record()
    for s_ in range(n):
        c = s_ % copies
        milo.decode_attn_profiled(qs[c], qsets[c], ks[c], vs[c], outs[c], evs[s_][0], evs[s_][1])
    torch.cuda.synchronize()
    kms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    qranks = qsets[0].ranks()
    nbytes = _algorithmic_bytes_8bit(qranks, wl)
    ok = all(f.status()[0] == 0 for f in qsets)
    for f in qsets:
        f.close()
    achieved = nbytes / (kms / 1e3) / 1e9
    return {"kernel": "decode_tc_kernel (8-bit mode)", "kernel_ms": kms, "bytes_per_step": nbytes,
            "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "decode_tokens_per_s": wl.batch / (kms / 1e3), "quantize_ms": statistics.median(qms), "status_ok": ok,
            "note": "token factors as int8 codes (asymmetric per rank channel, symmetric at full rank), dimension "
                    "factors bf16; same timing as the main kernel"}


def _decode_rope(torch, milo, wl, sets, qs, ks, vs, outs, steps, peak, ranks):
    """Pre-RoPE key factors (milo_decode_attn_rope): the whole call (key rebuild and rotation, decode,
    combine), timed with CUDA events around each eager call over the copies."""
    copies = len(sets)
    for c in range(copies):
        milo.decode_attn_rope(qs[c], sets[c], ks[c], vs[c], theta=1e6, out=outs[c])
    torch.cuda.synchronize()
    n = min(steps, 200)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for s_ in range(n):
        c = s_ % copies
        evs[s_][0].record()
        milo.decode_attn_rope(qs[c], sets[c], ks[c], vs[c], theta=1e6, out=outs[c])
        evs[s_][1].record()
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    ok = all(f.status()[0] == 0 for f in sets)
    keys = wl.kv_heads * wl.context * wl.head_dim * 2
    kf = int(ranks[0::2].sum()) * (wl.block_size + wl.head_dim) * 2
    vf = int(ranks[1::2].sum()) * (wl.block_size + wl.head_dim) * 2
    rest = 2 * wl.batch * wl.kv_heads * wl.suffix * wl.head_dim * 2 + 2 * wl.batch * wl.q_heads * wl.head_dim * 2
    nbytes = kf + 2 * keys + vf + rest  # rebuild reads the key factors, writes the keys; decode reads them back
    achieved = nbytes / (ms / 1e3) / 1e9
    return {"call_ms": ms, "bytes_per_step": nbytes, "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "decode_tokens_per_s": wl.batch / (ms / 1e3), "status_ok": ok,
            "note": "3 launches per call (key rebuild and rotation, decode over dense rotated keys, combine); "
                    "bytes: key factors read, rotated keys written and read back, value factors, suffix, q, out"}


def _oracle_layer(wl, L):
    """The oracle's compression of the workload's layer (fp64, stored factors as the decode reads them)."""
    import oracle
    from synth import from_storage
    dt = wl.dtype
    K, V = from_storage(L["K"], dt), from_storage(L["V"], dt)
    return oracle.compress_layer(K, V, wl.block_size, wl.budgets[0], wl.r_min)


def _save_layer(lay, path):
    """Writes the oracle layer's per-pool factors to .npy files that worker processes map read-only."""
    os.makedirs(path, exist_ok=True)
    H = len(lay["K"])
    for t in ("K", "V"):
        for h in range(H):
            pool = lay[t][h]
            np.save(os.path.join(path, f"{t}{h}_ranks.npy"), np.asarray(pool["ranks"], dtype=np.int64))
            np.save(os.path.join(path, f"{t}{h}_U.npy"), np.concatenate([u.T for u in pool["U"]], axis=0))
            np.save(os.path.join(path, f"{t}{h}_B.npy"), np.concatenate([b.T for b in pool["B"]], axis=0))
    return H


def _load_layer(path, H):
    lay = {"K": [], "V": []}
    for t in ("K", "V"):
        for h in range(H):
            ranks = np.load(os.path.join(path, f"{t}{h}_ranks.npy"))
            U = np.load(os.path.join(path, f"{t}{h}_U.npy"), mmap_mode="r")
            B = np.load(os.path.join(path, f"{t}{h}_B.npy"), mmap_mode="r")
            off = np.concatenate([[0], np.cumsum(ranks)])
            lay[t].append({"U": [np.asarray(U[a:b]).T for a, b in zip(off[:-1], off[1:])],
                           "B": [np.asarray(B[a:b]).T for a, b in zip(off[:-1], off[1:])]})
    return lay


def _cpu_worker(path, H, wl_name, k, seconds, ready, start, results):
    """One host core: decodes single queries of the workload with the oracle until `seconds` elapse."""
    try:
        try:
            from threadpoolctl import threadpool_limits
            threadpool_limits(1)
        except Exception:  # pragma: no cover
            pass
        import oracle
        from synth import WORKLOADS
        wl = WORKLOADS[wl_name]
        lay = _load_layer(path, H)
        q, Ks, Vs = (np.load(os.path.join(path, f"{x}.npy"), mmap_mode="r") for x in ("q", "K_suf", "V_suf"))
    except Exception as exc:  # pragma: no cover - reported to the parent, which stops waiting
        ready.put(("error", repr(exc)))
        return
    ready.put(("ready", k))
    start.wait()
    n = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        i = (k + n) % wl.batch
        oracle.decode_attention(np.asarray(q[i:i + 1]), lay, np.asarray(Ks[i:i + 1]), np.asarray(Vs[i:i + 1]))
        n += 1
    results.put((k, n, time.perf_counter() - t0))


def _cpu_baseline(wl, L, seconds):
    """The fp64 oracle, as it stands, on this host.  One core: whole decode steps of the batch until `seconds`
    elapse.  All cores: one process per core (spawned), each decoding single queries for `seconds`."""
    import multiprocessing as mp
    import shutil
    import tempfile

    import oracle
    from synth import from_storage
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(1)
    except Exception:  # pragma: no cover
        limiter = None
    dt = wl.dtype
    lay = _oracle_layer(wl, L)
    q = from_storage(L["q"], dt)
    Ks, Vs = from_storage(L["K_suf"], dt), from_storage(L["V_suf"], dt)
    steps = 0
    t0 = time.perf_counter()
    while True:
        oracle.decode_attention(q, lay, Ks, Vs)
        steps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    one = {"value": steps * wl.batch / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
           "sample": f"{steps} whole decode steps of {wl.name} (batch {wl.batch}) in {el:.1f} s, fp64 NumPy, "
                     f"1 BLAS thread"}
    del limiter
    cores = min(len(os.sched_getaffinity(0)), 64)
    tmp = tempfile.mkdtemp(prefix="milo_oracle_")
    try:
        H = _save_layer(lay, tmp)
        for x, a in (("q", q), ("K_suf", Ks), ("V_suf", Vs)):
            np.save(os.path.join(tmp, f"{x}.npy"), a)
        ctx = mp.get_context("spawn")
        ready, results, start = ctx.Queue(), ctx.Queue(), ctx.Event()
        procs = [ctx.Process(target=_cpu_worker, args=(tmp, H, wl.name, k, seconds, ready, start, results))
                 for k in range(cores)]
        for pr in procs:
            pr.start()
        try:
            for _ in procs:
                tag, what = ready.get(timeout=180)
                if tag == "error":
                    raise RuntimeError(f"oracle worker failed to start: {what}")
        except BaseException:
            for pr in procs:
                pr.terminate()
            raise
        start.set()
        got = [results.get(timeout=120 + 4 * seconds) for _ in procs]
        for pr in procs:
            pr.join(timeout=60)
        done = sum(n for _, n, _ in got)
        wall = max(t for _, _, t in got)
        many = {"value": done / wall, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                "sample": f"{done} single-query decodes of {wl.name} over {cores} processes (one per core, spawned, "
                          f"1 BLAS thread each) in {wall:.1f} s, fp64 NumPy"}
    except Exception as exc:  # pragma: no cover - reported, not fatal to the GPU line
        many = {"value": None, "unit": "tokens/s", "cores": cores, "kind": "oracle", "error": repr(exc)}
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    # the line's cpu_baseline is the all-core figure; the one-core figure sits beside it
    out = dict(many) if many.get("value") else dict(one)
    out["one_core"] = one
    return out


def run_reference(a):
    """The oracle timed on the host cores: `steps` bounded decode steps after `warmup` (rank 0 only)."""
    world, rank, _ = _dist()
    if rank != 0:
        return
    from synth import WORKLOADS, gen_layer
    import oracle
    from synth import from_storage
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:  # pragma: no cover
        pass
    wl = WORKLOADS[a.workload]
    L = gen_layer(wl)
    dt = wl.dtype
    K, V = from_storage(L["K"], dt), from_storage(L["V"], dt)
    lay = oracle.compress_layer(K, V, wl.block_size, wl.budgets[0], wl.r_min)
    q = from_storage(L["q"], dt)
    Ks, Vs = from_storage(L["K_suf"], dt), from_storage(L["V_suf"], dt)
    # each step decodes a bounded sample of the batch so the whole run stays within minutes
    per = max(1, min(wl.batch, int(os.environ.get("MILO_REF_ROWS", "2"))))
    for w in range(a.warmup):
        oracle.decode_attention(q[:per], lay, Ks[:per], Vs[:per])
    t0 = time.perf_counter()
    for s in range(a.steps):
        i = (s * per) % wl.batch
        sl = slice(i, min(wl.batch, i + per))
        oracle.decode_attention(q[sl], lay, Ks[sl], Vs[sl])
    el = time.perf_counter() - t0
    value = a.steps * per / el
    sample = f"{per} of {wl.batch} queries per step, fp64 NumPy oracle, 1 BLAS thread"
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * el / a.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(wl, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_milo(a):
    import torch
    world, rank, local = _dist()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    import decode_attention_milo_b200 as milo
    from synth import WORKLOADS, gen_layer
    wl = WORKLOADS[a.workload]
    dt = wl.dtype
    esize = 2 if dt == "bf16" else 4
    L = gen_layer(wl)
    dev = lambda x: _to_dev(x, dt, torch)
    Kd, Vd = dev(L["K"]), dev(L["V"])
    beta = wl.budgets[0]
    S = wl.suffix

    # --- compression, timed (one "compression" = the whole layer's K and V), with each kernel's share
    comp, kern = [], {k: [] for k in ("gram", "jacobi", "alloc", "project")}
    sweeps = None
    for i in range(4):
        st = torch.cuda.current_stream()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        for e in evs:  # torch creates the CUDA event on its first record
            e.record(st)
        torch.cuda.synchronize()
        e0.record(st)
        f = milo.compress_profiled(Kd, Vd, wl.block_size, beta, evs, wl.r_min)
        e1.record(st)
        torch.cuda.synchronize()
        if i:
            comp.append(e0.elapsed_time(e1))
            for k, name in enumerate(kern):
                kern[name].append(evs[k].elapsed_time(evs[k + 1]))
        if i == 3:
            d = f.describe()
            sweeps = _device_ints(torch, d["sweeps"], 2 * wl.kv_heads * wl.num_blocks)
            comp_ranks = f.ranks()
        f.close()

    # --- decode inputs, rotated over enough copies that the working set exceeds 3x L2
    probe = milo.compress(Kd, Vd, wl.block_size, beta, wl.r_min)
    ranks = probe.ranks()
    assert probe.status()[0] == 0
    step_bytes = _algorithmic_bytes(ranks, wl, esize)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    copies = max(2, math.ceil(3 * l2 / step_bytes))
    sets = [probe]
    for _ in range(copies - 1):
        sets.append(milo.compress(Kd, Vd, wl.block_size, beta, wl.r_min))
    del Kd, Vd
    qs = [dev(L["q"]) for _ in range(copies)]
    ks = [dev(L["K_suf"]) if S else None for _ in range(copies)]
    vs = [dev(L["V_suf"]) if S else None for _ in range(copies)]
    outs = [torch.empty_like(qs[0]) for _ in range(copies)]
    for c in range(copies):  # first call per factor object builds its work list (synchronises once)
        milo.decode_attn(qs[c], sets[c], ks[c], vs[c], out=outs[c])
    torch.cuda.synchronize()
    for f in sets:
        assert f.status()[0] == 0

    # CUDA graphs (the pages' launch-overhead remedy): one of a whole pass over the copies and one of the
    # first (steps mod copies) of them, so that warm-up and every timed window run exactly the steps asked.
    def capture(ncopies):
        if ncopies == 0:
            return None
        g_ = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            with torch.cuda.graph(g_, stream=cap):
                for c in range(ncopies):
                    milo.decode_attn(qs[c], sets[c], ks[c], vs[c], out=outs[c])
        torch.cuda.synchronize()
        return g_
    g_full = capture(copies)
    g_rest = {r: capture(r) for r in {a.steps % copies, a.warmup % copies} if r}

    def run_steps(k):
        for _ in range(k // copies):
            g_full.replay()
        if k % copies:
            g_rest[k % copies].replay()

    run_steps(a.warmup)
    torch.cuda.synchronize()
    steps = a.steps
    # repeated timed windows of `steps` steps each (the median is reported), enough of them that the clock
    # sampler sees the GPU under load for at least ~0.3 s
    probe_e = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    probe_e[0].record()
    run_steps(steps)
    probe_e[1].record()
    torch.cuda.synchronize()
    windows = max(5, min(2000, math.ceil(300.0 / max(probe_e[0].elapsed_time(probe_e[1]), 1e-3))))
    if world > 1:
        windows = int(_max_over_ranks(windows, world))
        torch.distributed.barrier()
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()
    wev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(windows)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        for e0, e1 in wev:
            e0.record(st)
            run_steps(steps)
            e1.record(st)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = _max_over_ranks(statistics.median(e0.elapsed_time(e1) for e0, e1 in wev), world)
    ms_step = ms / steps
    value = _job_value(world, wl.batch, steps, ms)
    per_call_ms = ms_step  # every step is one milo_decode_attn call
    kernels_per_call = sets[0].decode_launches(wl.batch, wl.q_heads, S)

    # --- the main decode kernel alone: events recorded by the library right around it, eager launches
    kt_steps = min(steps, 300)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(kt_steps)]
    for a_, b_ in evs:  # create the CUDA events (torch creates them lazily on first record)
        a_.record()
        b_.record()
    for s_ in range(kt_steps):
        c = s_ % copies
        milo.decode_attn_profiled(qs[c], sets[c], ks[c], vs[c], outs[c], evs[s_][0], evs[s_][1])
    torch.cuda.synchronize()
    kernel_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    peak, peak_kind = _peaks()
    dec8 = _decode_8bit(torch, milo, wl, sets, qs, ks, vs, outs, steps, peak) if dt == "bf16" else None
    decr = _decode_rope(torch, milo, wl, sets, qs, ks, vs, outs, steps, peak, ranks) if dt == "bf16" else None

    # --- end to end through the public API: pinned host inputs, copies inside the timed region.  Steps
    # alternate between two streams with their own device buffers, so the host-to-device copies of one
    # step overlap the decode of the previous one (as a serving loop would run them).
    ht = torch.int16 if dt == "bf16" else torch.float32
    hq = torch.from_numpy(np.ascontiguousarray(L["q"]).view(np.int16 if dt == "bf16" else np.float32)).pin_memory()
    hk = torch.from_numpy(np.ascontiguousarray(L["K_suf"]).view(np.int16 if dt == "bf16" else np.float32)).pin_memory()
    hv = torch.from_numpy(np.ascontiguousarray(L["V_suf"]).view(np.int16 if dt == "bf16" else np.float32)).pin_memory()
    houts = [torch.empty(qs[0].shape, dtype=ht).pin_memory() for _ in range(2)]
    e2e_steps = min(steps, 500)
    lanes = [torch.cuda.Stream() for _ in range(2)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(st)
    for ln in lanes:
        ln.wait_stream(st)
    for s_ in range(e2e_steps):
        c = s_ % 2
        ln = lanes[c]
        with torch.cuda.stream(ln):
            qd = qs[c].view(ht)
            qd.copy_(hq, non_blocking=True)
            if S:
                ks[c].view(ht).copy_(hk, non_blocking=True)
                vs[c].view(ht).copy_(hv, non_blocking=True)
            milo.decode_attn(qs[c], sets[c], ks[c], vs[c], out=outs[c], stream=ln)
            houts[c].copy_(outs[c].view(ht), non_blocking=True)
    for ln in lanes:
        st.wait_stream(ln)
    f1.record(st)
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(f0.elapsed_time(f1), world)
    hout = houts[0]
    h2d = hq.numel() * hq.element_size() + (2 * hk.numel() * hk.element_size() if S else 0)
    d2h = hout.numel() * hout.element_size()

    achieved = step_bytes / (kernel_ms / 1e3) / 1e9
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = _cpu_baseline(wl, L, a.cpu_seconds)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": a.warmup, "ms_per_step": ms_step, "timed_windows": windows, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": dt, "data": "synthetic",
            "config": _config(wl, world, ranks.sum(),
                              l2=f"inputs rotated over {copies} copies ({copies * step_bytes / 1e6:.0f} MB > 3x L2)",
                              launch="CUDA graphs over the copies; median of the timed windows"),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": DECODE_TRAFFIC.get((wl.name, _source_digest())),
                         "peak_kind": peak_kind,
                         "bytes_per_step": step_bytes, "kernel": "decode_tc_kernel" if dt == "bf16" else
                         "prefix_kernel", "kernel_ms": kernel_ms, "call_ms": per_call_ms,
                         "note": "achieved = algorithmic bytes per step / mean CUDA-event duration of the main "
                                 "decode kernel (events recorded by the library right before and after it, "
                                 f"{kt_steps} eager launches over the rotated copies)"},
            "e2e": {"value": _job_value(world, wl.batch, e2e_steps, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "compress": {"compressions_per_s": 1e3 / statistics.median(comp), "ms": statistics.median(comp),
                         "unit": "whole-layer compressions/s",
                         "roofline": _compress_roofline(torch, wl, esize, comp_ranks, sweeps, kern, peak)},
            "decode_8bit": dec8,
            "decode_pre_rope": decr,
            "gpu_launches": kernels_per_call * steps,
            "gpu_launches_note": f"{kernels_per_call} kernels per decode call x {steps} steps of one timed window "
                                 f"({windows} windows timed, the median reported)",
            "clocks": clk.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    del g_full, g_rest
    for f in sets:
        f.close()
    if world > 1:
        torch.distributed.destroy_process_group()


def run_profile(a):
    """N eager calls of one phase on one GPU: what an ncu capture of that phase's kernels runs."""
    import torch
    torch.cuda.set_device(0)
    import decode_attention_milo_b200 as milo
    from synth import WORKLOADS, gen_layer
    wl = WORKLOADS[a.workload]
    dt = wl.dtype
    L = gen_layer(wl)
    dev = lambda x: _to_dev(x, dt, torch)
    Kd, Vd = dev(L["K"]), dev(L["V"])
    beta = wl.budgets[0]
    t0 = time.time()
    if a.profile == "compress":
        for _ in range(a.calls):
            f = milo.compress(Kd, Vd, wl.block_size, beta, wl.r_min)
            torch.cuda.synchronize()
            assert f.status()[0] == 0
            f.close()
    else:
        f = milo.compress(Kd, Vd, wl.block_size, beta, wl.r_min)
        if a.profile == "decode8":
            f8 = milo.quantize(f)
            f.close()
            f = f8
        q = dev(L["q"])
        ks = dev(L["K_suf"]) if wl.suffix else None
        vs = dev(L["V_suf"]) if wl.suffix else None
        out = torch.empty_like(q)
        for _ in range(a.calls):
            if a.profile == "rope":
                milo.decode_attn_rope(q, f, ks, vs, theta=1e6, out=out)
            else:
                milo.decode_attn(q, f, ks, vs, out=out)
        torch.cuda.synchronize()
        assert f.status()[0] == 0
        f.close()
    print(json.dumps({"profile": a.profile, "workload": wl.name, "calls": a.calls, "wall_s": time.time() - t0}))


def main():
    a = _args()
    if a.profile:
        run_profile(a)
        return
    if a.impl == "reference":
        run_reference(a)
    else:
        run_milo(a)


if __name__ == "__main__":
    main()
