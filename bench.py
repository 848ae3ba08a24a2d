#!/usr/bin/env python
"""Benchmark of Flint's sink-aware attention (forward + backward) on B200.

One step = the whole hot path over one batch: RMSNorm+RoPE prologue, work
list, tcgen05 attention forward, backward preprocess (D, d_sink), tcgen05
backward (dK/dV and dQ) and the prologue backward - both C-ABI calls
(flint_attn_fwd, flint_attn_bwd). The metric counts masked FLOPs: 4*D*H*pairs
for the forward and 10*D*H*pairs for the backward (five GEMMs).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

The default workload is the 32768-token full-causal layer (32/4 heads). Other
workloads: ``--workload bshd_padded_bf16_B8_S8192_H32x4_W1024`` (the padded
calls, FLOPs over real tokens) and ``--workload decode_bf16_B64_C8192_H32x4_W4096``
(flint_attn_decode; metric: K/V bytes read per second, roofline against HBM).
``--impl reference`` times the FP64 oracle on the host cores for the same
workload and metric.

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch
(replicas, weak scaling); no data-path collective exists in this path. The
step time is the max over ranks of CUDA-event time. Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import flint_inputs as fi  # noqa: E402

METRIC = "sink-attention fwd/bwd TFLOP/s (masked FLOPs) and % of B200 BF16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
WORKLOADS = {w.name: w for w in fi.WORKLOADS}
DECODE_WORKLOADS = {w.name: w for w in [fi.DECODE_SLIDING_BF16]}
DECODE_METRIC = "decode step: KV-cache bytes read per second (one new token per sequence)"
DEFAULT_WORKLOAD = fi.FULL_BF16.name
L2_FLUSH_BYTES = 256 << 20


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="flint", choices=["flint", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS),
                    help="the default is the fwd+bwd layer the headline metric is quoted "
                         "on; decode_* workloads time flint_attn_decode instead")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="also time the step replayed from a CUDA graph (the forward and "
                         "backward calls captured once), reported under 'graph'")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--tokens", type=int, default=0,
                    help="run the workload as one document of this many tokens (smaller "
                         "cases for profiler captures); 0 keeps the workload's size")
    return ap.parse_args(argv)


# --------------------------------------------------------------------------- helpers

def real_lens(inp):
    """Real tokens per document (all of it unless the workload has padding)."""
    if "valid_lens" in inp:
        return [int(x) for x in inp["valid_lens"]]
    return list(inp["doc_lens"])


def visible_pairs(doc_lens, window: int) -> int:
    """Masked FLOP accounting: (query, key) pairs per head under the causal document
    mask whose window includes the current token (row i of a document sees min(i + 1, W)
    keys)."""
    total = 0
    for L in doc_lens:
        L = int(L)
        if window <= 0 or window >= L:
            total += L * (L + 1) // 2
        else:
            W = int(window)
            # rows 0..W-1 see i+1 keys, the rest see W keys
            total += W * (W + 1) // 2 + (L - W) * W
    return total


def decode_kv_bytes(cache_lens, window: int, num_kv_heads: int, head_dim: int = 128) -> int:
    """Bytes of K and V (bf16) the decode step reads: every visible slot, once."""
    total = 0
    for p in cache_lens:
        p = int(p)
        n = p + 1 if window <= 0 else min(p + 1, int(window))
        total += n
    return total * num_kv_heads * head_dim * 2 * 2


def flops_of(doc_lens, window, H, D=128):
    pairs = visible_pairs(doc_lens, window)
    return pairs, 4.0 * D * H * pairs, 10.0 * D * H * pairs


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def config_of(w, pairs, flops_step):
    return {
        "workload": f"{w.name} fwd+bwd",
        "tokens": w.total_tokens,
        "docs": "drawn U[128,8192]" if w.doc_lens is None else len(w.doc_lens),
        "padding": (f"trailing, real tokens per document drawn U{list(w.valid_range)}; "
                    "masked FLOPs count real tokens only") if w.valid_range else None,
        "heads_q": w.num_q_heads, "heads_kv": w.num_kv_heads, "head_dim": w.head_dim,
        "window": w.window if w.window > 0 else "full causal",
        "rope": bool(w.use_rope), "rope_theta": w.rope_theta if w.use_rope else None,
        "sink_std": w.sink_std,
        "masked_pairs_per_head": pairs, "flops_per_step": flops_step,
        "l2": "inputs larger than L2 (126 MB), plus a 256 MB L2 flush before every step",
        "parallelism": "replicas (one independent batch per GPU)",
        "outputs": "O, dq, dk, dv in float32 (fp32_out); LSE, dw_q, dw_k, d_sink float32",
    }


class ClockSampler:
    """nvidia-smi clock/throttle samples taken while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.proc = None
        self.path = os.path.join("/tmp", f"flint_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # nvidia-smi's start-up (driver and NVML initialisation) can hold up this
        # process's launches for a second or more; a step that short would time the
        # stall. Start timing once the first sample is written (at most 10 s).
        t_end = time.time() + 10.0
        while time.time() < t_end and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self, device_index=None):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    idx, clk, cmax, pw = int(parts[0]), float(parts[1]), float(parts[2]), float(parts[3])
                except ValueError:
                    continue
                if device_index is not None and idx != device_index:
                    continue
                mx = max(mx, cmax)
                if pw > 250.0:          # under load
                    sm.append(clk)
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples_under_load": len(sm)}


def kernel_source_sha(name):
    """Fingerprint of a kernel source's code: // comments and blank lines are left out,
    so recorded profiler counters stay attached to the code they measured."""
    path = os.path.join(ROOT, "sink_aware_sliding_head_b200", "csrc", name)
    try:
        with open(path) as f:
            lines = [ln.split("//", 1)[0].rstrip() for ln in f]
    except OSError:
        return None
    code = "\n".join(ln for ln in lines if ln)
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def traffic_for(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            entries = json.load(f)
    except Exception:
        return None
    for e in entries:
        if e.get("kernel") == kernel and e.get("workload") == workload and \
                e.get("source_sha") == kernel_source_sha(e.get("source", "")):
            return e.get("dram_bytes_per_launch")
    return None


def aggregate(times_ms, world, flops_step, steps, pg=None):
    """Whole-job numbers from this rank's CUDA-event times.

    times_ms: this rank's [total, fwd, bwd] milliseconds over `steps` steps. The
    slowest rank defines the step time (max over ranks through `pg`, any
    torch.distributed backend); every rank processed its own batch (weak
    scaling), so the job's throughput is world * flops_step * steps / time.
    Returns (value TFLOP/s, [total, fwd, bwd] ms maxed over ranks).
    """
    t = torch.tensor(list(times_ms), dtype=torch.float64)
    if pg is not None:
        dev = torch.device("cuda", torch.cuda.current_device()) if \
            pg.get_backend() == "nccl" else torch.device("cpu")
        t = t.to(dev)
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
    t = [float(x) for x in t.cpu().tolist()]
    return world * flops_step * steps / (t[0] * 1e-3) / 1e12, t


# --------------------------------------------------------------------------- CPU oracle

def oracle_sample(w, inp, seconds):
    """Time the FP64 oracle fwd+bwd on a prefix of the workload sized for ~seconds.

    Returns (flops, wall seconds, description). The prefix keeps the workload's
    heads, window and RoPE; for packed workloads it takes whole leading documents.
    """
    from oracle import flint_oracle as fo   # test infrastructure: CPU baseline leg only

    if "valid_lens" in inp:
        # the real tokens alone: the padded layer's real rows are exactly this layer
        idx, cu_v = [], [0]
        for d, (a, b) in enumerate(zip(inp["cu_doc_lens"][:-1].tolist(),
                                       inp["cu_doc_lens"][1:].tolist())):
            n = min(int(inp["valid_lens"][d]), b - a)
            idx.extend(range(a, a + n))
            cu_v.append(cu_v[-1] + n)
        idx = torch.tensor(idx)
        inp = dict(inp, q=inp["q"][idx], k=inp["k"][idx], v=inp["v"][idx],
                   dout=inp["dout"][idx], cu_doc_lens=torch.tensor(cu_v, dtype=torch.int32))

    def run(n_tok):
        cu = [int(c) for c in inp["cu_doc_lens"]]
        lens, acc = [], 0
        for a, b in zip(cu[:-1], cu[1:]):
            if acc >= n_tok:
                break
            take = min(b - a, n_tok - acc)
            lens.append(take)
            acc += take
        n_tok = acc
        cu_p = [0]
        for L in lens:
            cu_p.append(cu_p[-1] + L)
        sl = slice(0, n_tok)
        t0 = time.perf_counter()
        fo.flint_attn_bwd(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["w_q"], inp["w_k"],
                          inp["sink"], cu_p, w.window, w.use_rope, w.rope_theta, inp["dout"][sl])
        fo.flint_attn_fwd(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["w_q"], inp["w_k"],
                          inp["sink"], cu_p, w.window, w.use_rope, w.rope_theta)
        dt = time.perf_counter() - t0
        pairs, ff, fb = flops_of(lens, w.window, w.num_q_heads)
        return ff + fb, dt, n_tok

    f0, t0, n0 = run(256)
    # work grows ~quadratically (full causal) or linearly (windowed) with the prefix
    grow = 2.0 if w.window <= 0 else 1.0
    n = int(256 * max(1.0, seconds / max(t0, 1e-3)) ** (1.0 / grow))
    n = max(256, min(w.total_tokens, (n // 128) * 128))
    f, t, n = run(n)
    desc = (f"oracle fwd+bwd (FP64 NumPy) on the first {n} tokens of {w.name} "
            f"({w.num_q_heads}/{w.num_kv_heads} heads, same window/RoPE); masked FLOPs of that prefix")
    return f, t, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# --------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    inp = fi.make_inputs(w, with_grad_out=True)
    pairs, ff, fb = flops_of(real_lens(inp), w.window, w.num_q_heads)
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    total_f, total_t, desc = 0.0, 0.0, ""
    for i in range(args.warmup + args.steps):
        f, t, desc = oracle_sample(w, inp, per_step)
        if i >= args.warmup:
            total_f += f
            total_t += t
    value = total_f / total_t / 1e12
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, pairs, ff + fb),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- GPU arm

def decode_config(w, lens, kv_bytes):
    return {"workload": f"{w.name} decode step", "batch": w.batch,
            "cache_capacity": w.cache_capacity, "cache_lens": f"drawn U{list(w.lens_range)}",
            "mean_cache_len": sum(int(x) for x in lens) / len(lens),
            "heads_q": w.num_q_heads, "heads_kv": w.num_kv_heads, "head_dim": w.head_dim,
            "window": w.window if w.window > 0 else "unbounded", "rope": bool(w.use_rope),
            "kv_bytes_per_step": kv_bytes,
            "l2": "K/V windows (~0.5 GB) larger than L2, plus a 256 MB L2 flush before every step",
            "parallelism": "replicas (one independent batch per GPU)"}


def oracle_decode_sample(w, inp, seconds):
    """Time the FP64 decode oracle on leading sequences for ~seconds; returns (bytes, s, desc)."""
    from oracle import flint_oracle as fo   # test infrastructure: CPU baseline leg only

    def run(nb):
        sl = slice(0, nb)
        t0 = time.perf_counter()
        fo.decode(inp["q"][sl], inp["k"][sl], inp["v"][sl], inp["w_q"], inp["w_k"], inp["sink"],
                  inp["cache_lens"][sl], inp["k_cache"][sl], inp["v_cache"][sl], w.window,
                  w.use_rope, w.rope_theta)
        dt = time.perf_counter() - t0
        return decode_kv_bytes(inp["cache_lens"][sl].tolist(), w.window, w.num_kv_heads), dt

    b0, t0 = run(1)
    nb = max(1, min(w.batch, int(seconds / max(t0, 1e-3))))
    b, t = run(nb)
    return b, t, (f"oracle decode (FP64 NumPy) on the first {nb} of {w.batch} sequences of "
                  f"{w.name}; K/V bytes of those sequences")


def run_reference_decode(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return
    w = DECODE_WORKLOADS[args.workload]
    inp = fi.make_decode_inputs(w)
    lens = inp["cache_lens"].tolist()
    per_step = max(1.0, min(10.0, 120.0 / max(1, args.steps + args.warmup)))
    tb, tt, desc = 0, 0.0, ""
    for i in range(args.warmup + args.steps):
        b, t, desc = oracle_decode_sample(w, inp, per_step)
        if i >= args.warmup:
            tb += b
            tt += t
    value = tb / tt / 1e9
    line = {"impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(w, lens, decode_kv_bytes(lens, w.window, w.num_kv_heads)),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_decode(args):
    """flint_attn_decode on the serving shape: K/V bytes read per second."""
    from sink_aware_sliding_head_b200 import flint_attn as fa
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
        pg = dist
    w = DECODE_WORKLOADS[args.workload]
    cpu = fi.make_decode_inputs(w, seed=w.seed + rank)
    lens = cpu["cache_lens"].tolist()
    kv_bytes = decode_kv_bytes(lens, w.window, w.num_kv_heads)
    d = {k: v.to(dev) for k, v in cpu.items()}
    B, H, D = d["q"].shape
    p = fa.decode_params(B, w.cache_capacity, H, w.num_kv_heads, w.window, w.use_rope,
                         w.rope_theta)
    lib = fa.load_library()
    import ctypes
    ws = torch.empty(lib.flint_attn_decode_workspace_bytes(ctypes.byref(p)),
                     dtype=torch.uint8, device=dev)
    out = torch.empty(B, H, D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(B, H, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def call(src):
        # writing the new token's slot again with the same values keeps every step identical
        fa.decode(src["q"], src["k"], src["v"], src["w_q"], src["w_k"], src["sink"],
                  src["cache_lens"], d["k_cache"], d["v_cache"], w.window, w.use_rope,
                  w.rope_theta, out=out, lse=lse, workspace=ws)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        call(d)
    torch.cuda.synchronize(dev)
    code = lib.flint_attn_check_status(fa._ptr(ws), fa._stream_ptr())
    if code != 0:
        raise RuntimeError(f"device status {fa.STATUS.get(code, code)} during warm-up")
    # timed region: plain calls (a decode step is ~0.1 ms, so per-kernel profiling
    # events would distort it); the per-kernel split comes from a separate pass
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    clocks = ClockSampler() if rank == 0 else None
    if clocks:
        clocks.start()
    n0 = fa.launch_count()
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        call(d)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    if pg is not None:
        pg.barrier()
    launches = fa.launch_count() - n0
    clk = clocks.stop(local) if clocks else None
    t_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    fa.profile_reset()
    fa.profile_collect()
    fa.profile_reset()
    fa.profile_enable(True)
    for i in range(min(args.steps, 50)):
        flush.zero_()
        call(d)
    torch.cuda.synchronize(dev)
    fa.profile_enable(False)
    kern = fa.profile_collect()
    t = torch.tensor([t_ms], dtype=torch.float64)
    if pg is not None:
        t = t.to(dev)
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
    t_ms = float(t.cpu()[0])
    value = world * kv_bytes * args.steps / (t_ms * 1e-3) / 1e9

    # end to end: the new tokens' q, k, v and cache_lens in from pinned host memory,
    # out and LSE back, every step (the caches are device-resident serving state)
    names_in = ["q", "k", "v", "w_q", "w_k", "sink", "cache_lens"]
    host_in = {k: cpu[k].pin_memory() for k in names_in}
    dev_in = {k: torch.empty_like(d[k]) for k in names_in}
    host_out = {"out": torch.empty(out.shape, dtype=out.dtype, pin_memory=True),
                "lse": torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)}
    h2d = sum(x.numel() * x.element_size() for x in host_in.values())
    d2h = sum(x.numel() * x.element_size() for x in host_out.values())

    def e2e_step():
        for k in names_in:
            dev_in[k].copy_(host_in[k], non_blocking=True)
        call(dev_in)
        host_out["out"].copy_(out, non_blocking=True)
        host_out["lse"].copy_(lse, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    te = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64)
    if pg is not None:
        te = te.to(dev)
        pg.all_reduce(te, op=pg.ReduceOp.MAX)
    te_ms = float(te.cpu()[0])
    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return
    peaks, peak_src = read_peaks()
    attn = kern.get("decode", (0.0, 0))
    per_launch = attn[0] / max(attn[1], 1)
    achieved = kv_bytes / (per_launch * 1e-3) / 1e9 if attn[1] else None
    roofline = {"kernel": "decode", "bound": "hbm", "achieved": achieved,
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": (achieved or 0.0) / peaks["hbm_gbs"],
                "peak_kind": f"HBM copy bandwidth ({peak_src})",
                "traffic": traffic_for("decode", w.name),
                "algorithmic_bytes_per_launch": kv_bytes, "ms_per_launch": per_launch,
                "source": "decode.cu"}
    cpu_baseline = None
    if world == 1 and not args.no_cpu_baseline:
        b, tc, desc = oracle_decode_sample(w, cpu, min(args.cpu_seconds, 10.0))
        cpu_baseline = {"value": b / tc / 1e9, "unit": "GB/s", "cores": blas_threads(),
                        "kind": "oracle", "sample": desc, "seconds": tc}
    line = {
        "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) caches and new-token q/k/v, FP32 sinks)",
        "config": decode_config(w, lens, kv_bytes),
        "tokens_per_s": world * B * args.steps / (t_ms * 1e-3),
        "roofline": roofline,
        "kernels": {k: {"ms_per_launch": v[0] / v[1], "launches_profiled": v[1]}
                    for k, v in kern.items() if v[1] > 0},
        "gpu_launches": launches, "clocks": clk,
        "e2e": {"value": world * kv_bytes * args.steps / (te_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": te_ms / args.steps},
        "cpu_baseline": cpu_baseline,
    }
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


def main(argv=None):
    args = parse_args(argv)
    if args.workload in DECODE_WORKLOADS:
        if args.impl == "reference":
            run_reference_decode(args)
        else:
            run_decode(args)
        return
    if args.impl == "reference":
        run_reference(args)
        return
    from sink_aware_sliding_head_b200 import flint_attn as fa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    w = WORKLOADS[args.workload]
    # FP32 inputs run the split tensor-core kernels (fp16 hi/lo operands, three MMAs
    # per product); BF16 inputs the fp16-operand ones
    split = w.dtype == "fp32"
    fwd_name = "attn_fwd_x3_sm100" if split else "attn_fwd_sm100"
    if args.tokens > 0:
        import dataclasses
        w = dataclasses.replace(w, name=f"{w.name}@{args.tokens}", doc_lens=(args.tokens,),
                                total_tokens=args.tokens, drawn_len_range=None)
    cpu = fi.make_inputs(w, seed=w.seed + rank, with_grad_out=True)
    pairs, ff, fb = flops_of(real_lens(cpu), w.window, w.num_q_heads)
    flops_step = ff + fb
    d = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in cpu.items()}
    T, H, D = d["q"].shape
    p = fa.params_for(d["q"], d["k"], d["cu_doc_lens"], w.window, w.use_rope, w.rope_theta,
                      fp32_out=True)
    ws_f = fa.alloc_workspace(p, False, dev)
    ws_b = fa.alloc_workspace(p, True, dev)
    out = torch.empty(d["q"].shape, dtype=torch.float32, device=dev)
    lse = torch.empty(H, T, dtype=torch.float32, device=dev)
    # O and the gradients w.r.t. q, k, v in float32 (fp32_out): the configuration
    # the parity tests hold to max-abs 2e-2; bfloat16 storage alone exceeds that
    # for |grad| > 10, and bf16 O feeds D = dO . O of the sink gradient
    f32 = torch.float32
    grads = {"dq": torch.empty(d["q"].shape, dtype=f32, device=dev),
             "dk": torch.empty(d["k"].shape, dtype=f32, device=dev),
             "dv": torch.empty(d["v"].shape, dtype=f32, device=dev),
             "dw_q": torch.empty(D, dtype=torch.float32, device=dev),
             "dw_k": torch.empty(D, dtype=torch.float32, device=dev),
             "dsink": torch.empty(H, dtype=torch.float32, device=dev)}
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fwd_call(src, o=None, l=None):
        fa.fwd(src["q"], src["k"], src["v"], src["w_q"], src["w_k"], src["sink"],
               src["cu_doc_lens"], w.window, w.use_rope, w.rope_theta,
               out=out if o is None else o, lse=lse if l is None else l,
               workspace=ws_f, fp32_out=True, valid_lens=src.get("valid_lens"))

    def bwd_call(src, o=None, l=None, g=None):
        fa.bwd(src["q"], src["k"], src["v"], src["w_q"], src["w_k"], src["sink"],
               src["cu_doc_lens"], out if o is None else o, lse if l is None else l,
               src["dout"], w.window, w.use_rope, w.rope_theta,
               grads=grads if g is None else g, workspace=ws_b, fp32_out=True,
               valid_lens=src.get("valid_lens"))

    # ---- warm-up (also surfaces device-side timeouts before timing)
    for _ in range(args.warmup):
        flush.zero_()
        fwd_call(d)
        bwd_call(d)
    torch.cuda.synchronize(dev)
    lib = fa.load_library()
    for ws in (ws_f, ws_b):
        code = lib.flint_attn_check_status(fa._ptr(ws), fa._stream_ptr())
        if code != 0:
            raise RuntimeError(f"device status {fa.STATUS.get(code, code)} during warm-up")

    # ---- timed region: device-resident inputs
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler() if rank == 0 else None
    if clocks:
        clocks.start()
    fa.profile_reset()
    fa.profile_collect()
    fa.profile_reset()
    fa.profile_enable(True)
    n0 = fa.launch_count()
    barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        fwd_call(d)
        ev[i][1].record(stream)
        bwd_call(d)
        ev[i][2].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    launches = fa.launch_count() - n0
    fa.profile_enable(False)
    kern = fa.profile_collect()
    clk = clocks.stop() if clocks else None
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in ev)
    value, (tot_ms, fwd_ms, bwd_ms) = aggregate([fwd_ms + bwd_ms, fwd_ms, bwd_ms], world,
                                                flops_step, args.steps, pg)
    ms_step = tot_ms / args.steps

    # ---- the same step replayed from a CUDA graph (both calls captured once): the
    # launch overhead of the ~17 kernels per step drops out
    graph = None
    if args.graph:
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fwd_call(d)
            bwd_call(d)
        stream.wait_stream(side)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fwd_call(d)
            bwd_call(d)
        for _ in range(args.warmup):
            flush.zero_()
            g.replay()
        torch.cuda.synchronize(dev)
        gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
               for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.zero_()
            gev[i][0].record(stream)
            g.replay()
            gev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        g_val, (g_ms,) = aggregate([sum(e[0].elapsed_time(e[1]) for e in gev)], world,
                                   flops_step, args.steps, pg)
        graph = {"value": g_val, "unit": UNIT, "ms_per_step": g_ms / args.steps,
                 "note": "flint_attn_fwd + flint_attn_bwd captured once in a CUDA graph and "
                         "replayed, same inputs, same L2 flush before each step"}
        del g

    # ---- end to end: host (pinned) inputs -> device -> both calls -> host results.
    # Every step copies its inputs in and all its results (O, LSE, dq, dk, dv,
    # dw_q, dw_k, d_sink) out. The copies run on their own streams, double
    # buffered, so step i's compute overlaps the copy-in of step i+1 and the
    # copy-out of step i-1 (PCIe in both directions at once), as a training loop
    # that streams its batches would run it. Within a step, dO (read only by the
    # backward) is copied in while the forward runs, and O and LSE (final once
    # the forward ends) are copied out while the backward runs. The timed region
    # spans the first copy-in to the last copy-out.
    e2e = None
    if not args.no_e2e:
        names_fwd = ["q", "k", "v", "w_q", "w_k", "sink", "cu_doc_lens"]
        if "valid_lens" in cpu:
            names_fwd.append("valid_lens")
        names_in = names_fwd + ["dout"]
        host_in = [{k: cpu[k].pin_memory() for k in names_in} for _ in range(2)]
        dev_in = [{k: torch.empty_like(d[k]) for k in names_in} for _ in range(2)]
        dev_out = [{"out": out, "lse": lse, **grads}]
        dev_out.append({k: torch.empty_like(v) for k, v in dev_out[0].items()})
        host_out = [{k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                     for k, v in dev_out[0].items()} for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host_in[0].values())
        d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
        s_in = torch.cuda.Stream(dev)
        s_out = torch.cuda.Stream(dev)

        def e2e_run(n):
            """n pipelined steps; returns (start, end) events on the compute stream."""
            comp_done = [None, None]     # buffer b's inputs free / outputs written
            out_done = [None, None]      # buffer b's outputs copied to the host
            e_start = torch.cuda.Event(enable_timing=True)
            e_end = torch.cuda.Event(enable_timing=True)
            e_start.record(stream)
            s_in.wait_stream(stream)
            s_out.wait_stream(stream)
            for i in range(n):
                b = i & 1
                with torch.cuda.stream(s_in):
                    if comp_done[b] is not None:
                        s_in.wait_event(comp_done[b])
                    for k in names_fwd:
                        dev_in[b][k].copy_(host_in[b][k], non_blocking=True)
                    in_fwd = torch.cuda.Event()
                    in_fwd.record(s_in)
                    dev_in[b]["dout"].copy_(host_in[b]["dout"], non_blocking=True)
                    in_bwd = torch.cuda.Event()
                    in_bwd.record(s_in)
                stream.wait_event(in_fwd)
                if out_done[b] is not None:
                    stream.wait_event(out_done[b])
                o = dev_out[b]
                fwd_call(dev_in[b], o["out"], o["lse"])
                fwd_done = torch.cuda.Event()
                fwd_done.record(stream)
                stream.wait_event(in_bwd)
                bwd_call(dev_in[b], o["out"], o["lse"], o)
                comp_done[b] = torch.cuda.Event()
                comp_done[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(fwd_done)
                    for k in ("out", "lse"):
                        host_out[b][k].copy_(o[k], non_blocking=True)
                    s_out.wait_event(comp_done[b])
                    for k, v in o.items():
                        if k not in ("out", "lse"):
                            host_out[b][k].copy_(v, non_blocking=True)
                    out_done[b] = torch.cuda.Event()
                    out_done[b].record(s_out)
            stream.wait_stream(s_in)
            stream.wait_stream(s_out)
            e_end.record(stream)
            return e_start, e_end

        e2e_run(max(1, args.warmup))
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = e2e_run(args.steps)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_val, (t_e2e,) = aggregate([e0.elapsed_time(e1)], world, flops_step, args.steps, pg)
        e2e = {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": t_e2e / args.steps,
               "copies": "pinned host buffers; copy-in and copy-out on their own streams, "
                         "double buffered, overlapping the neighbouring steps' compute; dO "
                         "copied in during the forward, O and LSE copied out during the "
                         "backward"}

    # ---- the forward on its own (the layer's forward is the configuration whose
    # tensor-peak fraction is the target): the same calls, no backward in between,
    # so the clock is the forward's own rather than the power-capped step's
    fwd_only = None
    if ff > 0:
        fa.profile_reset()
        fa.profile_collect()
        fa.profile_reset()
        clocks_f = ClockSampler() if rank == 0 else None
        if clocks_f:
            clocks_f.start()
        fa.profile_enable(True)
        fo_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
                 for _ in range(args.steps)]
        barrier()
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.zero_()
            fo_ev[i][0].record(stream)
            fwd_call(d)
            fo_ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        fa.profile_enable(False)
        kf = fa.profile_collect()
        clk_f = clocks_f.stop() if clocks_f else None
        call_ms = sum(e[0].elapsed_time(e[1]) for e in fo_ev) / args.steps
        kms = kf.get(fwd_name, (0.0, 0))
        fwd_only = {
            "ms_per_call": call_ms,
            "call_tflops": ff / (call_ms * 1e-3) / 1e12,
            "kernel_ms": kms[0] / max(kms[1], 1),
            "kernel_tflops": (4.0 * D * H * pairs / (kms[0] / kms[1] * 1e-3) / 1e12
                              if kms[1] else None),
            "clocks": clk_f,
            "note": "flint_attn_fwd alone, the same steps with an L2 flush before each call"}

    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return

    # ---- roofline of the dominant kernel (live CUDA-event time per launch)
    peaks, peak_src = read_peaks()
    # bytes per element of the prologue's rows: bf16 in, fp16 q_hat / k_hat out; or
    # FP32 in, fp16 hi + lo parts out
    eb = 4 if split else 2
    algo = {  # algorithmic (useful) work per launch
        "attn_fwd_sm100": ("tensor", 4.0 * D * H * pairs),
        "attn_bwd_dkv_sm100": ("tensor", 8.0 * D * H * pairs),
        "attn_bwd_dq_sm100": ("tensor", 2.0 * D * H * pairs),
        "attn_fwd_x3_sm100": ("tensor", 4.0 * D * H * pairs),
        "attn_bwd_dkv_x3_sm100": ("tensor", 8.0 * D * H * pairs),
        "attn_bwd_dq_x3_sm100": ("tensor", 2.0 * D * H * pairs),
    }
    dom = max(kern.items(), key=lambda kv: kv[1][0])
    dname, (dms, dn) = dom
    per_launch_ms = dms / max(dn, 1)
    roofline = None
    if dname in algo:
        achieved = algo[dname][1] / (per_launch_ms * 1e-3) / 1e12
        # the split kernels issue three f16 MMAs per useful product: their useful-work
        # ceiling is a third of the f16/bf16 tensor peak
        mmas = 3.0 if "_x3_" in dname else 1.0
        peak = peaks["bf16_tflops"] / mmas
        src = {"attn_fwd_sm100": "attn_fwd_sm100.cu"}.get(
            dname, "attn_x3_sm100.cu" if mmas > 1 else "attn_bwd_sm100.cu")
        roofline = {"kernel": dname, "bound": "tensor", "achieved": achieved, "peak": peak,
                    "unit": "TFLOP/s", "frac": achieved / peak,
                    "peak_kind": f"bf16 burst ({peak_src})" +
                                 (" / 3 (three MMAs per product)" if mmas > 1 else "") +
                                 "; the kernel runs inside a power-capped step, see "
                                 "frac_of_sustained",
                    "frac_of_sustained": achieved * mmas / peaks["bf16_tflops_sustained"],
                    "peak_sustained": peaks["bf16_tflops_sustained"] / mmas,
                    "traffic": traffic_for(dname, w.name),
                    "algorithmic_flops_per_launch": algo[dname][1],
                    "ms_per_launch": per_launch_ms, "source": src}
    # ---- roofline of the HBM-bound prologue (RMSNorm + RoPE of q and k in one
    # launch): it reads the raw rows and writes the normalised ones,
    # 2 * (H + Hk) * D * 2 bytes per token (real tokens and padding alike)
    roofline_hbm = None
    pro = kern.get("prologue_rmsnorm_rope", (0.0, 0))
    if pro[1] >= 1:
        pair_bytes = 2.0 * (H + w.num_kv_heads) * D * eb * T
        pair_ms = pro[0] / pro[1]
        achieved = pair_bytes / (pair_ms * 1e-3) / 1e9
        roofline_hbm = {"kernel": "prologue_rmsnorm_rope", "bound": "hbm", "achieved": achieved,
                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": achieved / peaks["hbm_gbs"],
                        "peak_kind": f"HBM copy bandwidth ({peak_src})",
                        "traffic": traffic_for("prologue_rmsnorm_rope", w.name),
                        "algorithmic_bytes_per_launch": pair_bytes,
                        "bytes_per_token": pair_bytes / T, "ms_per_launch": pair_ms,
                        "source": "prologue.cu"}
    kernels = {k: {"ms_per_step": v[0] / args.steps, "launches": v[1],
                   "share": v[0] / max(sum(x[0] for x in kern.values()), 1e-9)}
               for k, v in kern.items() if v[1] > 0}
    fwd_attn = kern.get(fwd_name, (0.0, 0))
    fwd_kernel_tflops = (4.0 * D * H * pairs * fwd_attn[1] / (fwd_attn[0] * 1e-3) / 1e12
                         if fwd_attn[1] else None)

    cpu_baseline = None
    if world == 1 and not args.no_cpu_baseline:
        f, t, desc = oracle_sample(w, cpu, args.cpu_seconds)
        cpu_baseline = {"value": f / t / 1e12, "unit": UNIT, "cores": blas_threads(),
                        "kind": "oracle", "sample": desc, "seconds": t}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded N(0,1) q/k/v/dO, norm weights 1+0.1N, FP32 sinks)",
        "config": config_of(w, pairs, flops_step),
        "fwd_tflops": world * ff * args.steps / (fwd_ms * 1e-3) / 1e12,
        "bwd_tflops": world * fb * args.steps / (bwd_ms * 1e-3) / 1e12,
        "fwd_ms": fwd_ms / args.steps, "bwd_ms": bwd_ms / args.steps,
        "fwd_kernel_tflops": fwd_kernel_tflops,
        "fwd_only": fwd_only,
        "pct_of_peak": {
            "step_vs_bf16_sustained": value / world / peaks["bf16_tflops_sustained"],
            "fwd_kernel_vs_bf16_burst": (fwd_kernel_tflops or 0) / peaks["bf16_tflops"],
            "fwd_kernel_vs_nominal_2250": (fwd_kernel_tflops or 0) / 2250.0,
            "fwd_only_kernel_vs_bf16_burst": ((fwd_only or {}).get("kernel_tflops") or 0)
            / peaks["bf16_tflops"],
            "fwd_only_kernel_vs_nominal_2250": ((fwd_only or {}).get("kernel_tflops") or 0)
            / 2250.0,
            "peaks": peak_src},
        "roofline": roofline,
        "roofline_hbm": roofline_hbm,
        "kernels": kernels,
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": e2e,
        "graph": graph,
        "cpu_baseline": cpu_baseline,
    }
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
