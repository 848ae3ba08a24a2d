"""Full-size parity beyond sampled rows.

* The packed THD sliding layer (65536 tokens, W = 1024) forward and backward,
  every element of out, LSE, dq, dk, dv and d_sink / the norm-weight gradients
  over all tokens, against the whole-layer FP64 oracle (evaluated per document
  in worker processes; see oracle_pool.py).
* The S = 32768 full-causal forward, every element of out and LSE against the
  oracle (rows split across worker processes), and 4096 rows that cover every
  row position of the kernel's tile pair (32 tokens x 8 heads of a KV group)
  at many points of the sequence, in bfloat16 output.
* The S = 131072 full-causal forward on 1024 tokens x all 32 heads covering
  every tile-row position, and its backward on key rows that 1000-2000 query
  tokens (x 8 heads) see, so long dK/dV accumulations are compared at full size.
* dK and dV of the first keys of the S = 32768 and S = 131072 layers, which every
  query row of their group sees: the longest accumulations of the dK/dV kernel.
All run through the C ABI in the launch configuration bench.py times.
"""
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

import flint_inputs as fi
import oracle_pool
from oracle import flint_oracle as fo
from parity_util import (BF16_MAX_ABS, BF16_REL_RMS, DW_REL, compare, report_sums, run_bwd,
                         run_fwd, to_dev)

pytestmark = pytest.mark.gpu


def _np32(t):
    return t.detach().to("cpu", torch.float32).numpy()


def test_packed_whole_layer_every_element(cuda_lib):
    wl = fi.PACKED_BF16
    cpu = fi.make_inputs(wl)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, wl.window, wl.use_rope, wl.rope_theta, fp32_out=True)
    g = run_bwd(cuda_lib, d, out, lse, wl.window, wl.use_rope, wl.rope_theta)
    torch.cuda.synchronize()
    gpu = {"out": out, "lse": lse, "dq": g["dq"], "dk": g["dk"], "dv": g["dv"]}
    cu = [int(c) for c in cpu["cu_doc_lens"]]
    tasks = []
    for a, b in zip(cu[:-1], cu[1:]):
        if b == a:
            continue
        inp = {n: _np32(cpu[n][a:b]) for n in ("q", "k", "v", "dout")}
        inp.update({n: _np32(cpu[n]) for n in ("w_q", "w_k", "sink")})
        res = {n: _np32(gpu[n][a:b]) for n in ("out", "dq", "dk", "dv")}
        res["lse"] = _np32(lse[:, a:b])
        tasks.append((inp, res, wl.window, wl.use_rope, wl.rope_theta))
    tasks.sort(key=lambda t: -t[0]["q"].shape[0])          # longest documents first
    workers = max(1, min(len(tasks), os.cpu_count() or 1, 16))
    with mp.get_context("spawn").Pool(workers) as pool:
        results = pool.map(oracle_pool.doc_check, tasks, chunksize=1)
    for name in oracle_pool.ELEMENTWISE:
        mx = max(r[0][name][0] for r in results)
        e2 = sum(r[0][name][1] for r in results)
        r2 = sum(r[0][name][2] for r in results)
        bad = sum(r[0][name][3] for r in results)
        rel = float(np.sqrt(e2 / r2))
        print(f"WHOLE packed {name}: max_abs {mx:.3e} rel_rms {rel:.2e}", flush=True)
        assert bad == 0, f"{name}: {bad} non-finite values"
        assert mx <= BF16_MAX_ABS, f"{name}: max_abs {mx:.3e}"
        assert rel <= BF16_REL_RMS, f"{name}: rel_rms {rel:.3e}"
    ref = {n: sum(r[1][n] for r in results) for n in oracle_pool.SUMS}
    report_sums(g, ref, "packed whole layer")
    compare(g["dsink"], ref["dsink"], "bf16", "dsink")
    for name in ("dw_q", "dw_k"):
        compare(g[name], ref[name], "bf16", name, reduction=DW_REL)


def tile_position_rows(T, H, G=8, pair_tokens=32, per_position=16, seed=7):
    """(token, head) rows covering every (token mod 32, head mod 8) position of the
    forward's tile pair, each at per_position places spread over the sequence."""
    rng = np.random.default_rng(seed)
    rows = []
    n_pairs = T // pair_tokens
    for off in range(pair_tokens):
        for hm in range(G):
            bases = rng.choice(n_pairs, size=per_position, replace=False)
            for b in bases:
                rows.append((int(b) * pair_tokens + off, int(rng.integers(0, H // G)) * G + hm))
    return rows


def test_full_forward_every_tile_position(cuda_lib):
    wl = fi.FULL_BF16
    cpu = fi.make_inputs(wl, with_grad_out=False)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, wl.window, wl.use_rope, wl.rope_theta)
    torch.cuda.synchronize()
    rows = tile_position_rows(wl.total_tokens, wl.num_q_heads)
    assert len(rows) == 4096
    ro = fo.RowOracle(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                      cpu["cu_doc_lens"], wl.window, wl.use_rope, wl.rope_theta)
    ref = [ro.forward_row(t, h) for t, h in rows]
    idx_t = torch.tensor([t for t, _ in rows], device=out.device)
    idx_h = torch.tensor([h for _, h in rows], device=out.device)
    compare(out[idx_t, idx_h], np.stack([r[0] for r in ref]), "bf16", "out rows",
            out_bf16=True)
    compare(lse[idx_h, idx_t], np.array([r[1] for r in ref]), "bf16", "lse rows")


def test_full_forward_whole_layer_every_element(cuda_lib):
    wl = fi.FULL_BF16
    cpu = fi.make_inputs(wl, with_grad_out=False)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, wl.window, wl.use_rope, wl.rope_theta, fp32_out=True)
    torch.cuda.synchronize()
    T, step = wl.total_tokens, 512
    chunks = [list(range(t0, t0 + step)) for t0 in range(T - step, -1, -step)]  # longest first
    _check_rows_in_pool(wl, out, lse, chunks, "full forward (every row)")


def _check_rows_in_pool(wl, out, lse, chunks, label):
    """Compare the GPU's out / lse rows of every token in `chunks` (lists of tokens, all
    heads) with the oracle, one chunk per task in spawned workers."""
    tasks = []
    for toks in chunks:
        idx = torch.tensor(toks, device=out.device)
        tasks.append((toks, _np32(out[idx]), _np32(lse[:, idx])))
    workers = max(1, min(len(tasks), os.cpu_count() or 1, 16))
    with mp.get_context("spawn").Pool(workers, initializer=oracle_pool.init_forward_rows,
                                      initargs=(wl.name,)) as pool:
        results = pool.map(oracle_pool.forward_rows_check, tasks, chunksize=1)
    for name in ("out", "lse"):
        mx = max(r[name][0] for r in results)
        rel = float(np.sqrt(sum(r[name][1] for r in results) / sum(r[name][2] for r in results)))
        bad = sum(r[name][3] for r in results)
        print(f"WHOLE {label} {name}: max_abs {mx:.3e} rel_rms {rel:.2e}", flush=True)
        assert bad == 0, f"{name}: {bad} non-finite values"
        assert mx <= BF16_MAX_ABS, f"{name}: max_abs {mx:.3e}"
        assert rel <= BF16_REL_RMS, f"{name}: rel_rms {rel:.3e}"


def test_long_forward_every_tile_position(cuda_lib):
    """The 131072-token forward on 1024 tokens x all 32 heads: every (token mod 32,
    head) position of the kernel's tile pair at 32 places spread over the sequence."""
    wl = fi.LONG_FULL_BF16
    cpu = fi.make_inputs(wl, with_grad_out=False)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, wl.window, wl.use_rope, wl.rope_theta, fp32_out=True)
    torch.cuda.synchronize()
    del d
    rng = np.random.default_rng(11)
    n_pairs = wl.total_tokens // 32
    toks = sorted({int(b) * 32 + off for off in range(32)
                   for b in rng.choice(n_pairs, size=32, replace=False)}, reverse=True)
    assert len(toks) == 1024 and toks[0] < wl.total_tokens
    chunks = [toks[i:i + 64] for i in range(0, len(toks), 64)]
    _check_rows_in_pool(wl, out, lse, chunks, "long forward (tile positions)")


def test_long_backward_keys_with_many_viewers(cuda_lib):
    wl = fi.LONG_FULL_BF16
    cpu = fi.make_inputs(wl)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, wl.window, wl.use_rope, wl.rope_theta, fp32_out=True)
    g = run_bwd(cuda_lib, d, out, lse, wl.window, wl.use_rope, wl.rope_theta)
    torch.cuda.synchronize()
    T = wl.total_tokens
    keys = [T - 1000, T - 1001, T - 1500, T - 2000]       # 1000-2000 viewing tokens x 8 heads
    ro = fo.RowOracle(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                      cpu["cu_doc_lens"], wl.window, wl.use_rope, wl.rope_theta, dO=cpu["dout"])
    for kv in (0, wl.num_kv_heads - 1):
        dk, dv = ro.dkv_rows(keys, kv)
        compare(g["dk"][keys, kv], dk, "bf16", f"dk rows kv{kv}")
        compare(g["dv"][keys, kv], dv, "bf16", f"dv rows kv{kv}")


def _first_keys_check(cuda_lib, wl, keys, workers):
    """dK, dV of keys at the start of a full-causal document, which every query row of
    their group sees (the longest dK/dV accumulations of the layer), against the row
    oracle with the viewing query tokens split across spawned workers."""
    import dataclasses
    wl = dataclasses.replace(wl, backward=True)
    cpu = fi.make_inputs(wl, with_grad_out=True)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, wl.window, wl.use_rope, wl.rope_theta, fp32_out=True)
    g = run_bwd(cuda_lib, d, out, lse, wl.window, wl.use_rope, wl.rope_theta)
    torch.cuda.synchronize()
    gk = g["dk"][keys, 0].clone()
    gv = g["dv"][keys, 0].clone()
    del d, out, lse, g, cpu
    T = wl.total_tokens
    # row i costs ~i (its visible keys): equal-cost token ranges split at T * sqrt(k / n)
    n = 8 * workers
    bounds = sorted({0, T} | {int(T * np.sqrt(k / n)) for k in range(1, n)})
    tasks = [(keys, 0, a, b) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]
    tasks.reverse()                                       # the costly ranges first
    with mp.get_context("spawn").Pool(workers, initializer=oracle_pool.init_dkv_rows,
                                      initargs=(wl.name,)) as pool:
        parts = pool.map(oracle_pool.dkv_rows_part, tasks, chunksize=1)
    dk = sum(p[0] for p in parts)
    dv = sum(p[1] for p in parts)
    compare(gk, dk, "bf16", f"{wl.name} dk of keys {keys}")
    compare(gv, dv, "bf16", f"{wl.name} dv of keys {keys}")
    print(f"FIRST KEYS {wl.name}: dk max-abs {float(np.max(np.abs(gk.double().cpu().numpy() - dk))):.3e}"
          f", dv {float(np.max(np.abs(gv.double().cpu().numpy() - dv))):.3e}")


def _workers(gb_each):
    """Worker processes: at most 16, one per core, and as many as host memory holds."""
    try:
        ram_gb = os.sysconf("SC_PAGE_SIZE") * os.sysconf("SC_PHYS_PAGES") / 2 ** 30
    except (ValueError, OSError):
        ram_gb = 64.0
    return max(1, min(os.cpu_count() or 1, 16, int(ram_gb * 0.6 // gb_each)))


def test_full_backward_first_keys(cuda_lib):
    """The S = 32768 layer's first keys: 32768 x 8 viewing query rows each."""
    _first_keys_check(cuda_lib, fi.FULL_BF16, [0, 1, 2, 127, 128], _workers(2))


def test_long_backward_first_keys(cuda_lib):
    """The S = 131072 layer's first keys: 131072 x 8 viewing query rows each
    (the oracle's ~1.7e13 FLOPs take about 2.5 minutes on 16 cores)."""
    _first_keys_check(cuda_lib, fi.LONG_FULL_BF16, [0, 1, 128], _workers(6))
