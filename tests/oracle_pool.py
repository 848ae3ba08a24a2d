"""Whole-layer oracle comparisons split by document, run in worker processes.

Test infrastructure. Documents of a THD pack are independent (positions restart
per document, attention never crosses a boundary; the oracle pins check this
pack invariance for the forward and the backward), so the FP64 oracle of a
packed layer is the oracle of each document on its own, with d_sink and the
norm-weight gradients summed over documents. Each worker evaluates one document
and compares it with the GPU's rows there, returning only error statistics, so
multi-GB layers stay affordable. Start the pool with the ``spawn`` method.
"""
import numpy as np
from threadpoolctl import threadpool_limits

from oracle import flint_oracle as fo

ELEMENTWISE = ("out", "lse", "dq", "dk", "dv")
SUMS = ("dsink", "dw_q", "dw_k")


def doc_check(task):
    """task: (inputs of one document as float32 arrays, GPU results for its rows,
    window, use_rope, rope_theta). Returns ({name: (max_abs, sum_err2, sum_ref2,
    n_nonfinite)}, {sum name: this document's oracle value})."""
    inp, gpu, window, rope, theta = task
    L = inp["q"].shape[0]
    cu = np.array([0, L])
    with threadpool_limits(limits=2):     # the pool already runs one document per core
        O, lse = fo.flint_attn_fwd(inp["q"], inp["k"], inp["v"], inp["w_q"], inp["w_k"],
                                   inp["sink"], cu, window, rope, theta)
        R = fo.flint_attn_bwd(inp["q"], inp["k"], inp["v"], inp["w_q"], inp["w_k"],
                              inp["sink"], cu, window, rope, theta, inp["dout"])
    ref = {"out": O, "lse": lse, "dq": R["dq"], "dk": R["dk"], "dv": R["dv"]}
    stats = {}
    for name in ELEMENTWISE:
        g = np.asarray(gpu[name], dtype=np.float64)
        r = ref[name]
        bad = int(np.sum(~np.isfinite(g)))
        err = g - r
        stats[name] = (float(np.max(np.abs(err))) if err.size else 0.0,
                       float(np.sum(err * err)), float(np.sum(r * r)), bad)
    return stats, {name: R[name] for name in SUMS}


# ---------------------------------------------------------------------------
# Whole-layer forward of a long single-document layer, rows split across workers.
# Rows of the forward are independent, so each worker computes its share of
# query rows with RowOracle.forward_rows. Every worker draws the workload's
# inputs itself from their seed (the same generator the test used), so nothing
# large crosses the process boundary but the GPU rows it checks.
# ---------------------------------------------------------------------------
_ROW_ORACLE = None


def init_forward_rows(workload_name):
    global _ROW_ORACLE
    import flint_inputs as fi
    wl = {w.name: w for w in fi.WORKLOADS}[workload_name]
    cpu = fi.make_inputs(wl, with_grad_out=False)
    with threadpool_limits(limits=2):
        _ROW_ORACLE = fo.RowOracle(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"],
                                   cpu["sink"], cpu["cu_doc_lens"], wl.window, wl.use_rope,
                                   wl.rope_theta)


def forward_rows_check(task):
    """task: (query tokens, GPU out rows [n, H, D], GPU lse [H, n]).
    Returns {"out"/"lse": (max_abs, sum_err2, sum_ref2, n_nonfinite)}."""
    tokens, out, lse = task
    with threadpool_limits(limits=2):
        O, L = _ROW_ORACLE.forward_rows(tokens)
    stats = {}
    for name, g, r in (("out", out, O), ("lse", lse, L)):
        g = np.asarray(g, dtype=np.float64)
        err = g - r
        stats[name] = (float(np.max(np.abs(err))), float(np.sum(err * err)), float(np.sum(r * r)),
                       int(np.sum(~np.isfinite(g))))
    return stats


# ---------------------------------------------------------------------------
# Key rows of a long layer, their viewing query rows split across workers.
# RowOracle.dkv_rows restricted to a part of the query tokens gives that part's
# share of dk and dv (the shares add up: pinned on the CPU), so each worker takes
# a range of query tokens; every worker draws the inputs from their seed.
# ---------------------------------------------------------------------------
_DKV_ORACLE = None


def init_dkv_rows(workload_name):
    global _DKV_ORACLE
    import dataclasses
    import flint_inputs as fi
    wl = {w.name: w for w in fi.WORKLOADS}[workload_name]
    wl = dataclasses.replace(wl, backward=True)
    cpu = fi.make_inputs(wl, with_grad_out=True)
    with threadpool_limits(limits=1):
        _DKV_ORACLE = fo.RowOracle(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"],
                                   cpu["sink"], cpu["cu_doc_lens"], wl.window, wl.use_rope,
                                   wl.rope_theta, dO=cpu["dout"])


def dkv_rows_part(task):
    """task: (keys, kv, first query token, end query token). Returns this token
    range's share of (dk, dv) [n, D] for the keys."""
    keys, kv, t0, t1 = task
    with threadpool_limits(limits=1):
        return _DKV_ORACLE.dkv_rows(keys, kv, tokens=range(t0, t1))
