"""GPU parity: the CUDA library (through its C ABI) against the FP64 oracle.

Small cases compare every output element; the full-size workloads compare
sampled rows that the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import flint_inputs as fi
from oracle import flint_oracle as fo
from parity_util import check_grads, compare, f64, run_bwd, run_fwd, to_dev

pytestmark = pytest.mark.gpu


def oracle_full(d, w: fi.Workload, backward):
    O, lse = fo.flint_attn_fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                               d["cu_doc_lens"], w.window, w.use_rope, w.rope_theta)
    g = None
    if backward:
        g = fo.flint_attn_bwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                              d["cu_doc_lens"], w.window, w.use_rope, w.rope_theta, d["dout"])
    return O, lse, g


# ----------------------------------------------------------------------- FP32 tiny layer

def test_tiny_sliding_fp32_forward_backward(cuda_lib):
    w = fi.TINY_SLIDING_FP32
    cpu = fi.make_inputs(w)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, w.window, w.use_rope, w.rope_theta)
    O, L, g = oracle_full(cpu, w, True)
    compare(out, O, "fp32", "out")
    compare(lse, L, "fp32", "lse")
    gr = run_bwd(cuda_lib, d, out, lse, w.window, w.use_rope, w.rope_theta)
    torch.cuda.synchronize()
    for name in ["dq", "dk", "dv", "dw_q", "dw_k", "dsink"]:
        compare(gr[name], g[name], "fp32", name)


# ----------------------------------------------------------------------- BF16 small sweeps

SMALL_CASES = [
    # doc lengths, H, Hk, window, rope
    ([300], 32, 4, 64, True),
    ([257, 1, 130, 7], 32, 4, 63, True),
    ([200, 0, 333], 32, 4, 65, False),
    ([513], 32, 4, 1, True),
    ([129, 64], 32, 4, 2, False),
    ([600], 32, 4, 0, False),
    ([450], 32, 4, 10_000, True),
    ([31, 17, 290], 16, 2, 100, True),
    ([160, 96], 8, 1, 0, True),
    ([384], 16, 4, 128, False),      # G = 4
    ([70, 260], 4, 4, 50, True),     # G = 1
]


@pytest.mark.parametrize("lens,H,Hk,W,rope", SMALL_CASES)
def test_bf16_forward_small(cuda_lib, lens, H, Hk, W, rope):
    cpu = fi.make_custom(lens, H, Hk, dtype="bf16", seed=len(lens) * 7 + W % 97)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, W, rope, 1e6)
    O, L = fo.flint_attn_fwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                             cpu["cu_doc_lens"], W, rope, 1e6)
    compare(out, O, "bf16", "out")
    compare(lse, L, "bf16", "lse")


def test_bf16_forward_is_deterministic(cuda_lib):
    cpu = fi.make_custom([700, 300], 32, 4, dtype="bf16", seed=3)
    d = to_dev(cpu)
    o1, l1 = run_fwd(cuda_lib, d, 256, True, 1e6)
    o2, l2 = run_fwd(cuda_lib, d, 256, True, 1e6)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_bf16_sink_minus_inf_and_large_logits(cuda_lib):
    """Sinks at -inf reduce to plain softmax attention; large sinks dominate the row."""
    cpu = fi.make_custom([260, 140], 32, 4, dtype="bf16", seed=5)
    cpu["sink"][:8] = -float("inf")
    cpu["sink"][8:16] = 30.0
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, 90, True, 1e6)
    O, L = fo.flint_attn_fwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                             cpu["cu_doc_lens"], 90, True, 1e6)
    compare(out, O, "bf16", "out")
    compare(lse, L, "bf16", "lse")


# ----------------------------------------------------------------------- full-size workloads

def sample_rows(cu, H, n, seed):
    """Rows at document edges and tile edges, plus random ones."""
    rng = np.random.default_rng(seed)
    cu = [int(c) for c in cu]
    T = cu[-1]
    toks = {0, T - 1, 15, 16, 31, 32, 127, 128, 255}
    for a, b in zip(cu[:-1], cu[1:]):
        if b > a:
            toks |= {a, b - 1}
    toks = [t for t in toks if 0 <= t < T]
    toks += list(rng.integers(0, T, size=max(0, n - len(toks))))
    return [(int(t), int(rng.integers(0, H))) for t in toks[:n]]


@pytest.mark.parametrize("wl", [fi.SLIDING_BF16, fi.FULL_BF16, fi.PACKED_BF16, fi.LONG_FULL_BF16],
                         ids=lambda w: w.name)
def test_bf16_forward_full_size_sampled(cuda_lib, wl):
    cpu = fi.make_inputs(wl, with_grad_out=False)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, wl.window, wl.use_rope, wl.rope_theta)
    torch.cuda.synchronize()
    ro = fo.RowOracle(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                      cpu["cu_doc_lens"], wl.window, wl.use_rope, wl.rope_theta)
    rows = sample_rows(cpu["cu_doc_lens"], wl.num_q_heads, 48 if wl.total_tokens > 40000 else 96,
                       seed=1)
    ref_o = np.stack([ro.forward_row(t, h)[0] for t, h in rows])
    ref_l = np.array([ro.forward_row(t, h)[1] for t, h in rows])
    got_o = torch.stack([out[t, h] for t, h in rows])
    got_l = torch.stack([lse[h, t] for t, h in rows])
    compare(got_o, ref_o, "bf16", "out rows")
    compare(got_l, ref_l, "bf16", "lse rows")
    # properties that hold at every row: finite, |O| bounded by max |v| of the KV head
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    vmax = d["v"].float().abs().amax().item()
    assert out.float().abs().amax().item() <= vmax * 1.01


def test_bf16_sliding_forward_full_oracle(cuda_lib):
    """The 2 x 4096, W=512 layer against the whole-layer oracle (every element)."""
    wl = fi.SLIDING_BF16
    cpu = fi.make_inputs(wl, with_grad_out=False)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, wl.window, wl.use_rope, wl.rope_theta)
    O, L, _ = oracle_full(cpu, wl, False)
    compare(out, O, "bf16", "out")
    compare(lse, L, "bf16", "lse")


# ----------------------------------------------------------------------- BF16 backward

BWD_CASES = [c for i, c in enumerate(SMALL_CASES) if i in (0, 1, 2, 3, 5, 7, 9, 10)]


@pytest.mark.parametrize("lens,H,Hk,W,rope", BWD_CASES)
def test_bf16_backward_small(cuda_lib, lens, H, Hk, W, rope):
    cpu = fi.make_custom(lens, H, Hk, dtype="bf16", seed=len(lens) * 11 + W % 89)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, W, rope, 1e6, fp32_out=True)
    g = run_bwd(cuda_lib, d, out, lse, W, rope, 1e6, fp32_out=True)
    torch.cuda.synchronize()
    ref = fo.flint_attn_bwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                            cpu["cu_doc_lens"], W, rope, 1e6, cpu["dout"])
    check_grads(g, ref, label=f"small {lens} H{H}/{Hk} W{W}", window=W)


def test_bf16_backward_bf16_io(cuda_lib):
    """bf16 O into the backward and bf16 gradients out.

    Elementwise gradients: the stated bar plus one bf16 ulp of the value. The sink
    and norm-weight gradients are sums over every row of D = dO . O_bf16, whose
    bf16 rounding of O dominates their error; they are held to rel-RMS 1e-2.
    """
    lens, H, Hk, W, rope = [300, 77], 32, 4, 96, True
    cpu = fi.make_custom(lens, H, Hk, dtype="bf16", seed=21)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, W, rope, 1e6)
    g = run_bwd(cuda_lib, d, out, lse, W, rope, 1e6, fp32_out=False)
    torch.cuda.synchronize()
    assert out.dtype == torch.bfloat16
    assert g["dq"].dtype == torch.bfloat16 and g["dv"].dtype == torch.bfloat16
    ref = fo.flint_attn_bwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                            cpu["cu_doc_lens"], W, rope, 1e6, cpu["dout"])
    for name in ["dq", "dk", "dv"]:
        compare(g[name], ref[name], "bf16", name, out_bf16=True)
    for name in ["dw_q", "dw_k", "dsink"]:
        err = f64(g[name]) - ref[name]
        assert np.sqrt(np.mean(err ** 2)) <= 1e-2 * np.sqrt(np.mean(ref[name] ** 2)), name


def test_bf16_backward_is_deterministic(cuda_lib):
    cpu = fi.make_custom([500, 260], 32, 4, dtype="bf16", seed=9)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, 200, True, 1e6, fp32_out=True)
    g1 = run_bwd(cuda_lib, d, out, lse, 200, True, 1e6)
    g1 = {k: v.clone() for k, v in g1.items()}
    g2 = run_bwd(cuda_lib, d, out, lse, 200, True, 1e6)
    for k in g1:
        assert torch.equal(g1[k], g2[k]), k


def _prefix(cpu, n_tok, n_docs):
    p = {k: (v[:n_tok] if torch.is_tensor(v) and v.dim() == 3 else v) for k, v in cpu.items()}
    p["cu_doc_lens"] = cpu["cu_doc_lens"][:n_docs + 1].clone()
    p["cu_doc_lens"][-1] = n_tok
    p["doc_lens"] = None
    return p


@pytest.mark.parametrize("wl", [fi.PACKED_BF16, fi.LONG_FULL_BF16], ids=lambda w: w.name)
def test_bf16_backward_full_size_sampled(cuda_lib, wl):
    cpu = fi.make_inputs(wl)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, wl.window, wl.use_rope, wl.rope_theta, fp32_out=True)
    g = run_bwd(cuda_lib, d, out, lse, wl.window, wl.use_rope, wl.rope_theta)
    torch.cuda.synchronize()
    for name in ["dq", "dk", "dv", "dw_q", "dw_k", "dsink"]:
        assert torch.isfinite(g[name]).all(), name
    ro = fo.RowOracle(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                      cpu["cu_doc_lens"], wl.window, wl.use_rope, wl.rope_theta, dO=cpu["dout"])
    rows = sample_rows(cpu["cu_doc_lens"], wl.num_q_heads, 24, seed=2)
    compare(torch.stack([g["dq"][t, h] for t, h in rows]),
            np.stack([ro.dq_row(t, h) for t, h in rows]), "bf16", "dq rows")
    T = wl.total_tokens
    cu = [int(c) for c in cpu["cu_doc_lens"]]
    # key rows whose viewing queries are few enough for the oracle: the ends of documents
    offs = (0, 3, 40) if wl.window > 0 else (0, 5)
    keys = [(b - 1 - o, kv) for b in cu[1:4] for o in offs for kv in (0, 3)]
    keys = [(j, kv) for j, kv in keys if 0 <= j < T]
    ref = [ro.dkv_row(j, kv) for j, kv in keys]
    compare(torch.stack([g["dk"][j, kv] for j, kv in keys]), np.stack([r[0] for r in ref]),
            "bf16", "dk rows")
    compare(torch.stack([g["dv"][j, kv] for j, kv in keys]), np.stack([r[1] for r in ref]),
            "bf16", "dv rows")


@pytest.mark.parametrize("wl,n_tok,n_docs", [(fi.LONG_FULL_BF16, 4096, 1),
                                             (fi.PACKED_BF16, None, 2)],
                         ids=["long_full_prefix4096", "packed_first2docs"])
def test_bf16_backward_prefix_whole_layer(cuda_lib, wl, n_tok, n_docs):
    """d_sink, d norm weights and every gradient element on a prefix of the workload."""
    cpu = fi.make_inputs(wl)
    if n_tok is None:
        n_tok = int(cpu["cu_doc_lens"][n_docs])
    p = _prefix(cpu, n_tok, n_docs)
    d = to_dev(p)
    out, lse = run_fwd(cuda_lib, d, wl.window, wl.use_rope, wl.rope_theta, fp32_out=True)
    g = run_bwd(cuda_lib, d, out, lse, wl.window, wl.use_rope, wl.rope_theta)
    torch.cuda.synchronize()
    O, L = fo.flint_attn_fwd(p["q"], p["k"], p["v"], p["w_q"], p["w_k"], p["sink"],
                             p["cu_doc_lens"], wl.window, wl.use_rope, wl.rope_theta)
    compare(out, O, "bf16", "out")
    compare(lse, L, "bf16", "lse")
    ref = fo.flint_attn_bwd(p["q"], p["k"], p["v"], p["w_q"], p["w_k"], p["sink"],
                            p["cu_doc_lens"], wl.window, wl.use_rope, wl.rope_theta, p["dout"])
    check_grads(g, ref, label=f"{wl.name} prefix {n_tok}", window=wl.window)


# ----------------------------------------------------------------------- FMA-pipe exp2

def test_fma_pipe_exp2_error_bound(cuda_lib):
    """The polynomial exp2 used for part of the softmax stays within 7.5e-5 relative."""
    x = torch.linspace(-125.0, 9.0, 1 << 20, dtype=torch.float64)
    x = torch.cat([x, torch.rand(1 << 16, dtype=torch.float64) - 0.5])
    xf = x.float().cuda()
    y = cuda_lib.exp2_poly(xf).double().cpu()
    ref = torch.exp2(xf.double().cpu())
    rel = ((y - ref).abs() / ref).max().item()
    assert rel <= 7.6e-5, rel
    # exactly 1 at 0, monotone enough that no value is negative or NaN
    assert torch.isfinite(y).all() and (y > 0).all()
    # inputs below -125 (including -inf from the mask) clamp to about 2^-125
    low = cuda_lib.exp2_poly(torch.tensor([-float("inf"), -1e30, -200.0, -126.5],
                                          device="cuda")).cpu()
    assert (low <= 2.0 ** -124).all() and (low > 0).all()
