"""Pins of the FP64 oracle against facts the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed form,
a special case that reduces to a library routine, an invariant, an independent
brute-force restatement, finite differences, or torch.autograd over an
independent dense restatement.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import brute
from oracle import flint_oracle as fo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(lens, H, Hk, D, seed, qscale=1.0):
    rng = np.random.default_rng(seed)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    q = qscale * rng.standard_normal((T, H, D))
    k = qscale * rng.standard_normal((T, Hk, D))
    v = rng.standard_normal((T, Hk, D))
    wq = 1 + 0.1 * rng.standard_normal(D)
    wk = 1 + 0.1 * rng.standard_normal(D)
    sink = rng.standard_normal(H)
    dO = rng.standard_normal((T, H, D))
    return q, k, v, wq, wk, sink, cu, dO


def dense_mask(cu, window):
    """Independent boolean [T, T] mask: same document, causal, window counts current token."""
    T = int(cu[-1])
    doc = np.zeros(T, dtype=np.int64)
    for d in range(len(cu) - 1):
        doc[cu[d]:cu[d + 1]] = d
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    m = (doc[:, None] == doc[None, :]) & (j <= i)
    if window > 0:
        m &= (i - j) < window
    return m


# --------------------------------------------------------------------------
# Brute force
# --------------------------------------------------------------------------

@pytest.mark.parametrize("lens,H,Hk,D,window,rope", [
    ([7, 1, 12], 4, 2, 8, 3, True),
    ([20], 2, 1, 8, 0, False),
    ([5, 9], 4, 1, 128, 4, True),
    ([16, 16], 4, 4, 8, 1, True),
    ([11, 0, 6], 2, 1, 8, 100, True),
])
def test_vectorised_matches_bruteforce(lens, H, Hk, D, window, rope):
    q, k, v, wq, wk, sink, cu, _ = rand_case(lens, H, Hk, D, seed=sum(lens) + D)
    O, lse = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, window, rope, 1e4)
    Ob, lseb = brute.forward(q, k, v, wq, wk, sink, cu, window, rope, 1e4)
    np.testing.assert_allclose(O, np.array(Ob), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, np.array(lseb), atol=1e-12, rtol=0)


# --------------------------------------------------------------------------
# Special cases and closed forms
# --------------------------------------------------------------------------

def test_sink_minus_inf_is_sdpa_with_mask():
    """s = -inf removes the sink: plain windowed causal softmax attention (library routine)."""
    lens, H, Hk, D, W = [9, 14, 5], 4, 2, 16, 6
    rng = np.random.default_rng(3)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)])
    qh = rng.standard_normal((T, H, D))
    kh = rng.standard_normal((T, Hk, D))
    v = rng.standard_normal((T, Hk, D))
    sink = np.full(H, -np.inf)
    O, lse = fo.attention_forward(qh, kh, v, sink, cu, W)
    G = H // Hk
    qt = torch.from_numpy(qh).permute(1, 0, 2)                      # [H,T,D]
    kt = torch.from_numpy(kh).repeat_interleave(G, dim=1).permute(1, 0, 2)
    vt = torch.from_numpy(v).repeat_interleave(G, dim=1).permute(1, 0, 2)
    mask = torch.from_numpy(dense_mask(cu, W))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask)
    np.testing.assert_allclose(O, ref.permute(1, 0, 2).numpy(), atol=1e-12)
    # LSE without the sink is logsumexp over the visible keys
    z = torch.einsum("htd,hsd->hts", qt, kt) / math.sqrt(D)
    z = z.masked_fill(~mask, -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(z, -1).numpy(), atol=1e-12)


def test_window_at_least_doc_len_is_full_causal():
    q, k, v, wq, wk, sink, cu, _ = rand_case([13, 30, 2], 4, 2, 16, seed=5)
    O0, l0 = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, 0, True, 1e4)
    O1, l1 = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, 30, True, 1e4)
    O2, l2 = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, -5, True, 1e4)
    np.testing.assert_array_equal(O0, O1)
    np.testing.assert_array_equal(O0, O2)
    np.testing.assert_array_equal(l0, l1)


def test_zero_queries_closed_form():
    """q = 0: z = 0 so p_sink = e^s/(e^s+n_i), O_i = mean of visible v * n_i/(e^s+n_i).

    n_i = min(local position + 1, W); this pins the window, the document
    boundaries and the sink at once.
    """
    lens, H, Hk, D, W = [10, 1, 23], 4, 2, 8, 7
    q, k, v, wq, wk, sink, cu, _ = rand_case(lens, H, Hk, D, seed=11)
    q[:] = 0.0
    O, lse = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, W, True, 1e4)
    G = H // Hk
    for d in range(len(lens)):
        for t in range(cu[d], cu[d + 1]):
            p = t - cu[d]
            n = min(p + 1, W)
            for h in range(H):
                es = math.exp(sink[h])
                vm = v[t - n + 1:t + 1, h // G, :].mean(axis=0)
                np.testing.assert_allclose(O[t, h], n / (es + n) * vm, atol=1e-13)
                assert abs(lse[h, t] - math.log(es + n)) < 1e-13


def test_closed_form_golden_fixture():
    """Hand-derived values (tests/golden/closed_form_q0.json) for q = 0."""
    with open(os.path.join(GOLDEN, "closed_form_q0.json")) as f:
        g = json.load(f)
    cu = np.array(g["cu_doc_lens"])
    T = int(cu[-1])
    D = 2
    q = np.zeros((T, 1, D))
    k = np.ones((T, 1, D))
    v = np.array(g["v"], dtype=np.float64).reshape(T, 1, D)
    O, lse = fo.flint_attn_fwd(q, k, v, np.ones(D), np.ones(D), np.array([g["sink"]]),
                               cu, g["window"], False, 1e4)
    np.testing.assert_allclose(O[:, 0, :], np.array(g["expected_O"]), atol=1e-14)
    np.testing.assert_allclose(lse[0], np.log(np.array(g["expected_Z"])), atol=1e-14)


def test_window_one_closed_form():
    """W = 1: only the diagonal key, O_i = v_i e^{z_ii}/(e^{s}+e^{z_ii})."""
    lens, H, Hk, D = [6, 4], 2, 1, 16
    q, k, v, wq, wk, sink, cu, _ = rand_case(lens, H, Hk, D, seed=2)
    O, _ = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, 1, True, 1e4)
    for d in range(len(lens)):
        for t in range(cu[d], cu[d + 1]):
            pos = t - cu[d]
            for h in range(H):
                # norm and rotate both rows by hand (complex-number form of the rotation)
                def nr(x, w):
                    y = x * w / math.sqrt(float(np.mean(x * x)) + 1e-6)
                    zc = (y[:D // 2] + 1j * y[D // 2:]) * np.exp(
                        1j * pos * 1e4 ** (-2 * np.arange(D // 2) / D))
                    return np.concatenate([zc.real, zc.imag])
                z = float(nr(q[t, h], wq) @ nr(k[t, 0], wk)) / math.sqrt(D)
                expect = v[t, 0] * math.exp(z) / (math.exp(sink[h]) + math.exp(z))
                np.testing.assert_allclose(O[t, h], expect, atol=1e-12)


def test_constant_values_convexity():
    """v = c: O_i = (1 - p_sink_i) c with p_sink_i = e^{s_h - LSE_i}."""
    q, k, v, wq, wk, sink, cu, _ = rand_case([17, 8], 4, 1, 8, seed=4)
    v[:] = 2.5
    O, lse = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, 5, True, 1e4)
    psink = np.exp(sink[:, None] - lse)                               # [H, T]
    np.testing.assert_allclose(O, (1 - psink.T)[..., None] * 2.5 * np.ones_like(O), atol=1e-13)
    assert np.all(psink > 0) and np.all(psink < 1)


# --------------------------------------------------------------------------
# Prologue: RMSNorm and RoPE
# --------------------------------------------------------------------------

def test_rmsnorm_closed_forms():
    D, eps = 128, 1e-6
    x = np.full((1, 1, D), 3.0)
    y, _ = fo.rms_norm(x, np.ones(D), eps)
    np.testing.assert_allclose(y, 3.0 / math.sqrt(9.0 + eps), rtol=1e-15)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 3, D))
    y, _ = fo.rms_norm(x, np.ones(D), eps)
    ms = np.mean(x * x, -1)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, -1)), np.sqrt(ms / (ms + eps)), rtol=1e-13)


def test_rope_identity_at_zero_and_norm_preserving():
    rng = np.random.default_rng(1)
    D = 128
    x = rng.standard_normal((4, 3, D))
    ang = fo.rope_angles(np.array([0, 1, 77, 8191]), D, 1e6)
    y = fo.rope_neox(x, ang)
    np.testing.assert_array_equal(y[0], x[0])
    pair_norm = lambda a: a[..., :D // 2] ** 2 + a[..., D // 2:] ** 2
    np.testing.assert_allclose(pair_norm(y), pair_norm(x), rtol=1e-12)
    # transpose is the inverse
    np.testing.assert_allclose(fo.rope_neox_transpose(y, ang), x, atol=1e-13)
    # frequency 0 rotates by exactly the position (theta^0 = 1)
    assert ang[2, 0] == 77.0


def test_pack_invariance():
    """A document gives the same output alone or at any offset in a pack (relative positions)."""
    H, Hk, D = 4, 2, 16
    q, k, v, wq, wk, sink, cu, _ = rand_case([9, 21, 6], H, Hk, D, seed=8)
    O, lse = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, 8, True, 1e4)
    a, b = 9, 30
    Oa, la = fo.flint_attn_fwd(q[a:b], k[a:b], v[a:b], wq, wk, sink, np.array([0, 21]), 8, True, 1e4)
    np.testing.assert_allclose(O[a:b], Oa, atol=1e-13)
    np.testing.assert_allclose(lse[:, a:b], la, atol=1e-13)


def test_pack_invariance_backward():
    """Per-document gradients equal the packed layer's rows, and d_sink / the norm-weight
    gradients of the pack are the sums over its documents (what the per-document
    whole-layer comparisons in the GPU tests rely on)."""
    H, Hk, D = 4, 2, 16
    q, k, v, wq, wk, sink, cu, dO = rand_case([9, 0, 21, 6], H, Hk, D, seed=9)
    g = fo.flint_attn_bwd(q, k, v, wq, wk, sink, cu, 8, True, 1e4, dO)
    sums = {n: np.zeros_like(g[n]) for n in ("dsink", "dw_q", "dw_k")}
    cu = [int(c) for c in cu]
    for a, b in zip(cu[:-1], cu[1:]):
        if b == a:
            continue
        gd = fo.flint_attn_bwd(q[a:b], k[a:b], v[a:b], wq, wk, sink, np.array([0, b - a]), 8,
                               True, 1e4, dO[a:b])
        for n in ("dq", "dk", "dv"):
            np.testing.assert_allclose(gd[n], g[n][a:b], atol=1e-13)
        for n in sums:
            sums[n] += gd[n]
    for n in sums:
        np.testing.assert_allclose(sums[n], g[n], atol=1e-12)


# --------------------------------------------------------------------------
# GQA
# --------------------------------------------------------------------------

def test_gqa_equals_mha_with_repeated_kv():
    H, Hk, D = 8, 2, 16
    q, k, v, wq, wk, sink, cu, dO = rand_case([12, 7], H, Hk, D, seed=9)
    G = H // Hk
    kr, vr = np.repeat(k, G, axis=1), np.repeat(v, G, axis=1)
    O, lse = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, 4, True, 1e4)
    Or, lr = fo.flint_attn_fwd(q, kr, vr, wq, wk, sink, cu, 4, True, 1e4)
    np.testing.assert_allclose(O, Or, atol=1e-13)
    g = fo.flint_attn_bwd(q, k, v, wq, wk, sink, cu, 4, True, 1e4, dO)
    gr = fo.flint_attn_bwd(q, kr, vr, wq, wk, sink, cu, 4, True, 1e4, dO)
    np.testing.assert_allclose(g["dq"], gr["dq"], atol=1e-12)
    np.testing.assert_allclose(g["dk"], gr["dk"].reshape(-1, Hk, G, D).sum(2), atol=1e-12)
    np.testing.assert_allclose(g["dv"], gr["dv"].reshape(-1, Hk, G, D).sum(2), atol=1e-12)
    np.testing.assert_allclose(g["dsink"], gr["dsink"], atol=1e-12)


# --------------------------------------------------------------------------
# Backward
# --------------------------------------------------------------------------

def _loss(args, cu, W, rope, dO):
    q, k, v, wq, wk, sink = args
    O, _ = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, W, rope, 1e4)
    return float(np.sum(O * dO))


@pytest.mark.parametrize("W,rope", [(4, True), (0, False)])
def test_backward_finite_differences(W, rope):
    H, Hk, D = 4, 2, 8
    q, k, v, wq, wk, sink, cu, dO = rand_case([6, 9], H, Hk, D, seed=21)
    g = fo.flint_attn_bwd(q, k, v, wq, wk, sink, cu, W, rope, 1e4, dO)
    grads = [g["dq"], g["dk"], g["dv"], g["dw_q"], g["dw_k"], g["dsink"]]
    args = [q, k, v, wq, wk, sink]
    rng = np.random.default_rng(0)
    h = 1e-6
    for idx in range(6):
        for _ in range(2):
            u = rng.standard_normal(args[idx].shape)
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[idx] = plus[idx] + h * u
            minus[idx] = minus[idx] - h * u
            fd = (_loss(plus, cu, W, rope, dO) - _loss(minus, cu, W, rope, dO)) / (2 * h)
            an = float(np.sum(grads[idx] * u))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (idx, fd, an)


def _torch_dense_layer(q, k, v, wq, wk, sink, cu, W, rope, theta, eps=1e-6):
    """Independent float64 restatement with a dense mask, for torch.autograd."""
    T, H, D = q.shape
    Hk = k.shape[1]
    G = H // Hk
    pos = torch.zeros(T, dtype=torch.float64)
    for d in range(len(cu) - 1):
        pos[cu[d]:cu[d + 1]] = torch.arange(cu[d + 1] - cu[d], dtype=torch.float64)

    def norm_rope(x, w):
        y = x * torch.rsqrt((x * x).mean(-1, keepdim=True) + eps) * w
        if not rope:
            return y
        f = theta ** (-torch.arange(0, D, 2, dtype=torch.float64) / D)
        ang = pos[:, None] * f[None, :]
        cs = torch.polar(torch.ones_like(ang), ang)[:, None, :]
        yc = torch.complex(y[..., :D // 2], y[..., D // 2:]) * cs
        return torch.cat([yc.real, yc.imag], -1)

    qh, kh = norm_rope(q, wq), norm_rope(k, wk)
    kh = kh.repeat_interleave(G, 1)
    vv = v.repeat_interleave(G, 1)
    z = torch.einsum("thd,shd->hts", qh, kh) / math.sqrt(D)
    mask = torch.from_numpy(dense_mask(np.asarray(cu), W))
    z = z.masked_fill(~mask, -math.inf)
    zs = torch.cat([z, sink[:, None, None].expand(H, T, 1)], dim=-1)
    p = torch.softmax(zs, -1)[..., :T]
    return torch.einsum("hts,shd->thd", p, vv)


def test_backward_matches_torch_autograd_restatement():
    H, Hk, D = 4, 2, 16
    q, k, v, wq, wk, sink, cu, dO = rand_case([7, 1, 12], H, Hk, D, seed=31)
    for W, rope in [(5, True), (0, False), (3, False)]:
        g = fo.flint_attn_bwd(q, k, v, wq, wk, sink, cu, W, rope, 1e4, dO)
        ts = [torch.tensor(a, requires_grad=True) for a in (q, k, v, wq, wk, sink)]
        O = _torch_dense_layer(*ts, cu, W, rope, 1e4)
        O.backward(torch.from_numpy(dO))
        for name, t in zip(["dq", "dk", "dv", "dw_q", "dw_k", "dsink"], ts):
            np.testing.assert_allclose(g[name], t.grad.numpy(), atol=1e-11, err_msg=name)
        Of, _ = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, W, rope, 1e4)
        np.testing.assert_allclose(Of, O.detach().numpy(), atol=1e-12)


def test_dsink_closed_form_and_rmsnorm_orthogonality():
    """d s_h = -sum_i p_sink_i (dO_i . O_i); dq (raw) is orthogonal to q per row (up to eps)."""
    H, Hk, D = 4, 1, 32
    q, k, v, wq, wk, sink, cu, dO = rand_case([11, 19], H, Hk, D, seed=12)
    O, lse = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, 6, True, 1e4)
    g = fo.flint_attn_bwd(q, k, v, wq, wk, sink, cu, 6, True, 1e4, dO)
    psink = np.exp(sink[:, None] - lse)
    Dv = np.sum(dO * O, -1).T
    np.testing.assert_allclose(g["dsink"], -np.sum(psink * Dv, -1), atol=1e-12)
    # RMSNorm makes the layer invariant to q -> c q (up to eps), so <dq, q> ~ 0
    dots = np.abs(np.sum(g["dq"] * q, -1))
    scale = np.linalg.norm(g["dq"], axis=-1) * np.linalg.norm(q, axis=-1)
    assert np.max(dots / scale) < 1e-5


def test_row_oracle_matches_whole_layer():
    H, Hk, D = 4, 2, 16
    q, k, v, wq, wk, sink, cu, dO = rand_case([13, 25], H, Hk, D, seed=40)
    for W, rope in [(6, True), (0, False)]:
        O, lse = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, W, rope, 1e4)
        g = fo.flint_attn_bwd(q, k, v, wq, wk, sink, cu, W, rope, 1e4, dO)
        ro = fo.RowOracle(q, k, v, wq, wk, sink, cu, W, rope, 1e4, dO=dO)
        for t, h in [(0, 0), (12, 3), (13, 1), (37, 2), (20, 0)]:
            o, l = ro.forward_row(t, h)
            np.testing.assert_allclose(o, O[t, h], atol=1e-13)
            assert abs(l - lse[h, t]) < 1e-13
            np.testing.assert_allclose(ro.dq_row(t, h), g["dq"][t, h], atol=1e-12)
        for j, kv in [(0, 0), (12, 1), (30, 0), (37, 1)]:
            dk, dv = ro.dkv_row(j, kv)
            np.testing.assert_allclose(dk, g["dk"][j, kv], atol=1e-12)
            np.testing.assert_allclose(dv, g["dv"][j, kv], atol=1e-12)


def test_row_oracle_batched_forward_rows_match_whole_layer():
    """RowOracle.forward_rows (query rows taken as chunks of a logit matrix) equals
    the whole-layer forward, for rows of several documents, small chunks included."""
    H, Hk, D = 4, 2, 16
    q, k, v, wq, wk, sink, cu, _ = rand_case([40, 0, 33, 5], H, Hk, D, seed=42)
    for W, rope in [(9, True), (0, False)]:
        O, L = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, W, rope, 1e4)
        ro = fo.RowOracle(q, k, v, wq, wk, sink, cu, W, rope, 1e4)
        toks = [0, 1, 17, 39, 40, 41, 72, 73, 77]
        for chunk in (3, 64, 1000):
            o, l = ro.forward_rows(toks, chunk=chunk)
            np.testing.assert_allclose(o, O[toks], atol=1e-13)
            np.testing.assert_allclose(l, L[:, toks], atol=1e-13)


def test_row_oracle_batched_key_rows_match_whole_layer():
    """RowOracle.dkv_rows (query rows taken as chunks of a logit matrix) equals the
    whole-layer backward, for keys seen by many rows, small chunks included."""
    H, Hk, D = 4, 2, 16
    q, k, v, wq, wk, sink, cu, dO = rand_case([40, 0, 33], H, Hk, D, seed=41)
    for W, rope in [(9, True), (0, False)]:
        g = fo.flint_attn_bwd(q, k, v, wq, wk, sink, cu, W, rope, 1e4, dO)
        ro = fo.RowOracle(q, k, v, wq, wk, sink, cu, W, rope, 1e4, dO=dO)
        keys = [0, 5, 39, 40, 41, 72]
        for kv in range(Hk):
            for chunk in (3, 64, 1000):
                dk, dv = ro.dkv_rows(keys, kv, chunk=chunk)
                np.testing.assert_allclose(dk, g["dk"][keys, kv], atol=1e-12)
                np.testing.assert_allclose(dv, g["dv"][keys, kv], atol=1e-12)


def test_row_oracle_key_rows_split_by_query_tokens_add_up():
    """dkv_rows restricted to the query tokens of each part of a partition adds up to
    the whole-layer backward (how a long layer's rows are split across processes)."""
    H, Hk, D = 4, 2, 16
    q, k, v, wq, wk, sink, cu, dO = rand_case([60, 21], H, Hk, D, seed=43)
    for W, rope in [(0, True), (13, False)]:
        g = fo.flint_attn_bwd(q, k, v, wq, wk, sink, cu, W, rope, 1e4, dO)
        ro = fo.RowOracle(q, k, v, wq, wk, sink, cu, W, rope, 1e4, dO=dO)
        keys = [0, 1, 30, 59, 60]
        parts = [range(0, 7), range(7, 31), [31, 33, 35], [32, 34] + list(range(36, 81))]
        for kv in range(Hk):
            dk = np.zeros((len(keys), D))
            dv = np.zeros((len(keys), D))
            for part in parts:
                a, b = ro.dkv_rows(keys, kv, chunk=5, tokens=part)
                dk += a
                dv += b
            np.testing.assert_allclose(dk, g["dk"][keys, kv], atol=1e-12)
            np.testing.assert_allclose(dv, g["dv"][keys, kv], atol=1e-12)
            # a part that no viewing query falls in contributes nothing
            a, b = ro.dkv_rows([59], kv, tokens=range(0, 59))
            assert not np.any(a) and not np.any(b)


def test_config_constants_golden():
    """Constants the Flint pages print, as used by the workloads."""
    with open(os.path.join(GOLDEN, "flint_config_constants.json")) as f:
        g = json.load(f)
    from flint_inputs import WORKLOADS, SLIDING_BF16
    c = g["constants"]
    assert SLIDING_BF16.head_dim == c["head_dim"]
    assert SLIDING_BF16.num_q_heads == c["num_attention_heads"]
    assert SLIDING_BF16.num_kv_heads == c["num_key_value_heads"]
    for w in WORKLOADS:
        assert w.rms_eps == c["rms_norm_eps"]
    # the default window of 513 includes the current token: 512 earlier keys + itself
    lens = [600]
    n = [min(p + 1, c["sliding_window"]) for p in range(600)]
    assert n[-1] == 513
    q, k, v, wq, wk, sink, cu, _ = rand_case(lens, 1, 1, 4, seed=0)
    q[:] = 0
    _, lse = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, c["sliding_window"], True, 1e4)
    np.testing.assert_allclose(lse[0], np.log(np.exp(sink[0]) + np.array(n)), atol=1e-12)


# ----------------------------------------------------------------------------
# Decode (one new token per sequence over a KV cache)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("W,rope", [(0, False), (1, True), (5, True), (64, False)])
def test_decode_equals_last_row_of_the_layer(W, rope):
    """Decoding token p over a cache of tokens 0..p-1 is row p of the whole layer."""
    H, Hk, D, C = 4, 2, 16, 40
    lens = [1, 9, 23, 37]                  # tokens per sequence, the last one is new
    rng = np.random.default_rng(11 + W)
    wq = 1 + 0.1 * rng.standard_normal(D)
    wk = 1 + 0.1 * rng.standard_normal(D)
    sink = rng.standard_normal(H)
    B = len(lens)
    q_new = np.zeros((B, H, D)); k_new = np.zeros((B, Hk, D)); v_new = np.zeros((B, Hk, D))
    kc = rng.standard_normal((B, Hk, C, D)); vc = rng.standard_normal((B, Hk, C, D))
    rows, lses = [], []
    for b, L in enumerate(lens):
        q = rng.standard_normal((L, H, D)); k = rng.standard_normal((L, Hk, D))
        v = rng.standard_normal((L, Hk, D))
        cu = np.array([0, L])
        O, lse = fo.flint_attn_fwd(q, k, v, wq, wk, sink, cu, W, rope, 1e4)
        rows.append(O[L - 1]); lses.append(lse[:, L - 1])
        k_hat = fo.prologue(k, wk, np.arange(L), rope, 1e4, 1e-6)
        kc[b, :, :L - 1, :] = k_hat[:L - 1].transpose(1, 0, 2)
        vc[b, :, :L - 1, :] = v[:L - 1].transpose(1, 0, 2)
        q_new[b], k_new[b], v_new[b] = q[L - 1], k[L - 1], v[L - 1]
        want_k = k_hat[L - 1]
    lens_cached = np.array(lens) - 1
    out, lse, kc2, vc2 = fo.decode(q_new, k_new, v_new, wq, wk, sink, lens_cached, kc, vc,
                                   W, rope, 1e4)
    np.testing.assert_allclose(out, np.stack(rows), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, np.stack(lses), rtol=0, atol=1e-12)
    np.testing.assert_allclose(kc2[B - 1, :, lens_cached[-1], :], want_k, rtol=0, atol=1e-12)
    # slots other than the new one are untouched
    for b, p in enumerate(lens_cached):
        mask = np.ones(C, bool); mask[p] = False
        assert np.array_equal(kc2[b][:, mask], kc[b][:, mask])
        assert np.array_equal(vc2[b][:, p], v_new[b])


def test_decode_window_one_closed_form():
    """W = 1: only the new key is visible; O = (1 - p_sink) v_new, LSE = log(e^s + e^z)."""
    H, Hk, D, C = 4, 1, 8, 10
    rng = np.random.default_rng(5)
    B = 3
    q = rng.standard_normal((B, H, D)); k = rng.standard_normal((B, Hk, D))
    v = rng.standard_normal((B, Hk, D))
    wq = np.ones(D); wk = np.ones(D); sink = rng.standard_normal(H)
    kc = rng.standard_normal((B, Hk, C, D)); vc = rng.standard_normal((B, Hk, C, D))
    lens = np.array([0, 4, 9])
    out, lse, _, _ = fo.decode(q, k, v, wq, wk, sink, lens, kc, vc, 1, False, 1e4)
    for b in range(B):
        qh = q[b] / np.sqrt(np.mean(q[b] ** 2, axis=-1, keepdims=True) + 1e-6)
        kh = k[b, 0] / np.sqrt(np.mean(k[b, 0] ** 2) + 1e-6)
        for h in range(H):
            z = qh[h] @ kh / math.sqrt(D)
            ps = math.exp(sink[h]) / (math.exp(sink[h]) + math.exp(z))
            np.testing.assert_allclose(out[b, h], (1 - ps) * v[b, 0], rtol=0, atol=1e-12)
            assert abs(lse[b, h] - math.log(math.exp(sink[h]) + math.exp(z))) < 1e-12


# ----------------------------------------------------------------------------
# Padding (trailing padding in every document; BSHD is cu = [0, S, 2S, ...])
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("lens,valid,H,Hk,D,window,rope", [
    ([10, 10, 10], [10, 4, 0], 4, 2, 8, 0, True),      # BSHD, S = 10
    ([7, 12, 5], [3, 12, 1], 2, 1, 8, 3, True),         # THD with per-document padding
    ([16], [9], 4, 4, 8, 1, False),
])
def test_padded_matches_bruteforce(lens, valid, H, Hk, D, window, rope):
    q, k, v, wq, wk, sink, cu, _ = rand_case(lens, H, Hk, D, seed=sum(valid) + D)
    O, lse = fo.flint_attn_fwd_padded(q, k, v, wq, wk, sink, cu, valid, window, rope, 1e4)
    Ob, lseb = brute.forward(q, k, v, wq, wk, sink, cu, window, rope, 1e4, valid_lens=valid)
    np.testing.assert_allclose(O, np.array(Ob), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, np.array(lseb), atol=1e-12, rtol=0)
    # padded rows: the sink alone
    for d, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        for t in range(a + valid[d], b):
            assert np.all(O[t] == 0.0)
            np.testing.assert_array_equal(lse[:, t], sink)


def test_padded_backward_finite_differences():
    """Gradients of the padded layer, including zeros at every padded token."""
    lens, valid, H, Hk, D = [6, 5], [4, 2], 2, 1, 8
    q, k, v, wq, wk, sink, cu, dO = rand_case(lens, H, Hk, D, seed=2)
    g = fo.flint_attn_bwd_padded(q, k, v, wq, wk, sink, cu, valid, 3, True, 1e4, dO)

    def loss(q_, k_, v_, wq_, wk_, s_):
        O, _ = fo.flint_attn_fwd_padded(q_, k_, v_, wq_, wk_, s_, cu, valid, 3, True, 1e4)
        return float(np.sum(O * dO))

    args = [q, k, v, wq, wk, sink]
    names = ["dq", "dk", "dv", "dw_q", "dw_k", "dsink"]
    h = 1e-6
    for ai, name in enumerate(names):
        x = args[ai]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            xp = x.copy(); xp[i] += h
            xm = x.copy(); xm[i] -= h
            ap = list(args); ap[ai] = xp
            am = list(args); am[ai] = xm
            fd[i] = (loss(*ap) - loss(*am)) / (2 * h)
        np.testing.assert_allclose(g[name], fd, rtol=1e-6, atol=1e-8)
    for t in (4, 5, 6 + 2, 6 + 3, 6 + 4):                # padded tokens
        assert np.all(g["dq"][t] == 0) and np.all(g["dk"][t] == 0) and np.all(g["dv"][t] == 0)
