"""FP64 CPU oracle for Flint's sink-aware attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this module. The CUDA library never
calls it, and it shares no code with the CUDA library.

What it computes, step by step, with the passage each step follows:

* Per-head RMSNorm on q and k: Flint layers page
  (nemo_automodel.components.models.flint.layers), ``FlintAttention`` class
  summary (an RMSNorm applied to each head) and its ``q_norm``/``k_norm``/``eps``
  attributes;
  the epsilon is ``rms_norm_eps`` = 1e-6 on the Flint config page
  (nemo_automodel.components.models.flint.config, ``FlintConfig``).
* NeoX RoPE: Flint layers page, ``FlintAttention._apply_rope`` (each channel in
  the first half of a head rotates with the matching channel of the second
  half), applied to all head channels on sliding layers and not at all on full
  layers (Flint config page, ``FlintConfig`` docstring; ``use_rope`` on the
  layers page). Positions are document-local for THD (``FlintAttention.forward``,
  ``position_ids``).
* Causal window that includes the current token (``FlintConfig`` docstring;
  attention utils page, ``preprocess_args_and_kwargs_for_attn``: a positive
  left window counts visible keys including the current token, negative or
  None is unbounded).
* Block-diagonal document mask over THD packing (``cu_seqlens`` [documents+1]
  on the attention utils page; the causal document mask of ``SequenceLayout.allowed``
  on the mistral_large4 attention page).
* A learned, unscaled FP32 sink logit per query head that enters only the
  softmax denominator, with a zero value: ``_FlintSinkParameters.forward`` and
  ``FlintAttention.forward`` (the sink is one more softmax category whose value
  vector is zero) on the Flint layers page.
* GQA with contiguous groups: head h reads KV head floor(h / (H / Hk)).

Readings where the pages are silent: the softmax scale is 1/sqrt(head_dim);
the norm weight is one [D] vector shared by all heads of q (and one for k),
applied as w * x / sqrt(mean(x^2) + eps); norm comes before RoPE; RoPE
frequencies are theta^(-2j/D) for j < D/2; W <= 0 is unbounded.

The forward is the plain definition of softmax attention over the visible set
plus the sink category. To keep memory bounded it is evaluated for blocks of at
most ``BLOCK`` query rows at a time; nothing else is reordered. The backward is
the analytic gradient of the same definition.
"""
from __future__ import annotations

import numpy as np

BLOCK = 512


# ----------------------------------------------------------------------------
# Document layout
# ----------------------------------------------------------------------------

def doc_bounds(cu_doc_lens):
    """List of (start, end) token ranges, one per document (THD ``cu_seqlens``)."""
    cu = np.asarray(cu_doc_lens, dtype=np.int64)
    return [(int(cu[d]), int(cu[d + 1])) for d in range(len(cu) - 1)]


def doc_positions(cu_doc_lens):
    """Document-local positions: 0, 1, ... restarting at every document start."""
    cu = np.asarray(cu_doc_lens, dtype=np.int64)
    pos = np.zeros(int(cu[-1]), dtype=np.int64)
    for a, b in doc_bounds(cu):
        pos[a:b] = np.arange(b - a)
    return pos


def visible_keys(i, d0, window):
    """Key range [lo, i] visible from query token i of a document starting at d0.

    The window includes the current token: key j is visible iff d0 <= j <= i and
    (window <= 0 or i - j < window).
    """
    lo = d0 if window <= 0 else max(d0, i - window + 1)
    return lo, i


# ----------------------------------------------------------------------------
# Prologue: per-head RMSNorm, then NeoX RoPE
# ----------------------------------------------------------------------------

def rms_norm(x, w, eps):
    """w * x / sqrt(mean_c x_c^2 + eps) over the last (head_dim) axis.

    Returns the normalised tensor and the per-row factor r = (mean x^2 + eps)^-1/2.
    """
    x = np.asarray(x, dtype=np.float64)
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * np.asarray(w, dtype=np.float64), r


def rope_angles(pos, head_dim, theta):
    """Angles [T, D/2]: position times theta^(-2j/D) for frequency index j."""
    j = np.arange(head_dim // 2, dtype=np.float64)
    inv_freq = float(theta) ** (-2.0 * j / head_dim)
    return np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]


def rope_neox(x, ang):
    """Rotate channel j with channel j + D/2 of every head by angle ang[t, j].

    x: [T, heads, D]; ang: [T, D/2].
    """
    h = x.shape[-1] // 2
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_neox_transpose(g, ang):
    """Transpose (= inverse) of ``rope_neox``: rotation by the negated angle."""
    h = g.shape[-1] // 2
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    g1, g2 = g[..., :h], g[..., h:]
    return np.concatenate([g1 * c + g2 * s, g2 * c - g1 * s], axis=-1)


def prologue(x, w, pos, use_rope, theta, eps):
    """x [T, heads, D] -> x_hat: RMSNorm with weight w, then RoPE at positions pos [T]."""
    y, _ = rms_norm(x, w, eps)
    if use_rope:
        y = rope_neox(y, rope_angles(pos, x.shape[-1], theta))
    return y


def prologue_backward(x, w, g_hat, pos, use_rope, theta, eps):
    """Gradients of ``prologue`` w.r.t. x and w, given the gradient g_hat of x_hat.

    With y = x r w, r = (mean x^2 + eps)^-1/2 and u = dy * w:
    dx = r u - x r^3 (1/D) sum_c u_c x_c, and dw = sum over rows of dy * x r.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    D = x.shape[-1]
    dy = g_hat
    if use_rope:
        dy = rope_neox_transpose(g_hat, rope_angles(pos, D, theta))
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    dw = np.sum(dy * x * r, axis=tuple(range(x.ndim - 1)))
    u = dy * w
    dx = r * u - x * (r ** 3) * np.sum(u * x, axis=-1, keepdims=True) / D
    return dx, dw


# ----------------------------------------------------------------------------
# Attention core with a sink category
# ----------------------------------------------------------------------------

def _group(h, H, Hk):
    return h // (H // Hk)


def _block_logits(q_hat, k_hat, a, b, lo, window, h_list, kv, scale):
    """Scaled logits [len(h_list), b-a, b-lo] with -inf outside the visible set."""
    q = q_hat[a:b][:, h_list, :]                       # [n, g, D]
    k = k_hat[lo:b, kv, :]                             # [m, D]
    z = scale * (q.transpose(1, 0, 2) @ k.T)         # [g, n, m]
    i = np.arange(a, b)[:, None]
    j = np.arange(lo, b)[None, :]
    vis = j <= i
    if window > 0:
        vis &= (i - j) < window
    z = np.where(vis[None, :, :], z, -np.inf)
    return z


def _sink_softmax(z, sink_g):
    """Softmax over [z_i., s_h]: returns p [g,n,m], p_sink [g,n], lse [g,n]."""
    s = sink_g[:, None]                                # [g, 1]
    m = np.maximum(np.max(z, axis=-1), s)              # [g, n]
    e = np.exp(z - m[..., None])
    es = np.exp(s - m)
    Z = es + np.sum(e, axis=-1)
    p = e / Z[..., None]
    return p, es / Z, m + np.log(Z)


def attention_forward(q_hat, k_hat, v, sink, cu_doc_lens, window, scale=None):
    """Sink-aware causal (windowed) GQA attention over THD documents.

    q_hat [T,H,D], k_hat/v [T,Hk,D], sink [H] (unscaled logits).
    Returns O [T,H,D] and LSE [H,T] = ln(e^{s_h} + sum_j e^{z_ij}).
    """
    T, H, D = q_hat.shape
    Hk = k_hat.shape[1]
    G = H // Hk
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    sink = np.asarray(sink, dtype=np.float64)
    O = np.zeros((T, H, v.shape[-1]))
    lse = np.zeros((H, T))
    for d0, d1 in doc_bounds(cu_doc_lens):
        for a in range(d0, d1, BLOCK):
            b = min(a + BLOCK, d1)
            lo = d0 if window <= 0 else max(d0, a - window + 1)
            for kv in range(Hk):
                hs = list(range(kv * G, (kv + 1) * G))
                z = _block_logits(q_hat, k_hat, a, b, lo, window, hs, kv, scale)
                p, _, l = _sink_softmax(z, sink[hs])
                O[a:b, kv * G:(kv + 1) * G, :] = (p @ v[lo:b, kv, :]).transpose(1, 0, 2)
                lse[kv * G:(kv + 1) * G, a:b] = l
    return O, lse


def attention_backward(q_hat, k_hat, v, sink, cu_doc_lens, window, dO, scale=None):
    """Analytic gradients of ``attention_forward`` for the loss sum(dO * O).

    D_i = dO_i . O_i; dv_j = sum_i p_ij dO_i; dz_ij = p_ij (dO_i . v_j - D_i);
    dq_hat_i = scale sum_j dz_ij k_hat_j; dk_hat_j = scale sum_i dz_ij q_hat_i;
    d sink_h = -sum_i p_sink_i D_i (the sink's value is zero).
    Returns dq_hat, dk_hat, dv, dsink.
    """
    T, H, D = q_hat.shape
    Hk = k_hat.shape[1]
    G = H // Hk
    scale = 1.0 / np.sqrt(D) if scale is None else scale
    sink = np.asarray(sink, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    O, _ = attention_forward(q_hat, k_hat, v, sink, cu_doc_lens, window, scale)
    Dvec = np.sum(dO * O, axis=-1)                     # [T, H]
    dq = np.zeros_like(q_hat)
    dk = np.zeros_like(k_hat)
    dv = np.zeros_like(v, dtype=np.float64)
    dsink = np.zeros(H)
    for d0, d1 in doc_bounds(cu_doc_lens):
        for a in range(d0, d1, BLOCK):
            b = min(a + BLOCK, d1)
            lo = d0 if window <= 0 else max(d0, a - window + 1)
            for kv in range(Hk):
                hs = list(range(kv * G, (kv + 1) * G))
                z = _block_logits(q_hat, k_hat, a, b, lo, window, hs, kv, scale)
                p, ps, _ = _sink_softmax(z, sink[hs])            # [g,n,m], [g,n]
                dOb = dO[a:b, kv * G:(kv + 1) * G, :]             # [n,g,D]
                Di = Dvec[a:b, kv * G:(kv + 1) * G].T             # [g,n]
                dOg = dOb.transpose(1, 0, 2)                      # [g,n,D]
                dv[lo:b, kv, :] += (p.transpose(0, 2, 1) @ dOg).sum(axis=0)
                dp = dOg @ v[lo:b, kv, :].T                       # [g,n,m]
                dz = p * (dp - Di[..., None])
                dq[a:b, kv * G:(kv + 1) * G, :] += scale * (dz @ k_hat[lo:b, kv, :]).transpose(1, 0, 2)
                dk[lo:b, kv, :] += scale * (dz.transpose(0, 2, 1) @
                                            q_hat[a:b][:, hs, :].transpose(1, 0, 2)).sum(axis=0)
                dsink[hs] -= np.sum(ps * Di, axis=-1)
    return dq, dk, dv, dsink


# ----------------------------------------------------------------------------
# Whole layer: prologue + attention (+ backward)
# ----------------------------------------------------------------------------

def _f64(x):
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def flint_attn_fwd(q, k, v, w_q, w_k, sink, cu_doc_lens, window, use_rope,
                   rope_theta, eps=1e-6, scale=None):
    """Prologue on q and k, then sink-aware attention. Returns O [T,H,D], LSE [H,T]."""
    q, k, v, w_q, w_k, sink = map(_f64, (q, k, v, w_q, w_k, sink))
    cu = np.asarray(_f64(cu_doc_lens), dtype=np.int64)
    pos = doc_positions(cu)
    q_hat = prologue(q, w_q, pos, use_rope, rope_theta, eps)
    k_hat = prologue(k, w_k, pos, use_rope, rope_theta, eps)
    return attention_forward(q_hat, k_hat, v, sink, cu, window, scale)


def flint_attn_bwd(q, k, v, w_q, w_k, sink, cu_doc_lens, window, use_rope,
                   rope_theta, dO, eps=1e-6, scale=None):
    """Gradients of sum(dO * O) w.r.t. the raw q, k, v, both norm weights and the sinks.

    Returns a dict with dq, dk, dv, dw_q, dw_k, dsink.
    """
    q, k, v, w_q, w_k, sink, dO = map(_f64, (q, k, v, w_q, w_k, sink, dO))
    cu = np.asarray(_f64(cu_doc_lens), dtype=np.int64)
    pos = doc_positions(cu)
    q_hat = prologue(q, w_q, pos, use_rope, rope_theta, eps)
    k_hat = prologue(k, w_k, pos, use_rope, rope_theta, eps)
    dqh, dkh, dv, dsink = attention_backward(q_hat, k_hat, v, sink, cu, window, dO, scale)
    dq, dwq = prologue_backward(q, w_q, dqh, pos, use_rope, rope_theta, eps)
    dk, dwk = prologue_backward(k, w_k, dkh, pos, use_rope, rope_theta, eps)
    return {"dq": dq, "dk": dk, "dv": dv, "dw_q": dwq, "dw_k": dwk, "dsink": dsink}


# ----------------------------------------------------------------------------
# Padding (attention utils page: a BSHD attention_mask; TE takes trailing
# padding only): document d holds valid_lens[d] real tokens followed by padding
# ----------------------------------------------------------------------------

def _valid_tokens(cu, valid_lens):
    """Indices of the real tokens and the cu_doc_lens of the documents they form."""
    idx, cu_v = [], [0]
    for d, (a, b) in enumerate(doc_bounds(cu)):
        n = max(0, min(int(valid_lens[d]), b - a))
        idx.extend(range(a, a + n))
        cu_v.append(cu_v[-1] + n)
    return np.asarray(idx, dtype=np.int64), np.asarray(cu_v, dtype=np.int64)


def flint_attn_fwd_padded(q, k, v, w_q, w_k, sink, cu_doc_lens, valid_lens, window, use_rope,
                          rope_theta, eps=1e-6, scale=None):
    """Forward with trailing padding in every document.

    Padded tokens are excluded as keys; a padded query sees no key, so its row
    is the sink alone: O = 0 and LSE = sink_h (the sink stays valid). Padding is
    trailing, so a real token keeps its position and its visible keys, and the
    real rows are exactly the layer over the documents' real prefixes.
    """
    q, k, v, sink = map(_f64, (q, k, v, sink))
    cu = np.asarray(_f64(cu_doc_lens), dtype=np.int64)
    idx, cu_v = _valid_tokens(cu, _f64(valid_lens))
    T, H, D = q.shape
    O = np.zeros((T, H, D))
    lse = np.repeat(sink[:, None], T, axis=1)
    if len(idx):
        O_v, lse_v = flint_attn_fwd(q[idx], k[idx], v[idx], w_q, w_k, sink, cu_v, window,
                                    use_rope, rope_theta, eps, scale)
        O[idx] = O_v
        lse[:, idx] = lse_v
    return O, lse


def flint_attn_bwd_padded(q, k, v, w_q, w_k, sink, cu_doc_lens, valid_lens, window, use_rope,
                          rope_theta, dO, eps=1e-6, scale=None):
    """Gradients of sum(dO * O) for ``flint_attn_fwd_padded``.

    Padded rows of O are constant, so every gradient at a padded token is zero
    and padded rows add nothing to d_sink (their D = dO . O is 0) or to the
    norm-weight gradients.
    """
    q, k, v, dO = map(_f64, (q, k, v, dO))
    cu = np.asarray(_f64(cu_doc_lens), dtype=np.int64)
    idx, cu_v = _valid_tokens(cu, _f64(valid_lens))
    D = q.shape[-1]
    out = {"dq": np.zeros(q.shape), "dk": np.zeros(k.shape), "dv": np.zeros(v.shape),
           "dw_q": np.zeros(D), "dw_k": np.zeros(D), "dsink": np.zeros(len(_f64(sink)))}
    if len(idx):
        g = flint_attn_bwd(q[idx], k[idx], v[idx], w_q, w_k, sink, cu_v, window, use_rope,
                           rope_theta, dO[idx], eps, scale)
        for name in ("dq", "dk", "dv"):
            out[name][idx] = g[name]
        for name in ("dw_q", "dw_k", "dsink"):
            out[name] = g[name]
    return out


# ----------------------------------------------------------------------------
# Sampled rows, for sizes where the whole layer is too slow on a CPU
# ----------------------------------------------------------------------------

def _doc_of(cu, t):
    """(start, end) of the document holding token t."""
    d = int(np.searchsorted(cu, t, side="right") - 1)
    while cu[d + 1] <= t:          # skip empty documents that share a start
        d += 1
    return int(cu[d]), int(cu[d + 1])


class RowOracle:
    """Selected outputs of one layer, each computed on its own from the definition.

    Used where the whole layer is too large for a CPU: a query row (t, h) needs
    only its own visible keys; a key row (j, kv) needs the query rows that see it.
    The normalised keys of the whole input are computed once (T * Hk * D work).
    """

    def __init__(self, q, k, v, w_q, w_k, sink, cu_doc_lens, window, use_rope,
                 rope_theta, dO=None, eps=1e-6, scale=None):
        # q and dO rows are converted to float64 when a row needs them (the
        # whole tensors can be several GB in float64); k, v are converted once.
        self._q_src, self._dO_src = q, dO
        self.k, self.v, self.w_q, self.w_k, self.sink = map(_f64, (k, v, w_q, w_k, sink))
        self.cu = np.asarray(_f64(cu_doc_lens), dtype=np.int64)
        self.pos = doc_positions(self.cu)
        self.window, self.use_rope, self.theta, self.eps = window, use_rope, rope_theta, eps
        T, H, D = q.shape
        self.H, self.Hk, self.D = H, self.k.shape[1], D
        self.scale = 1.0 / np.sqrt(D) if scale is None else scale
        self.k_hat = prologue(self.k, self.w_k, self.pos, use_rope, rope_theta, eps)
        # contiguous copy per KV head: row products then read memory in order
        self.k_hat_kv = [np.ascontiguousarray(self.k_hat[:, g, :]) for g in range(self.Hk)]
        self.v_kv = [np.ascontiguousarray(self.v[:, g, :]) for g in range(self.Hk)]

    def _q_row(self, t, h):
        return _f64(self._q_src[t:t + 1, h:h + 1, :])

    def _dO_row(self, t, h):
        return _f64(self._dO_src[t, h, :])

    def _q_hat(self, t, h):
        return prologue(self._q_row(t, h), self.w_q, self.pos[t:t + 1],
                        self.use_rope, self.theta, self.eps)[0, 0]

    def _row(self, t, h):
        """Visible key range, probabilities over it, p_sink, LSE and O for row (t, h)."""
        d0, _ = _doc_of(self.cu, t)
        lo, hi = visible_keys(t, d0, self.window)
        kv = _group(h, self.H, self.Hk)
        z = self.scale * (self.k_hat_kv[kv][lo:hi + 1] @ self._q_hat(t, h))
        m = max(float(np.max(z)), float(self.sink[h]))
        e = np.exp(z - m)
        Z = np.exp(self.sink[h] - m) + np.sum(e)
        p = e / Z
        return lo, hi, kv, p, np.exp(self.sink[h] - m) / Z, m + np.log(Z), p @ self.v_kv[kv][lo:hi + 1]

    def forward_row(self, t, h):
        """(O[t, h, :], LSE[h, t])."""
        _, _, _, _, _, lse, o = self._row(t, h)
        return o, lse

    def dq_row(self, t, h):
        """Gradient of sum(dO * O) w.r.t. the raw q[t, h, :]."""
        lo, hi, kv, p, _, _, o = self._row(t, h)
        dO = self._dO_row(t, h)
        Di = float(dO @ o)
        dz = p * (self.v_kv[kv][lo:hi + 1] @ dO - Di)
        g_hat = self.scale * (dz @ self.k_hat_kv[kv][lo:hi + 1])
        dx, _ = prologue_backward(self._q_row(t, h), self.w_q, g_hat[None, None, :],
                                  self.pos[t:t + 1], self.use_rope, self.theta, self.eps)
        return dx[0, 0]

    def dkv_row(self, j, kv):
        """Gradients w.r.t. the raw k[j, kv, :] and v[j, kv, :]."""
        d0, d1 = _doc_of(self.cu, j)
        hi = d1 if self.window <= 0 else min(d1, j + self.window)
        G = self.H // self.Hk
        dk_hat = np.zeros(self.D)
        dv = np.zeros(self.v.shape[-1])
        for i in range(j, hi):
            for h in range(kv * G, (kv + 1) * G):
                lo, _, _, p, _, _, o = self._row(i, h)
                pij = p[j - lo]
                dO = self._dO_row(i, h)
                Di = float(dO @ o)
                dv += pij * dO
                dz = pij * (float(dO @ self.v[j, kv]) - Di)
                dk_hat += self.scale * dz * self._q_hat(i, h)
        dx, _ = prologue_backward(self.k[j:j + 1, kv:kv + 1, :], self.w_k, dk_hat[None, None, :],
                                  self.pos[j:j + 1], self.use_rope, self.theta, self.eps)
        return dx[0, 0], dv


    def forward_rows(self, tokens, chunk=256):
        """``forward_row`` for every head of several query tokens at once.

        The same definition: each row (t, h) takes its own visible keys, the
        unscaled sink logit joins its softmax denominator with a zero value, and
        O and LSE follow. Rows are taken ``chunk`` at a time as one matrix of
        logits per KV head. Returns O [n, H, D] and LSE [H, n].
        """
        tokens = [int(t) for t in tokens]
        G = self.H // self.Hk
        O = np.zeros((len(tokens), self.H, self.v.shape[-1]))
        L = np.zeros((self.H, len(tokens)))
        for kv in range(self.Hk):
            K, V = self.k_hat_kv[kv], self.v_kv[kv]
            pairs = [(n, t, h) for n, t in enumerate(tokens) for h in range(kv * G, (kv + 1) * G)]
            for c0 in range(0, len(pairs), chunk):
                part = pairs[c0:c0 + chunk]
                bounds = [visible_keys(t, _doc_of(self.cu, t)[0], self.window) for _, t, _ in part]
                lo = min(b[0] for b in bounds)
                hi = max(b[1] for b in bounds) + 1
                qh = np.stack([self._q_hat(t, h) for _, t, h in part])
                s_h = np.array([self.sink[h] for _, _, h in part])
                z = self.scale * (qh @ K[lo:hi].T)
                col = np.arange(lo, hi)[None, :]
                vis = (col >= np.array([b[0] for b in bounds])[:, None]) & \
                      (col <= np.array([b[1] for b in bounds])[:, None])
                z = np.where(vis, z, -np.inf)
                m = np.maximum(np.max(z, axis=1), s_h)
                e = np.exp(z - m[:, None])
                Z = np.exp(s_h - m) + np.sum(e, axis=1)
                o = (e @ V[lo:hi]) / Z[:, None]
                for r, (n, _, h) in enumerate(part):
                    O[n, h] = o[r]
                    L[h, n] = m[r] + np.log(Z[r])
        return O, L

    def dkv_rows(self, keys, kv, chunk=256, tokens=None):
        """``dkv_row`` for several keys of KV head ``kv`` at once.

        The same definition: every query row (i, h) that sees a key contributes
        p_ij dO_i to dv_j and scale * p_ij (dO_i . v_j - D_i) q_hat_i to dk_hat_j,
        with p, D_i = dO_i . O_i and O_i from that row's full visible set. The
        query rows are taken ``chunk`` at a time as one matrix of logits, so keys
        with thousands of viewing rows stay affordable. Returns (dk, dv) [n, D].

        ``tokens`` (optional): only query rows whose token is in this collection
        contribute. dv_j and dk_hat_j are sums over rows and the transpose of the
        prologue is linear in dk_hat_j, so the results for a partition of the
        viewing tokens add up to the whole (a long layer's rows can be split
        across processes).
        """
        keys = [int(j) for j in keys]
        G = self.H // self.Hk
        heads = list(range(kv * G, (kv + 1) * G))
        # query tokens that see any of the keys
        rows = set()
        for j in keys:
            d0, d1 = _doc_of(self.cu, j)
            hi = d1 if self.window <= 0 else min(d1, j + self.window)
            rows.update(range(j, hi))
        if tokens is not None:
            rows &= {int(t) for t in tokens}
        rows = sorted(rows)
        pairs = [(i, h) for i in rows for h in heads]
        K, V = self.k_hat_kv[kv], self.v_kv[kv]
        kidx = np.asarray(keys)
        dk_hat = np.zeros((len(keys), self.D))
        dv = np.zeros((len(keys), self.v.shape[-1]))
        for c0 in range(0, len(pairs), chunk):
            part = pairs[c0:c0 + chunk]
            bounds = [visible_keys(i, _doc_of(self.cu, i)[0], self.window) for i, _ in part]
            lo = min(b[0] for b in bounds)
            hi = max(b[1] for b in bounds) + 1
            qh = np.stack([self._q_hat(i, h) for i, h in part])           # [r, D]
            dO = np.stack([self._dO_row(i, h) for i, h in part])          # [r, D]
            s_h = np.array([self.sink[h] for _, h in part])
            z = self.scale * (qh @ K[lo:hi].T)                            # [r, m]
            col = np.arange(lo, hi)[None, :]
            vis = (col >= np.array([b[0] for b in bounds])[:, None]) & \
                  (col <= np.array([b[1] for b in bounds])[:, None])
            z = np.where(vis, z, -np.inf)
            m = np.maximum(np.max(z, axis=1), s_h)
            e = np.exp(z - m[:, None])
            Z = np.exp(s_h - m) + np.sum(e, axis=1)
            p = e / Z[:, None]                                            # [r, m]
            O = p @ V[lo:hi]                                              # [r, D]
            Di = np.sum(dO * O, axis=1)                                   # [r]
            inside = (kidx >= lo) & (kidx < hi)
            for n in np.nonzero(inside)[0]:
                j = kidx[n]
                pj = p[:, j - lo]                                         # [r]
                dv[n] += pj @ dO
                dz = pj * (dO @ self.v[j, kv] - Di)
                dk_hat[n] += self.scale * (dz @ qh)
        dk = np.zeros_like(dk_hat)
        for n, j in enumerate(keys):
            dx, _ = prologue_backward(self.k[j:j + 1, kv:kv + 1, :], self.w_k,
                                      dk_hat[n][None, None, :], self.pos[j:j + 1],
                                      self.use_rope, self.theta, self.eps)
            dk[n] = dx[0, 0]
        return dk, dv


# ----------------------------------------------------------------------------
# Decode: one new token per sequence attending over its KV cache
# ----------------------------------------------------------------------------

def decode(q, k_new, v_new, w_q, w_k, sink, cache_lens, k_cache, v_cache, window,
           use_rope, rope_theta, eps=1e-6, scale=None, store=None):
    """The layer's forward for the next token of B cached sequences.

    Same definition as ``flint_attn_fwd``, restricted to one query row: sequence
    b has ``cache_lens[b]`` = p tokens cached (positions 0..p-1), so the new token
    sits at position p (RoPE angle and causal index). Its normalised, rotated key
    and its value are written into slot p of the caches first, and attention
    reads the caches: the query sees slots j with max(0, p - W + 1) <= j <= p
    (W <= 0: all of 0..p), plus the sink category.

    q [B, H, D], k_new / v_new [B, Hk, D] are the raw projections of the new
    token; the caches are [B, Hk, C, D] (head-major per sequence) and hold
    normalised, rotated keys. ``store`` maps a row to the value the cache holds
    after the write (rounding to the cache dtype); None keeps it exact.
    Returns out [B, H, D], lse [B, H] and the updated caches.
    """
    q, k_new, v_new, w_q, w_k, sink = map(_f64, (q, k_new, v_new, w_q, w_k, sink))
    kc = _f64(k_cache).copy()
    vc = _f64(v_cache).copy()
    lens = np.asarray(_f64(cache_lens), dtype=np.int64)
    B, H, D = q.shape
    Hk = k_new.shape[1]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    keep = (lambda x: x) if store is None else store
    out = np.zeros((B, H, D))
    lse = np.zeros((B, H))
    for b in range(B):
        p = int(lens[b])
        pos = np.array([p])
        q_hat = prologue(q[b][None], w_q, pos, use_rope, rope_theta, eps)[0]      # [H, D]
        k_hat = prologue(k_new[b][None], w_k, pos, use_rope, rope_theta, eps)[0]  # [Hk, D]
        kc[b, :, p, :] = keep(k_hat)
        vc[b, :, p, :] = keep(v_new[b])
        lo, _ = visible_keys(p, 0, window)
        for h in range(H):
            g = _group(h, H, Hk)
            z = scale * (kc[b, g, lo:p + 1, :] @ q_hat[h])                       # [n]
            pr, _, l = _sink_softmax(z[None, None, :], sink[h:h + 1])
            out[b, h] = pr[0, 0] @ vc[b, g, lo:p + 1, :]
            lse[b, h] = l[0, 0]
    return out, lse, kc, vc
