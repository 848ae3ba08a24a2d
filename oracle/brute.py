"""Pure-Python brute-force restatement of Flint's sink-aware attention forward.

TEST INFRASTRUCTURE ONLY (same import rule as ``flint_oracle``). It shares no
helper with ``flint_oracle``: every step is written out again with scalar loops
and the ``math`` module, for tiny inputs (T <= 64, H <= 4), so that the two can
be compared to ~1e-12.

Per query token i of document [d0, d1), head h (KV head h // (H/Hk)):
  x_hat = w * x / sqrt(mean(x^2) + eps)      (per-head RMSNorm, Flint layers page,
                                              FlintAttention; eps from FlintConfig)
  NeoX rotation of channels (j, j + D/2) by (i - d0) * theta^(-2j/D)
                                             (FlintAttention._apply_rope)
  visible keys: d0 <= j <= i and (W <= 0 or i - j < W)
                                             (FlintConfig docstring; attention utils
                                              page, preprocess_args_and_kwargs_for_attn)
  softmax over {z_ij} and the sink logit s_h (not scaled); the sink's value is zero
                                             (FlintAttention.forward,
                                              _FlintSinkParameters.forward)
"""
from __future__ import annotations

import math


def _norm_rope_row(x, w, pos, use_rope, theta, eps):
    D = len(x)
    ms = 0.0
    for c in range(D):
        ms += x[c] * x[c]
    ms /= D
    r = 1.0 / math.sqrt(ms + eps)
    y = [x[c] * r * w[c] for c in range(D)]
    if not use_rope:
        return y
    half = D // 2
    out = [0.0] * D
    for j in range(half):
        ang = pos * (theta ** (-2.0 * j / D))
        c, s = math.cos(ang), math.sin(ang)
        out[j] = y[j] * c - y[j + half] * s
        out[j + half] = y[j + half] * c + y[j] * s
    return out


def forward(q, k, v, w_q, w_k, sink, cu_doc_lens, window, use_rope, theta,
            eps=1e-6, scale=None, valid_lens=None):
    """q [T][H][D], k/v [T][Hk][D] nested lists (or arrays); returns O [T][H][D], LSE [H][T].

    valid_lens[d] (optional): document d's first valid_lens[d] tokens are real,
    the rest are padding - excluded as keys, and as queries they see no key, so
    only the sink remains (O = 0, LSE = the sink logit).
    """
    T = len(q)
    H = len(q[0])
    Hk = len(k[0])
    D = len(q[0][0])
    G = H // Hk
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    cu = [int(c) for c in cu_doc_lens]
    doc_start = [0] * T
    doc_valid = [0] * T                 # first padded token of the token's document
    for d in range(len(cu) - 1):
        n = cu[d + 1] - cu[d] if valid_lens is None else min(int(valid_lens[d]), cu[d + 1] - cu[d])
        for t in range(cu[d], cu[d + 1]):
            doc_start[t] = cu[d]
            doc_valid[t] = cu[d] + n
    kh = [[_norm_rope_row([float(a) for a in k[t][g]], [float(a) for a in w_k],
                          t - doc_start[t], use_rope, theta, eps) for g in range(Hk)]
          for t in range(T)]
    O = [[[0.0] * D for _ in range(H)] for _ in range(T)]
    lse = [[0.0] * T for _ in range(H)]
    for i in range(T):
        d0 = doc_start[i]
        for h in range(H):
            g = h // G
            qh = _norm_rope_row([float(a) for a in q[i][h]], [float(a) for a in w_q],
                                i - d0, use_rope, theta, eps)
            keys = [j for j in range(d0, i + 1)
                    if (window <= 0 or i - j < window) and j < doc_valid[i]]
            if i >= doc_valid[i]:
                keys = []                   # a padded query sees no key
            logits = []
            for j in range(len(keys)):
                dot = 0.0
                for c in range(D):
                    dot += qh[c] * kh[keys[j]][g][c]
                logits.append(scale * dot)
            s = float(sink[h])
            m = max(logits + [s])
            Z = math.exp(s - m) if s != -math.inf else 0.0
            for z in logits:
                Z += math.exp(z - m)
            for jj, j in enumerate(keys):
                p = math.exp(logits[jj] - m) / Z
                for c in range(D):
                    O[i][h][c] += p * float(v[j][g][c])
            lse[h][i] = m + math.log(Z)
    return O, lse
