"""Why the tensor-core operands are fp16 and why O is compared in float32.

The backward of BF16 inputs rounds at a few points only: the normalised,
rotated q_hat / k_hat (MMA operands), P and dS (fp16 operands of the dV, dQ, dK
products), and O as stored by the forward (D = dO . O is formed from it). This
test emulates those rounding points in float64 arithmetic on the oracle's own
steps, on the degenerate window W = 1 (every row attends to itself and the
sink, the largest per-row gradients of the sweeps), and checks the three facts
the precision plan rests on against the max-abs bar of 2e-2:

* fp16 operands with O in float32 stay well inside the bar;
* bf16 operands with O in float32 do not;
* O stored in bf16 alone moves dk past the bar, whatever the operands.
"""
import numpy as np
import pytest
import torch

import flint_inputs as fi
from oracle import flint_oracle as fo

BAR = 2e-2


def _round(dtype):
    if dtype is None:
        return lambda x: x
    return lambda x: torch.from_numpy(np.asarray(x, np.float32)).to(dtype).double().numpy()


@pytest.fixture(scope="module")
def case():
    lens, H, Hk, W, rope, theta = [513], 32, 4, 1, True, 1e6
    cpu = fi.make_custom(lens, H, Hk, dtype="bf16", seed=len(lens) * 11 + W % 89)
    x = {n: cpu[n].double().numpy() for n in ("q", "k", "v", "w_q", "w_k", "sink", "dout")}
    cu = cpu["cu_doc_lens"].numpy()
    ref = fo.flint_attn_bwd(x["q"], x["k"], x["v"], x["w_q"], x["w_k"], x["sink"], cu, W, rope,
                            theta, x["dout"])
    return dict(x=x, cu=cu, H=H, Hk=Hk, W=W, rope=rope, theta=theta, ref=ref)


def emulate(c, operands, o_store):
    """Gradients with q_hat, k_hat, P, dS rounded to `operands` and O to `o_store`."""
    x, cu, H, Hk, W = c["x"], c["cu"], c["H"], c["Hk"], c["W"]
    r_op, r_o = _round(operands), _round(o_store)
    pos = fo.doc_positions(cu)
    qh = r_op(fo.prologue(x["q"], x["w_q"], pos, c["rope"], c["theta"], 1e-6))
    kh = r_op(fo.prologue(x["k"], x["w_k"], pos, c["rope"], c["theta"], 1e-6))
    O, lse = fo.attention_forward(qh, kh, x["v"], x["sink"], cu, W)
    Dv = np.sum(x["dout"] * r_o(O), axis=-1)                        # [T, H]
    G, scale = H // Hk, 1.0 / np.sqrt(qh.shape[-1])
    dq, dk, dv = np.zeros_like(qh), np.zeros_like(kh), np.zeros_like(x["v"])
    for d0, d1 in fo.doc_bounds(cu):
        i = np.arange(d0, d1)[:, None]
        j = np.arange(d0, d1)[None, :]
        vis = (j <= i) & ((i - j) < W if W > 0 else True)
        for h in range(H):
            g = h // G
            z = scale * qh[d0:d1, h] @ kh[d0:d1, g].T
            P = r_op(np.where(vis, np.exp(z - lse[h, d0:d1, None]), 0.0))
            dp = x["dout"][d0:d1, h] @ x["v"][d0:d1, g].T
            dS = r_op(P * (dp - Dv[d0:d1, h, None]))
            dv[d0:d1, g] += P.T @ x["dout"][d0:d1, h]
            dq[d0:d1, h] += scale * dS @ kh[d0:d1, g]
            dk[d0:d1, g] += scale * dS.T @ qh[d0:d1, h]
    gq, _ = fo.prologue_backward(x["q"], x["w_q"], dq, pos, c["rope"], c["theta"], 1e-6)
    gk, _ = fo.prologue_backward(x["k"], x["w_k"], dk, pos, c["rope"], c["theta"], 1e-6)
    return {"dq": gq, "dk": gk, "dv": dv}


def max_err(c, e):
    return {n: float(np.abs(e[n] - c["ref"][n]).max()) for n in ("dq", "dk", "dv")}


def test_fp16_operands_with_float32_o_are_well_inside_the_bar(case):
    err = max_err(case, emulate(case, torch.float16, None))
    assert max(err.values()) < BAR / 4, err


def test_bf16_operands_break_the_bar(case):
    fp16 = max_err(case, emulate(case, torch.float16, None))
    bf16 = max_err(case, emulate(case, torch.bfloat16, None))
    assert bf16["dk"] > BAR, bf16
    for n in ("dq", "dk", "dv"):
        assert bf16[n] > 4 * fp16[n], (n, bf16, fp16)


def test_o_stored_in_bf16_alone_moves_dk_past_the_bar(case):
    err = max_err(case, emulate(case, None, torch.bfloat16))
    assert err["dk"] > BAR, err
