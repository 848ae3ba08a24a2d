"""GPU parity of flint_attn_fwd_padded / flint_attn_bwd_padded (trailing padding
in every document) against the FP64 oracle, through the C ABI.

Real rows are held to the BF16 bar. Padded rows are checked exactly: out = 0,
lse = the sink logit, and every gradient row at a padded token is 0.
"""
import numpy as np
import pytest
import torch

import flint_inputs as fi
from oracle import flint_oracle as fo
from parity_util import check_grads, compare, f64, to_dev

pytestmark = pytest.mark.gpu


def padded_rows(cu, valid):
    rows = []
    for d, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        rows.extend(range(a + max(0, min(valid[d], b - a)), b))
    return rows


def run_padded(cuda_lib, d, valid_dev, W, rope, theta):
    out, lse = cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                            d["cu_doc_lens"], W, rope, theta, fp32_out=True,
                            valid_lens=valid_dev, check_status=True)
    g = cuda_lib.bwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     out, lse, d["dout"], W, rope, theta, fp32_out=True, valid_lens=valid_dev,
                     check_status=True)
    torch.cuda.synchronize()
    return out, lse, g


@pytest.mark.parametrize("lens,valid,W,rope", [
    ([300, 300, 300], [300, 150, 1], 0, True),       # BSHD, S = 300
    ([300, 300, 300], [17, 300, 256], 128, True),
    ([700, 333, 1], [500, 0, 1], 64, False),          # THD with per-document padding
])
def test_padded_matches_oracle(cuda_lib, lens, valid, W, rope):
    cpu = fi.make_custom(lens, 32, 4, dtype="bf16", seed=23)
    d = to_dev(cpu)
    vd = torch.tensor(valid, dtype=torch.int32, device="cuda")
    out, lse, g = run_padded(cuda_lib, d, vd, W, rope, 1e4)
    O, L = fo.flint_attn_fwd_padded(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"],
                                    cpu["sink"], cpu["cu_doc_lens"], valid, W, rope, 1e4)
    R = fo.flint_attn_bwd_padded(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"],
                                 cpu["sink"], cpu["cu_doc_lens"], valid, W, rope, 1e4,
                                 cpu["dout"])
    compare(out, O, "bf16", "out")
    compare(lse, L, "bf16", "lse")
    check_grads(g, R, label="padded")
    cu = [int(c) for c in cpu["cu_doc_lens"]]
    rows = padded_rows(cu, valid)
    assert rows
    assert torch.all(out[rows] == 0)
    assert torch.equal(lse[:, rows], cpu["sink"].cuda()[:, None].expand(-1, len(rows)))
    for name in ("dq", "dk", "dv"):
        assert torch.all(g[name][rows] == 0), name


def test_full_valid_lengths_equal_the_unpadded_call(cuda_lib):
    lens = [513, 300]
    cpu = fi.make_custom(lens, 32, 4, dtype="bf16", seed=4)
    d = to_dev(cpu)
    vd = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out_p, lse_p, g_p = run_padded(cuda_lib, d, vd, 128, True, 1e6)
    out, lse = cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                            d["cu_doc_lens"], 128, True, 1e6, fp32_out=True)
    g = cuda_lib.bwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     out, lse, d["dout"], 128, True, 1e6, fp32_out=True)
    torch.cuda.synchronize()
    assert torch.equal(out_p, out) and torch.equal(lse_p, lse)
    for name in g:
        assert torch.equal(g_p[name], g[name]), name


def test_bshd_8192_equals_the_layer_on_the_real_tokens(cuda_lib):
    """At scale (2 x 8192 slots): the real rows of the padded call are the layer over
    the real tokens alone - bit for bit for O, LSE, dq, dk, dv (same tiles, same
    order), to rounding for the sums over rows (d_sink, norm-weight gradients)."""
    S, valid = 8192, [8192, 5000]
    cpu = fi.make_custom([S, S], 32, 4, dtype="bf16", seed=8)
    d = to_dev(cpu)
    vd = torch.tensor(valid, dtype=torch.int32, device="cuda")
    out_p, lse_p, g_p = run_padded(cuda_lib, d, vd, 1024, True, 1e6)
    idx = torch.cat([torch.arange(0, valid[0]), torch.arange(S, S + valid[1])]).cuda()
    c = {k: d[k][idx] for k in ("q", "k", "v", "dout")}
    cu_c = torch.tensor([0, valid[0], valid[0] + valid[1]], dtype=torch.int32, device="cuda")
    out, lse = cuda_lib.fwd(c["q"], c["k"], c["v"], d["w_q"], d["w_k"], d["sink"], cu_c, 1024,
                            True, 1e6, fp32_out=True)
    g = cuda_lib.bwd(c["q"], c["k"], c["v"], d["w_q"], d["w_k"], d["sink"], cu_c, out, lse,
                     c["dout"], 1024, True, 1e6, fp32_out=True)
    torch.cuda.synchronize()
    assert torch.equal(out_p[idx], out) and torch.equal(lse_p[:, idx], lse)
    for name in ("dq", "dk", "dv"):
        assert torch.equal(g_p[name][idx], g[name]), name
    for name in ("dsink", "dw_q", "dw_k"):
        np.testing.assert_allclose(f64(g_p[name]), f64(g[name]), rtol=1e-4, atol=1e-4)
    rows = padded_rows([0, S, 2 * S], valid)
    assert torch.all(out_p[rows] == 0)
    for name in ("dq", "dk", "dv"):
        assert torch.all(g_p[name][rows] == 0), name


def test_fp32_padding_needs_a_tensor_core_group_size(cuda_lib):
    """FP32 inputs with G = 3 run the CUDA-core kernels, which have no padded form."""
    cpu = fi.make_custom([64], 3, 1, dtype="fp32", seed=1)
    d = to_dev(cpu)
    vd = torch.tensor([10], dtype=torch.int32, device="cuda")
    with pytest.raises(cuda_lib.FlintError) as e:
        cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     0, False, 1e4, valid_lens=vd)
    assert e.value.code == 2


def test_padding_contents_do_not_touch_real_rows(cuda_lib):
    """Whatever finite values a caller leaves in the padding (here +-3e7, far outside
    fp16's range) must not change the real rows: padded tokens are excluded from the
    attention and from the choice of the fp16 operand scales of v and dO."""
    lens, valid, W, rope, theta = [300, 300, 300], [300, 150, 1], 0, True, 1e6
    cpu = fi.make_custom(lens, 32, 4, dtype="bf16", seed=12)
    cu = [int(c) for c in cpu["cu_doc_lens"]]
    pad = padded_rows(cu, valid)
    gen = torch.Generator().manual_seed(5)
    for name in ("q", "k", "v", "dout"):
        t = cpu[name]
        noise = torch.sign(torch.randn(len(pad), *t.shape[1:], generator=gen)) * 3e7
        t[pad] = noise.to(t.dtype)
    d = to_dev(cpu)
    vd = torch.tensor(valid, dtype=torch.int32, device="cuda")
    out, lse, g = run_padded(cuda_lib, d, vd, W, rope, theta)
    O, L = fo.flint_attn_fwd_padded(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"],
                                    cpu["sink"], cpu["cu_doc_lens"], valid, W, rope, theta)
    R = fo.flint_attn_bwd_padded(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"],
                                 cpu["sink"], cpu["cu_doc_lens"], valid, W, rope, theta,
                                 cpu["dout"])
    real = [t for t in range(cu[-1]) if t not in set(pad)]
    compare(out[real], O[real], "bf16", "out")
    compare(lse[:, real], L[:, real], "bf16", "lse")
    for name in ("dq", "dk", "dv"):
        compare(g[name][real], R[name][real], "bf16", name)
        assert torch.all(g[name][pad] == 0), name
    assert torch.all(out[pad] == 0)
    compare(g["dsink"], R["dsink"], "bf16", "dsink")
