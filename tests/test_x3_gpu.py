"""FP32 inputs on the split tensor-core path: every operand enters the tcgen05
MMAs as fp16 hi and lo parts and every product takes three MMAs
(hi*hi + hi*lo + lo*hi), so the FP32 parity bar of 1e-4 max-abs holds on the
tensor cores (Flint config page: FP32 is the native attention_compute_dtype).

Every output element is compared with the FP64 oracle. The per-row outputs
(out, lse, dq, dk, dv) are held to max-abs 1e-4 at every size. d_sink and the
norm-weight gradients sum a head's T rows and all T*H rows: each row brings the
relative error of the split products (measured 1e-6 .. 2e-6 on the dq, dk, dv
rows) and the sums cancel heavily (|sum| is far below the sum of the rows'
magnitudes), so they are held to 1e-4 + 1e-5 * max|ref|. The 256-token FP32
layer meets the plain 1e-4 on every output, sums included
(test_parity_gpu.test_tiny_sliding_fp32_forward_backward). Raw errors are
printed (pytest -s) next to the bars.
"""
import numpy as np
import pytest
import torch

import flint_inputs as fi
from oracle import flint_oracle as fo
from parity_util import FP32_MAX_ABS, f64, to_dev

pytestmark = pytest.mark.gpu

SUM_REL = 1e-5
SUMS = ("dsink", "dw_q", "dw_k")
SPLIT_KERNELS = ("attn_fwd_x3_sm100", "attn_bwd_dkv_x3_sm100", "attn_bwd_dq_x3_sm100")
CORE_KERNELS = ("attn_fwd_fp32", "attn_bwd_dkv_fp32", "attn_bwd_dq_fp32")


def _check(name, gpu, ref, bar_rel=0.0):
    g, r = f64(gpu), np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (name, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{name}: non-finite GPU values"
    err = float(np.max(np.abs(g - r))) if r.size else 0.0
    bar = FP32_MAX_ABS + bar_rel * (float(np.max(np.abs(r))) if r.size else 0.0)
    print(f"X3 {name}: max_abs {err:.3e} (bar {bar:.3e}, max|ref| "
          f"{float(np.max(np.abs(r))) if r.size else 0.0:.3g})")
    assert err <= bar, f"{name}: max_abs {err:.3e} > {bar:.3e}"


def _run(cuda_lib, cpu, W, rope, theta, valid=None):
    d = to_dev(cpu)
    vd = None if valid is None else torch.tensor(valid, dtype=torch.int32, device="cuda")
    cuda_lib.profile_reset(); cuda_lib.profile_collect(); cuda_lib.profile_reset()
    cuda_lib.profile_enable(True)
    out, lse = cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                            d["cu_doc_lens"], W, rope, theta, valid_lens=vd, check_status=True)
    g = cuda_lib.bwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     out, lse, d["dout"], W, rope, theta, valid_lens=vd, check_status=True)
    torch.cuda.synchronize()
    cuda_lib.profile_enable(False)
    return out, lse, g, cuda_lib.profile_collect()


def _oracle(cpu, W, rope, theta):
    O, L = fo.flint_attn_fwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                             cpu["cu_doc_lens"], W, rope, theta)
    R = fo.flint_attn_bwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                          cpu["cu_doc_lens"], W, rope, theta, cpu["dout"])
    return O, L, R


def _compare_all(out, lse, g, O, L, R, label):
    _check(f"{label} out", out, O)
    _check(f"{label} lse", lse, L)
    for name in ("dq", "dk", "dv"):
        _check(f"{label} {name}", g[name], R[name])
    for name in SUMS:
        _check(f"{label} {name}", g[name], R[name], SUM_REL)


CASES = [
    # doc lengths, H, Hk, window, rope, theta
    ([300], 32, 4, 64, True, 1e4),
    ([257, 1, 130, 7], 32, 4, 63, True, 1e6),
    ([200, 0, 333], 32, 4, 0, False, 1e6),
    ([513], 32, 4, 1, True, 1e4),
    ([129, 64], 32, 4, 2, False, 1e6),
    ([31, 17, 290], 16, 2, 100, True, 1e6),
    ([160, 96], 8, 1, 0, True, 1e4),          # G = 8
    ([384], 16, 4, 128, False, 1e6),          # G = 4
    ([70, 260], 4, 4, 50, True, 1e4),         # G = 1
    ([333], 8, 4, 0, True, 1e4),              # G = 2
    ([200, 99], 16, 1, 77, False, 1e6),       # G = 16
    ([1100], 32, 4, 0, True, 1e6),            # many key tiles per query tile
]


@pytest.mark.parametrize("lens,H,Hk,W,rope,theta", CASES)
def test_split_path_matches_oracle(cuda_lib, lens, H, Hk, W, rope, theta):
    cpu = fi.make_custom(lens, H, Hk, dtype="fp32", seed=sum(lens) + H + W)
    out, lse, g, k = _run(cuda_lib, cpu, W, rope, theta)
    for name in SPLIT_KERNELS:
        assert k[name][1] == 1, name
    for name in CORE_KERNELS:
        assert k[name][1] == 0, name
    assert out.dtype == torch.float32 and g["dv"].dtype == torch.float32
    O, L, R = _oracle(cpu, W, rope, theta)
    _compare_all(out, lse, g, O, L, R, f"{lens} H{H}/{Hk} W{W}")


def test_other_group_sizes_stay_on_cuda_cores(cuda_lib):
    """G = 3 has no tensor-core tile; FP32 inputs then run the CUDA-core kernels."""
    lens, W = [150, 40], 33
    cpu = fi.make_custom(lens, 6, 2, dtype="fp32", seed=5)
    out, lse, g, k = _run(cuda_lib, cpu, W, True, 1e4)
    for name in CORE_KERNELS:
        assert k[name][1] == 1, name
    for name in SPLIT_KERNELS:
        assert k[name][1] == 0, name
    O, L, R = _oracle(cpu, W, True, 1e4)
    _compare_all(out, lse, g, O, L, R, "G3")


@pytest.mark.parametrize("which,factor", [("v", 1e-6), ("v", 1e5), ("dout", 1e-8),
                                          ("dout", 1e4)])
def test_split_operand_range(cuda_lib, which, factor):
    """v and dO far from N(0,1): their parts are scaled by a power of two chosen from
    the tensor's max |x|, which the epilogues divide out. Each output is compared
    relative to its own scale (an output that scales by c as gpu / c against
    oracle / c)."""
    scale_of = {"dout": {"out": 0, "lse": 0, "dq": 1, "dk": 1, "dv": 1, "dw_q": 1, "dw_k": 1,
                         "dsink": 1},
                "v": {"out": 1, "lse": 0, "dq": 1, "dk": 1, "dv": 0, "dw_q": 1, "dw_k": 1,
                      "dsink": 1}}[which]
    W, rope, theta = 96, True, 1e6
    cpu = fi.make_custom([300, 77, 150], 32, 4, dtype="fp32", seed=43)
    cpu[which] = (cpu[which].double() * factor).to(torch.float32)
    out, lse, g, _ = _run(cuda_lib, cpu, W, rope, theta)
    O, L, R = _oracle(cpu, W, rope, theta)
    got = {"out": out, "lse": lse, **g}
    want = {"out": O, "lse": L, **R}
    for name, p in scale_of.items():
        c = factor ** p
        _check(f"{name} ({which} x {factor:g})", f64(got[name]) / c,
               np.asarray(want[name]) / c, SUM_REL if name in SUMS else 0.0)


def test_split_path_with_padding(cuda_lib):
    """The padded calls on the split path: real rows as the oracle's padded layer,
    padding rows out = 0, lse = sink, zero gradients."""
    lens, valid, W, rope, theta = [300, 300], [120, 300], 0, True, 1e4
    cpu = fi.make_custom(lens, 32, 4, dtype="fp32", seed=6)
    out, lse, g, k = _run(cuda_lib, cpu, W, rope, theta, valid=valid)
    assert k["attn_fwd_x3_sm100"][1] == 1
    O, L = fo.flint_attn_fwd_padded(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"],
                                    cpu["sink"], cpu["cu_doc_lens"], valid, W, rope, theta)
    R = fo.flint_attn_bwd_padded(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"],
                                 cpu["sink"], cpu["cu_doc_lens"], valid, W, rope, theta,
                                 cpu["dout"])
    _compare_all(out, lse, g, O, L, R, "padded")
    assert torch.all(out[120:300] == 0)
    assert torch.all(g["dq"][120:300] == 0) and torch.all(g["dv"][120:300] == 0)


def test_split_path_full_size_sampled(cuda_lib):
    """The 32768-token full-causal layer with FP32 inputs: sampled rows of every output
    against the row oracle at max-abs 1e-4, including the keys at the document start,
    which every one of the 32768 x 8 query rows of their group sees (the longest
    accumulation of the dK/dV kernel)."""
    wl = fi.FULL_FP32
    cpu = fi.make_inputs(wl)
    d = to_dev(cpu)
    out, lse, g, k = _run(cuda_lib, cpu, wl.window, wl.use_rope, wl.rope_theta)
    for name in SPLIT_KERNELS:
        assert k[name][1] == 1, name
    ro = fo.RowOracle(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                      cpu["cu_doc_lens"], wl.window, wl.use_rope, wl.rope_theta, dO=cpu["dout"])
    T = wl.total_tokens
    toks = [0, 1, 127, 128, 255, 4095, 16383, 16384, T - 129, T - 1]
    O, L = ro.forward_rows(toks)
    _check("full fp32 out rows", out[toks], O)
    _check("full fp32 lse rows", lse[:, toks], L)
    rng = np.random.default_rng(3)
    rows = [(t, int(rng.integers(0, wl.num_q_heads))) for t in toks]
    _check("full fp32 dq rows", torch.stack([g["dq"][t, h] for t, h in rows]),
           np.stack([ro.dq_row(t, h) for t, h in rows]))
    for kv, keys in ((0, [0, 1, 127, 128, 16383]), (3, [T - 130, T - 1])):
        dk, dv = ro.dkv_rows(keys, kv)
        _check(f"full fp32 dk rows kv{kv}", g["dk"][keys, kv], dk)
        _check(f"full fp32 dv rows kv{kv}", g["dv"][keys, kv], dv)
