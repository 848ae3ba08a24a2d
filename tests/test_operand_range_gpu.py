"""BF16 (and FP32 at the fp16 boundary) inputs whose dO or v lie outside the range
fp16 represents well.

The tensor-core operands are IEEE fp16: normal numbers span 6.1e-5 .. 65504. A
training backward often sees dO of 1e-6 .. 1e-8 (a loss averaged over many
tokens), and nothing bounds v. The Flint config page's FlintConfig docstring
says fp16 compute needs a loss-scaling policy for small gradients; the library
applies one itself: the fp16 copies of dO and v are multiplied by a power of two
chosen from each tensor's largest magnitude, and the FP32 epilogues divide it
out again, exactly. These cases scale dO or v by factors from 1e-6 to 1e5 and
hold every output to the parity bar relative to the data's own scale: an
output that scales by c is compared as (gpu / c) against (oracle / c).
"""
import numpy as np
import pytest
import torch

import flint_inputs as fi
from oracle import flint_oracle as fo
from parity_util import DW_REL, compare, to_dev

pytestmark = pytest.mark.gpu

# How each result scales when dO or v is multiplied by c (O = P v; the
# gradients are linear in dO; dq, dk, d_sink and the norm-weight gradients go
# through dP = dO . v and D = dO . O, so they scale with both).
OUT_SCALE = {"dout": {"out": 0, "lse": 0, "dq": 1, "dk": 1, "dv": 1, "dw_q": 1, "dw_k": 1,
                      "dsink": 1},
             "v": {"out": 1, "lse": 0, "dq": 1, "dk": 1, "dv": 0, "dw_q": 1, "dw_k": 1,
                   "dsink": 1}}


def _scaled_inputs(dtype, which, factor, seed):
    cpu = fi.make_custom([300, 77, 150], 32, 4, dtype=dtype, seed=seed)
    t = cpu["dout"] if which == "dout" else cpu["v"]
    # scale, then round to the input dtype again: the oracle reads the same values
    cpu[which] = (t.double() * factor).to(t.dtype)
    return cpu


@pytest.mark.parametrize("which,factor", [("dout", 1e-6), ("dout", 1e-8), ("dout", 1e3),
                                          ("dout", 1e5), ("v", 1e-6), ("v", 1e3),
                                          ("v", 1e5)])
def test_bf16_operand_range(cuda_lib, which, factor):
    W, rope, theta = 96, True, 1e6
    cpu = _scaled_inputs("bf16", which, factor, seed=41)
    d = to_dev(cpu)
    out, lse = cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                            d["cu_doc_lens"], W, rope, theta, fp32_out=True, check_status=True)
    g = cuda_lib.bwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     out, lse, d["dout"], W, rope, theta, fp32_out=True, check_status=True)
    torch.cuda.synchronize()
    O, L = fo.flint_attn_fwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                             cpu["cu_doc_lens"], W, rope, theta)
    R = fo.flint_attn_bwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                          cpu["cu_doc_lens"], W, rope, theta, cpu["dout"])
    got = {"out": out, "lse": lse, **g}
    want = {"out": O, "lse": L, **R}
    for name, p in OUT_SCALE[which].items():
        c = factor ** p
        gv = got[name].double().cpu() / c
        red = {"dw_q": DW_REL, "dw_k": DW_REL}.get(name, 0.0)
        compare(gv, np.asarray(want[name]) / c, "bf16", f"{name} ({which} x {factor:g})",
                reduction=red)


@pytest.mark.parametrize("which,factor", [("v", 1e5), ("dout", 1e-7)])
def test_fp32_compute_f16_operand_range(cuda_lib, which, factor):
    """FP32 inputs at the fp16 boundary: any float32 magnitude reaches the fp16 operands."""
    W, rope, theta = 128, True, 1e4
    cpu = _scaled_inputs("fp32", which, factor, seed=43)
    d = to_dev(cpu)
    out, lse = cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                            d["cu_doc_lens"], W, rope, theta, compute_f16=True, fp32_out=True,
                            check_status=True)
    g = cuda_lib.bwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     out, lse, d["dout"], W, rope, theta, compute_f16=True, fp32_out=True,
                     check_status=True)
    torch.cuda.synchronize()
    O, L = fo.flint_attn_fwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                             cpu["cu_doc_lens"], W, rope, theta)
    R = fo.flint_attn_bwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                          cpu["cu_doc_lens"], W, rope, theta, cpu["dout"])
    got = {"out": out, "lse": lse, **g}
    want = {"out": O, "lse": L, **R}
    for name, p in OUT_SCALE[which].items():
        c = factor ** p
        red = {"dw_q": DW_REL, "dw_k": DW_REL}.get(name, 0.0)
        compare(got[name].double().cpu() / c, np.asarray(want[name]) / c, "bf16",
                f"{name} ({which} x {factor:g})", reduction=red)
