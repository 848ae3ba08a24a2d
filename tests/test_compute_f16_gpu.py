"""FP32 inputs at the fp16 attention boundary (params.compute_f16, the Flint config
page's attention_compute_dtype='fp16'): RMSNorm and RoPE in FP32, q_hat, k_hat, v
and dO as fp16 tensor-core operands, out in fp16 (or float32 with fp32_out).
Held to the BF16 bar against the FP64 oracle; the run must use the tcgen05 kernels.
"""
import pytest
import torch

import flint_inputs as fi
from oracle import flint_oracle as fo
from parity_util import check_grads, compare, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fp32_out", [False, True])
def test_compute_f16_matches_oracle(cuda_lib, fp32_out):
    lens, W, rope = [700, 333, 1], 128, True
    cpu = fi.make_custom(lens, 32, 4, dtype="fp32", seed=31)
    d = to_dev(cpu)
    cuda_lib.profile_reset(); cuda_lib.profile_collect(); cuda_lib.profile_reset()
    cuda_lib.profile_enable(True)
    out, lse = cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                            d["cu_doc_lens"], W, rope, 1e4, compute_f16=True, fp32_out=fp32_out,
                            check_status=True)
    g = cuda_lib.bwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     out, lse, d["dout"], W, rope, 1e4, compute_f16=True, fp32_out=fp32_out,
                     check_status=True)
    torch.cuda.synchronize()
    cuda_lib.profile_enable(False)
    k = cuda_lib.profile_collect()
    for name in ("attn_fwd_sm100", "attn_bwd_dkv_sm100", "attn_bwd_dq_sm100"):
        assert k[name][1] == 1, name
    for name in ("attn_fwd_fp32", "attn_bwd_dkv_fp32", "attn_bwd_dq_fp32"):
        assert k[name][1] == 0, name
    assert out.dtype == (torch.float32 if fp32_out else torch.float16)
    assert g["dq"].dtype == torch.float32
    O, L = fo.flint_attn_fwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                             cpu["cu_doc_lens"], W, rope, 1e4)
    R = fo.flint_attn_bwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                          cpu["cu_doc_lens"], W, rope, 1e4, cpu["dout"])
    compare(out, O, "bf16", "out")
    compare(lse, L, "bf16", "lse")
    check_grads(g, R, label="compute_f16")


def test_compute_f16_with_padding(cuda_lib):
    lens, valid, W = [300, 300], [120, 300], 0
    cpu = fi.make_custom(lens, 32, 4, dtype="fp32", seed=6)
    d = to_dev(cpu)
    vd = torch.tensor(valid, dtype=torch.int32, device="cuda")
    out, lse = cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                            d["cu_doc_lens"], W, False, 1e4, compute_f16=True, valid_lens=vd,
                            check_status=True)
    O, L = fo.flint_attn_fwd_padded(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"],
                                    cpu["sink"], cpu["cu_doc_lens"], valid, W, False, 1e4)
    torch.cuda.synchronize()
    assert out.dtype == torch.float16
    compare(out, O, "bf16", "out")
    compare(lse, L, "bf16", "lse")
    assert torch.all(out[120:300] == 0)
