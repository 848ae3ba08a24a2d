"""The no-allocation backward preprocess against the regular backward.

``flint_attn_bwd_preprocess_static`` serves callers that cannot allocate device
memory where they run: it takes only inputs and outputs and keeps its scratch
in a fixed array inside the library. Its d_sink must equal the one the regular
``flint_attn_bwd`` (which uses a caller workspace) returns, call after call,
for every storage type of out the forward can write.
This file is collected after the parity files on purpose, so that under -x a
failure here stops none of them.
"""
import pytest
import torch

import flint_inputs as fi
from parity_util import compare, to_dev

pytestmark = pytest.mark.gpu

# (input dtype, fp32_out, compute_f16) -> out is bf16 / fp32 / fp32 / fp16 / fp32
TYPE_CASES = [("bf16", True, False), ("bf16", False, False), ("fp32", False, False),
              ("fp32", False, True), ("fp32", True, True)]


@pytest.mark.parametrize("dtype,fp32_out,compute_f16", TYPE_CASES)
def test_static_preprocess_matches_regular_backward(cuda_lib, dtype, fp32_out, compute_f16):
    lens, H, Hk, W, rope = [700, 333, 1], 32, 4, 128, True
    cpu = fi.make_custom(lens, H, Hk, dtype=dtype, seed=17)
    d = to_dev(cpu)
    kw = dict(fp32_out=fp32_out, compute_f16=compute_f16, check_status=True)
    out, lse = cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                            d["cu_doc_lens"], W, rope, 1e6, **kw)
    g = cuda_lib.bwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     out, lse, d["dout"], W, rope, 1e6, **kw)
    torch.cuda.synchronize()
    want_out = (torch.float32 if (fp32_out or (dtype == "fp32" and not compute_f16))
                else torch.float16 if compute_f16 else torch.bfloat16)
    assert out.dtype == want_out
    dsink_regular = g["dsink"].clone()
    rowsum = (d["dout"].double() * out.double()).sum(-1).transpose(0, 1)   # [H, T]
    for _ in range(2):                      # two calls in a row share the scratch
        D, dsink = cuda_lib.bwd_preprocess_static(out, d["dout"], lse, d["sink"])
        torch.cuda.synchronize()
        compare(dsink, dsink_regular.double().cpu().numpy(), "fp32", "dsink")
        compare(D, rowsum.cpu().numpy(), "fp32", "D")


def test_static_preprocess_empty_batch(cuda_lib):
    """T = 0: null token tensors are accepted and d_sink comes back zero."""
    H = 32
    empty = torch.empty(0, H, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(H, 0, device="cuda")
    sink = torch.randn(H, device="cuda")
    D, dsink = cuda_lib.bwd_preprocess_static(empty, empty, lse, sink,
                                              dsink=torch.full((H,), 7.0, device="cuda"))
    torch.cuda.synchronize()
    assert D.shape == (H, 0)
    assert torch.all(dsink == 0)


def test_static_preprocess_rejects_too_many_heads(cuda_lib):
    T, H = 16, 256
    out = torch.zeros(T, H, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(H, T, device="cuda")
    sink = torch.zeros(H, device="cuda")
    with pytest.raises(cuda_lib.FlintError) as e:
        cuda_lib.bwd_preprocess_static(out, out, lse, sink)
    assert e.value.code == 3          # FLINT_ERR_WORKSPACE, nothing launched
