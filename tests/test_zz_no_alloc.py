"""The no-allocation backward preprocess against the regular backward.

``flint_attn_bwd_preprocess_static`` serves callers that cannot allocate device
memory where they run: it takes only inputs and outputs and keeps its scratch
in a fixed array inside the library. Its d_sink must equal the one the regular
``flint_attn_bwd`` (which uses a caller workspace) returns, call after call.
This file is collected after the parity files on purpose, so that under -x a
failure here stops none of them.
"""
import pytest
import torch

import flint_inputs as fi
from parity_util import compare, run_bwd, run_fwd, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fp32_out", [True, False])
def test_static_preprocess_matches_regular_backward(cuda_lib, fp32_out):
    lens, H, Hk, W, rope = [700, 333, 1], 32, 4, 128, True
    cpu = fi.make_custom(lens, H, Hk, dtype="bf16", seed=17)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, W, rope, 1e6, fp32_out=fp32_out)
    g = run_bwd(cuda_lib, d, out, lse, W, rope, 1e6, fp32_out=fp32_out)
    torch.cuda.synchronize()
    dsink_regular = g["dsink"].clone()
    rowsum = (d["dout"].float() * out.float()).sum(-1).transpose(0, 1)   # [H, T]
    for _ in range(2):                      # two calls in a row share the scratch
        D, dsink = cuda_lib.bwd_preprocess_static(out, d["dout"], lse, d["sink"],
                                                  fp32_out=fp32_out)
        torch.cuda.synchronize()
        compare(dsink, dsink_regular.double().cpu().numpy(), "fp32", "dsink")
        compare(D, rowsum.double().cpu().numpy(), "bf16", "D")


def test_static_preprocess_rejects_too_many_heads(cuda_lib):
    T, H = 16, 256
    out = torch.zeros(T, H, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(H, T, device="cuda")
    sink = torch.zeros(H, device="cuda")
    with pytest.raises(cuda_lib.FlintError) as e:
        cuda_lib.bwd_preprocess_static(out, out, lse, sink)
    assert e.value.code == 3          # FLINT_ERR_WORKSPACE, nothing launched
