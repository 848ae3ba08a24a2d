"""An empty batch (every document of length 0, T = 0) through the C ABI.

The [T, ...] tensors are empty (their pointers are null); the forward writes
nothing and the backward writes zero d_sink and norm-weight gradients, which is
what the oracle's definition gives for a batch without tokens (a sum over no
rows). (This file sorts after the parity files, so a failure here stops none
of them.)
"""
import numpy as np
import pytest
import torch

import flint_inputs as fi
from oracle import flint_oracle as fo
from parity_util import f64, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("W,rope", [(0, False), (64, True)])
def test_empty_batch(cuda_lib, W, rope):
    cpu = fi.make_custom([0, 0], 32, 4, dtype="bf16", seed=3)
    d = to_dev(cpu)
    out, lse = cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                            d["cu_doc_lens"], W, rope, 1e4, fp32_out=True, check_status=True)
    g = cuda_lib.bwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     out, lse, d["dout"], W, rope, 1e4, fp32_out=True, check_status=True)
    torch.cuda.synchronize()
    assert out.shape == (0, 32, 128) and lse.shape == (32, 0)
    for name in ("dq", "dk", "dv"):
        assert g[name].numel() == 0, name
    ref = fo.flint_attn_bwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                            cpu["cu_doc_lens"], W, rope, 1e4, cpu["dout"])
    for name in ("dsink", "dw_q", "dw_k"):
        assert np.array_equal(f64(g[name]), ref[name]), name
        assert not np.any(ref[name])
