"""GQA group sizes G = 2 and G = 16 on the tensor-core path, against the oracle.

The library accepts G in {1, 2, 4, 8, 16} for BF16 inputs; a 128-row tile is
then R = 128 / G tokens x G heads (R = 64 and R = 8 here). Every element of the
forward and of the backward is compared on ragged documents, with and without a
window and RoPE. (This file sorts after the parity files, so a failure here
stops none of them.)
"""
import pytest
import torch

import flint_inputs as fi
from oracle import flint_oracle as fo
from parity_util import check_grads, compare, run_bwd, run_fwd, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lens,H,Hk,W,rope", [
    ([300, 77], 32, 16, 96, True),       # G = 2, R = 64
    ([190, 1, 65], 32, 16, 0, False),
    ([300, 77], 32, 2, 96, True),        # G = 16, R = 8
    ([190, 1, 65], 32, 2, 0, False),
    ([129], 16, 1, 17, True),            # G = 16, one KV head
])
def test_group_size(cuda_lib, lens, H, Hk, W, rope):
    cpu = fi.make_custom(lens, H, Hk, dtype="bf16", seed=31 + H // Hk)
    d = to_dev(cpu)
    out, lse = run_fwd(cuda_lib, d, W, rope, 1e6, fp32_out=True)
    g = run_bwd(cuda_lib, d, out, lse, W, rope, 1e6, fp32_out=True)
    torch.cuda.synchronize()
    O, L = fo.flint_attn_fwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                             cpu["cu_doc_lens"], W, rope, 1e6)
    compare(out, O, "bf16", "out")
    compare(lse, L, "bf16", "lse")
    ref = fo.flint_attn_bwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                            cpu["cu_doc_lens"], W, rope, 1e6, cpu["dout"])
    check_grads(g, ref, label=f"group size {H // Hk}")
