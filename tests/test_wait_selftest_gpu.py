"""Failure detection on the device, without a GPU fault.

The bounded mbarrier wait that every pipelined kernel uses must give up after
its limit, report FLINT_ERR_TIMEOUT through the status word (read by
flint_attn_check_status), and leave the CUDA context usable: the kernel exits
normally, and a layer call made afterwards still matches the oracle. The wait
in question is on a barrier that nothing completes; no kernel faults, traps or
hangs. (This file sorts last, so a failure here stops nothing else.)
"""
import pytest
import torch

import flint_inputs as fi
from oracle import flint_oracle as fo
from parity_util import compare, to_dev

pytestmark = pytest.mark.gpu

FLINT_OK, FLINT_ERR_TIMEOUT = 0, 5


def test_wait_that_nothing_completes_times_out(cuda_lib):
    code, completed = cuda_lib.selftest_wait(2_000_000, arrive_first=False)   # ~1 ms
    assert code == FLINT_ERR_TIMEOUT
    assert not completed


def test_completed_wait_passes(cuda_lib):
    code, completed = cuda_lib.selftest_wait(2_000_000, arrive_first=True)
    assert code == FLINT_OK
    assert completed


def test_context_is_usable_after_a_timeout(cuda_lib):
    code, _ = cuda_lib.selftest_wait(1000, arrive_first=False)
    assert code == FLINT_ERR_TIMEOUT
    cpu = fi.make_custom([300, 45], 32, 4, dtype="bf16", seed=12)
    d = to_dev(cpu)
    out, lse = cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                            d["cu_doc_lens"], 64, True, 1e4, fp32_out=True, check_status=True)
    torch.cuda.synchronize()
    O, L = fo.flint_attn_fwd(cpu["q"], cpu["k"], cpu["v"], cpu["w_q"], cpu["w_k"], cpu["sink"],
                             cpu["cu_doc_lens"], 64, True, 1e4)
    compare(out, O, "bf16", "out")
    compare(lse, L, "bf16", "lse")
