"""The forward and backward calls inside a CUDA graph.

A call is stream work only (a status-word memset and kernel launches on
caller-owned buffers, no host synchronisation), so a training step can capture
flint_attn_fwd + flint_attn_bwd once and replay the graph. Replays must give the
same bits as eager calls, also after new inputs are copied into the captured
buffers, and leave the status word clean.
"""
import pytest
import torch

import flint_inputs as fi
from parity_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_fwd_bwd_replay_from_a_cuda_graph(cuda_lib, dtype):
    lens, H, Hk, W, rope, theta = [300, 77, 150], 32, 4, 96, True, 1e6
    d = to_dev(fi.make_custom(lens, H, Hk, dtype=dtype, seed=12))
    p = cuda_lib.params_for(d["q"], d["k"], d["cu_doc_lens"], W, rope, theta, fp32_out=True)
    ws_f = cuda_lib.alloc_workspace(p, False)
    ws_b = cuda_lib.alloc_workspace(p, True)
    T, D = d["q"].shape[0], d["q"].shape[2]
    f32 = dict(dtype=torch.float32, device="cuda")
    out = torch.empty(T, H, D, **f32)
    lse = torch.empty(H, T, **f32)
    grads = {"dq": torch.empty(T, H, D, **f32), "dk": torch.empty(T, Hk, D, **f32),
             "dv": torch.empty(T, Hk, D, **f32), "dw_q": torch.empty(D, **f32),
             "dw_k": torch.empty(D, **f32), "dsink": torch.empty(H, **f32)}
    results = {"out": out, "lse": lse, **grads}

    def step():
        cuda_lib.fwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     W, rope, theta, out=out, lse=lse, workspace=ws_f, fp32_out=True)
        cuda_lib.bwd(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cu_doc_lens"],
                     out, lse, d["dout"], W, rope, theta, grads=grads, workspace=ws_b,
                     fp32_out=True)

    def snapshot():
        torch.cuda.synchronize()
        return {k: v.clone() for k, v in results.items()}

    step()
    eager = snapshot()
    # warm-up on a side stream, as torch asks before a capture
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for v in results.values():
        v.zero_()
    graph.replay()
    replayed = snapshot()
    for k in results:
        assert torch.equal(replayed[k], eager[k]), k
    # new inputs in the captured buffers: a replay equals a fresh eager call
    d2 = to_dev(fi.make_custom(lens, H, Hk, dtype=dtype, seed=13))
    for k in ("q", "k", "v", "dout", "w_q", "w_k", "sink"):
        d[k].copy_(d2[k])
    graph.replay()
    replayed = snapshot()
    step()
    eager = snapshot()
    for k in results:
        assert torch.equal(replayed[k], eager[k]), k
        assert not torch.equal(replayed[k], torch.zeros_like(replayed[k])), k
    lib = cuda_lib.load_library()
    for ws in (ws_f, ws_b):
        assert lib.flint_attn_check_status(cuda_lib._ptr(ws), cuda_lib._stream_ptr()) == 0
