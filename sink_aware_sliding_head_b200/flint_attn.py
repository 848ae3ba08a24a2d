"""Python binding of the C ABI in ``include/flint_attn.h`` (ctypes).

Argument marshalling only: tensors are allocated with torch on the current CUDA
device and passed as raw device pointers together with torch's current stream.
Every step of the computation runs in the library's CUDA kernels. There is no
CPU or PyTorch fallback: if the library is missing or a call fails, an error is
raised.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libflint_attn.so")

FLINT_BF16 = 0
FLINT_FP32 = 1

STATUS = {0: "FLINT_OK", 1: "FLINT_ERR_INVALID_ARG", 2: "FLINT_ERR_UNSUPPORTED",
          3: "FLINT_ERR_WORKSPACE", 4: "FLINT_ERR_CUDA", 5: "FLINT_ERR_TIMEOUT"}

EXPORTED = ["flint_attn_workspace_bytes", "flint_attn_fwd", "flint_attn_bwd",
            "flint_attn_check_status", "flint_status_string", "flint_attn_version",
            "flint_attn_profile_enable", "flint_attn_profile_collect",
            "flint_attn_profile_reset", "flint_attn_launch_count",
            "flint_attn_bwd_preprocess_static", "flint_attn_exp2_poly",
            "flint_attn_decode_workspace_bytes", "flint_attn_decode",
            "flint_attn_fwd_padded", "flint_attn_bwd_padded", "flint_attn_selftest_wait"]


class Params(ctypes.Structure):
    """Mirror of ``flint_attn_params_t``."""
    _fields_ = [
        ("total_tokens", ctypes.c_int32),
        ("num_docs", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("use_rope", ctypes.c_int32),
        ("rope_theta", ctypes.c_float),
        ("rms_eps", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
        ("dtype", ctypes.c_int32),
        ("fp32_out", ctypes.c_int32),
        ("compute_f16", ctypes.c_int32),
    ]


class DecodeParams(ctypes.Structure):
    """Mirror of ``flint_decode_params_t``."""
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("cache_capacity", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("use_rope", ctypes.c_int32),
        ("rope_theta", ctypes.c_float),
        ("rms_eps", ctypes.c_float),
        ("softmax_scale", ctypes.c_float),
        ("dtype", ctypes.c_int32),
        ("fp32_out", ctypes.c_int32),
    ]


class FlintError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


_lib = None


def load_library(path: str = LIB_PATH):
    """Load (once) and return the ctypes handle; raises if the library is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"CUDA library not built: {path} (run python -m "
                          "sink_aware_sliding_head_b200.build)")
    lib = ctypes.CDLL(path)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    P = ctypes.POINTER(Params)
    lib.flint_attn_workspace_bytes.argtypes = [P, ctypes.c_int]
    lib.flint_attn_workspace_bytes.restype = sz
    lib.flint_attn_fwd.argtypes = [P] + [vp] * 9 + [vp, sz, vp]
    lib.flint_attn_fwd.restype = ctypes.c_int
    lib.flint_attn_bwd.argtypes = [P] + [vp] * 16 + [vp, sz, vp]
    lib.flint_attn_bwd.restype = ctypes.c_int
    lib.flint_attn_fwd_padded.argtypes = [P] + [vp] * 10 + [vp, sz, vp]
    lib.flint_attn_fwd_padded.restype = ctypes.c_int
    lib.flint_attn_bwd_padded.argtypes = [P] + [vp] * 17 + [vp, sz, vp]
    lib.flint_attn_bwd_padded.restype = ctypes.c_int
    lib.flint_attn_check_status.argtypes = [vp, vp]
    lib.flint_attn_check_status.restype = ctypes.c_int
    lib.flint_status_string.argtypes = [ctypes.c_int]
    lib.flint_status_string.restype = ctypes.c_char_p
    lib.flint_attn_version.argtypes = []
    lib.flint_attn_version.restype = ctypes.c_char_p
    lib.flint_attn_profile_enable.argtypes = [ctypes.c_int]
    lib.flint_attn_profile_enable.restype = None
    lib.flint_attn_profile_collect.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_char_p),
                                               ctypes.POINTER(ctypes.c_double),
                                               ctypes.POINTER(ctypes.c_longlong)]
    lib.flint_attn_profile_collect.restype = ctypes.c_int
    lib.flint_attn_profile_reset.argtypes = []
    lib.flint_attn_profile_reset.restype = None
    lib.flint_attn_launch_count.argtypes = []
    lib.flint_attn_launch_count.restype = ctypes.c_longlong
    lib.flint_attn_bwd_preprocess_static.argtypes = [P] + [vp] * 6 + [vp]
    lib.flint_attn_bwd_preprocess_static.restype = ctypes.c_int
    lib.flint_attn_exp2_poly.argtypes = [vp, vp, ctypes.c_int32, vp]
    lib.flint_attn_exp2_poly.restype = ctypes.c_int
    lib.flint_attn_selftest_wait.argtypes = [ctypes.c_int64, ctypes.c_int32, vp, vp]
    lib.flint_attn_selftest_wait.restype = ctypes.c_int
    DP = ctypes.POINTER(DecodeParams)
    lib.flint_attn_decode_workspace_bytes.argtypes = [DP]
    lib.flint_attn_decode_workspace_bytes.restype = sz
    lib.flint_attn_decode.argtypes = [DP] + [vp] * 11 + [vp, sz, vp]
    lib.flint_attn_decode.restype = ctypes.c_int
    _lib = lib
    return lib


def make_params(total_tokens, num_docs, num_q_heads, num_kv_heads, window, use_rope,
                rope_theta, dtype, head_dim=128, rms_eps=1e-6, softmax_scale=0.0,
                fp32_out=False, compute_f16=False) -> Params:
    return Params(int(total_tokens), int(num_docs), int(num_q_heads), int(num_kv_heads),
                  int(head_dim), int(window), 1 if use_rope else 0, float(rope_theta),
                  float(rms_eps), float(softmax_scale), int(dtype), 1 if fp32_out else 0,
                  1 if compute_f16 else 0)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FLINT_BF16
    if t.dtype == torch.float32:
        return FLINT_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream_ptr(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(code: int, where: str):
    if code != 0:
        raise FlintError(code, where)


def params_for(q, k, cu_doc_lens, window, use_rope, rope_theta, rms_eps=1e-6,
               softmax_scale=0.0, fp32_out=False, compute_f16=False) -> Params:
    T, H, D = q.shape
    return make_params(T, cu_doc_lens.numel() - 1, H, k.shape[1], window, use_rope, rope_theta,
                       _dtype_code(q), head_dim=D, rms_eps=rms_eps, softmax_scale=softmax_scale,
                       fp32_out=fp32_out, compute_f16=compute_f16)


def workspace_bytes(params: Params, backward: bool) -> int:
    return int(load_library().flint_attn_workspace_bytes(ctypes.byref(params), int(backward)))


def alloc_workspace(params: Params, backward: bool, device=None) -> torch.Tensor:
    n = workspace_bytes(params, backward)
    if n == 0:
        raise FlintError(1, "flint_attn_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def fwd(q, k, v, q_norm_w, k_norm_w, sink, cu_doc_lens, window, use_rope, rope_theta,
        rms_eps=1e-6, softmax_scale=0.0, out=None, lse=None, workspace=None, stream=None,
        check_status=False, fp32_out=False, valid_lens=None, compute_f16=False):
    """Forward through ``flint_attn_fwd``. Returns (out [T,H,D], lse [H,T] fp32).

    ``fp32_out``: out is float32 (pass it unchanged to ``bwd`` with the same flag).
    ``valid_lens``: int32 [num_docs] on the device, the real tokens at the start of
    each document (trailing padding; ``flint_attn_fwd_padded``).
    ``compute_f16`` (float32 inputs): the fp16 attention boundary; out is float16
    unless ``fp32_out``.
    """
    lib = load_library()
    p = params_for(q, k, cu_doc_lens, window, use_rope, rope_theta, rms_eps, softmax_scale,
                   fp32_out, compute_f16)
    T, H, D = q.shape
    if out is None:
        odt = torch.float32 if fp32_out else (torch.float16 if compute_f16 else q.dtype)
        out = torch.empty(q.shape, dtype=odt, device=q.device)
    if lse is None:
        lse = torch.empty(H, T, dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(p, False, q.device)
    st = _stream_ptr(stream)
    if valid_lens is None:
        code = lib.flint_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w),
                                  _ptr(k_norm_w), _ptr(sink), _ptr(cu_doc_lens), _ptr(out),
                                  _ptr(lse), _ptr(workspace), workspace.numel(), st)
    else:
        code = lib.flint_attn_fwd_padded(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(q_norm_w), _ptr(k_norm_w), _ptr(sink),
                                         _ptr(cu_doc_lens), _ptr(valid_lens), _ptr(out),
                                         _ptr(lse), _ptr(workspace), workspace.numel(), st)
    _check(code, "flint_attn_fwd")
    if check_status:
        _check(lib.flint_attn_check_status(_ptr(workspace), st), "flint_attn_fwd (device)")
    return out, lse


def bwd(q, k, v, q_norm_w, k_norm_w, sink, cu_doc_lens, out, lse, dout, window, use_rope,
        rope_theta, rms_eps=1e-6, softmax_scale=0.0, grads=None, workspace=None, stream=None,
        check_status=False, fp32_out=False, valid_lens=None, compute_f16=False):
    """Backward through ``flint_attn_bwd`` (``flint_attn_bwd_padded`` with ``valid_lens``).

    Returns a dict with dq, dk, dv (input dtype, or float32 with ``fp32_out``),
    dw_q, dw_k, dsink (fp32). ``out`` must be the forward's result with the same
    ``fp32_out``.
    """
    lib = load_library()
    p = params_for(q, k, cu_doc_lens, window, use_rope, rope_theta, rms_eps, softmax_scale,
                   fp32_out, compute_f16)
    T, H, D = q.shape
    gdt = torch.float32 if (fp32_out or q.dtype == torch.float32) else q.dtype
    if grads is None:
        grads = {
            "dq": torch.empty(q.shape, dtype=gdt, device=q.device),
            "dk": torch.empty(k.shape, dtype=gdt, device=q.device),
            "dv": torch.empty(v.shape, dtype=gdt, device=q.device),
            "dw_q": torch.empty(D, dtype=torch.float32, device=q.device),
            "dw_k": torch.empty(D, dtype=torch.float32, device=q.device),
            "dsink": torch.empty(H, dtype=torch.float32, device=q.device),
        }
    if workspace is None:
        workspace = alloc_workspace(p, True, q.device)
    st = _stream_ptr(stream)
    g = [_ptr(grads[n]) for n in ("dq", "dk", "dv", "dw_q", "dw_k", "dsink")]
    if valid_lens is None:
        code = lib.flint_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w),
                                  _ptr(k_norm_w), _ptr(sink), _ptr(cu_doc_lens), _ptr(out),
                                  _ptr(lse), _ptr(dout), *g, _ptr(workspace), workspace.numel(),
                                  st)
    else:
        code = lib.flint_attn_bwd_padded(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(q_norm_w), _ptr(k_norm_w), _ptr(sink),
                                         _ptr(cu_doc_lens), _ptr(valid_lens), _ptr(out),
                                         _ptr(lse), _ptr(dout), *g, _ptr(workspace),
                                         workspace.numel(), st)
    _check(code, "flint_attn_bwd")
    if check_status:
        _check(lib.flint_attn_check_status(_ptr(workspace), st), "flint_attn_bwd (device)")
    return grads


def profile_enable(on: bool = True):
    """Bracket each later kernel launch with CUDA events on its stream."""
    load_library().flint_attn_profile_enable(1 if on else 0)


def profile_reset():
    load_library().flint_attn_profile_reset()


def profile_collect():
    """{kernel name: (total ms, launches)} over the launches timed so far."""
    lib = load_library()
    n = 32
    names = (ctypes.c_char_p * n)()
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_longlong * n)()
    k = lib.flint_attn_profile_collect(n, names, ms, cnt)
    return {names[i].decode(): (ms[i], cnt[i]) for i in range(min(k, n))}


def launch_count() -> int:
    """Kernels the library has launched since it was loaded."""
    return int(load_library().flint_attn_launch_count())


def bwd_preprocess_static(out, dout, lse, sink, d_rowsum=None, dsink=None, stream=None):
    """D = rowsum(dout * out) [H,T] and d_sink [H] through the no-allocation entry point.

    For callers that cannot allocate device memory where they run: the library
    uses a fixed scratch array of its own instead of a caller workspace (see
    ``flint_attn_bwd_preprocess_static`` in include/flint_attn.h for its limits).
    The input type is dout's (bfloat16 or float32); out's type says how the
    forward stored it: bfloat16 inputs take a bfloat16 or float32 out (fp32_out),
    float32 inputs a float32 out, or float16 for the fp16 compute boundary
    (compute_f16).
    """
    lib = load_library()
    if out.dim() != 3 or dout.shape != out.shape:
        raise ValueError(f"out {tuple(out.shape)} and dout {tuple(dout.shape)} must both be [T,H,D]")
    T, H, D = out.shape
    if lse.shape != (H, T) or lse.dtype != torch.float32:
        raise ValueError(f"lse must be float32 [H,T] = [{H},{T}], got {lse.dtype} {tuple(lse.shape)}")
    if sink.shape != (H,) or sink.dtype != torch.float32:
        raise ValueError(f"sink must be float32 [H] = [{H}], got {sink.dtype} {tuple(sink.shape)}")
    allowed = {torch.bfloat16: (torch.bfloat16, torch.float32),
               torch.float32: (torch.float32, torch.float16)}
    if dout.dtype not in allowed or out.dtype not in allowed[dout.dtype]:
        raise TypeError(f"unsupported pair: dout {dout.dtype}, out {out.dtype}")
    fp32_out = out.dtype == torch.float32
    compute_f16 = out.dtype == torch.float16
    p = make_params(T, 1, H, 1, 0, False, 0.0, _dtype_code(dout), head_dim=D,
                    fp32_out=fp32_out, compute_f16=compute_f16)
    if d_rowsum is None:
        d_rowsum = torch.empty(H, T, dtype=torch.float32, device=dout.device)
    if dsink is None:
        dsink = torch.empty(H, dtype=torch.float32, device=dout.device)
    code = lib.flint_attn_bwd_preprocess_static(ctypes.byref(p), _ptr(out), _ptr(dout), _ptr(lse),
                                                _ptr(sink), _ptr(d_rowsum), _ptr(dsink),
                                                _stream_ptr(stream))
    _check(code, "flint_attn_bwd_preprocess_static")
    return d_rowsum, dsink


def decode_params(batch, cache_capacity, num_q_heads, num_kv_heads, window, use_rope,
                  rope_theta, rms_eps=1e-6, softmax_scale=0.0, fp32_out=False,
                  head_dim=128) -> DecodeParams:
    return DecodeParams(int(batch), int(cache_capacity), int(num_q_heads), int(num_kv_heads),
                        int(head_dim), int(window), 1 if use_rope else 0, float(rope_theta),
                        float(rms_eps), float(softmax_scale), FLINT_BF16,
                        1 if fp32_out else 0)


def decode(q, k, v, q_norm_w, k_norm_w, sink, cache_lens, k_cache, v_cache, window, use_rope,
           rope_theta, rms_eps=1e-6, softmax_scale=0.0, out=None, lse=None, workspace=None,
           stream=None, check_status=False, fp32_out=False):
    """One new token per sequence through ``flint_attn_decode``.

    q [B,H,D], k, v [B,Hk,D] bf16 (raw projections of the new tokens); cache_lens
    [B] int32 on the device; k_cache, v_cache [B,Hk,C,D] bf16, updated in place
    at slot cache_lens[b]. Returns (out [B,H,D], lse [B,H] fp32).
    """
    lib = load_library()
    B, H, D = q.shape
    Hk, C = k_cache.shape[1], k_cache.shape[2]
    p = decode_params(B, C, H, Hk, window, use_rope, rope_theta, rms_eps, softmax_scale,
                      fp32_out, D)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32 if fp32_out else q.dtype,
                          device=q.device)
    if lse is None:
        lse = torch.empty(B, H, dtype=torch.float32, device=q.device)
    if workspace is None:
        n = lib.flint_attn_decode_workspace_bytes(ctypes.byref(p))
        if n == 0:
            raise FlintError(1, "flint_attn_decode_workspace_bytes")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    st = _stream_ptr(stream)
    code = lib.flint_attn_decode(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(q_norm_w),
                                 _ptr(k_norm_w), _ptr(sink), _ptr(cache_lens), _ptr(k_cache),
                                 _ptr(v_cache), _ptr(out), _ptr(lse), _ptr(workspace),
                                 workspace.numel(), st)
    _check(code, "flint_attn_decode")
    if check_status:
        _check(lib.flint_attn_check_status(_ptr(workspace), st), "flint_attn_decode (device)")
    return out, lse


def exp2_poly(x: torch.Tensor) -> torch.Tensor:
    """Diagnostic: the kernels' FMA-pipe 2^x evaluated on the device (fp32, even length)."""
    y = torch.empty_like(x)
    _check(load_library().flint_attn_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream_ptr()),
           "flint_attn_exp2_poly")
    return y


def selftest_wait(wait_cycles: int, arrive_first: bool, stream=None):
    """Bounded-wait self-test on the device: (flint_attn_check_status code, completed).

    A wait that nothing completes must give FLINT_ERR_TIMEOUT and completed = False.
    """
    lib = load_library()
    status = torch.zeros(64, dtype=torch.int32, device="cuda")
    st = _stream_ptr(stream)
    _check(lib.flint_attn_selftest_wait(int(wait_cycles), 1 if arrive_first else 0,
                                        _ptr(status), st), "flint_attn_selftest_wait")
    code = lib.flint_attn_check_status(_ptr(status), st)      # synchronises the stream
    return code, bool(status[1].item())


def version() -> str:
    return load_library().flint_attn_version().decode()
