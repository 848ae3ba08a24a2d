"""Seeded synthetic inputs for Flint's sink-aware attention.

This module only draws random numbers and describes workload shapes. It holds
none of the attention arithmetic, so both the FP64 oracle (``oracle/``) and the
CUDA library's harness (``tests/``, ``bench.py``) can use it without sharing any
of the method's code.

Shapes follow the Flint config page (nemo_automodel.components.models.flint.config,
``FlintConfig``): head_dim 128, 32 query heads over 4 KV heads, rms_norm_eps 1e-6.
Documents are packed THD-style: ``cu_doc_lens`` is int32 [documents + 1], the
format the attention utils page (nemo_automodel.components.attention.utils,
``preprocess_args_and_kwargs_for_attn``) gives for ``cu_seqlens``.

Draw order is fixed: document lengths, q, k, v, w_q, w_k, sink, dO. Every draw
is FP32 from one CPU ``torch.Generator``; tensors are then cast to the workload
dtype. The oracle reads the cast values as FP64, so both sides see the same
numbers.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic Flint attention layer.

    ``window`` > 0 counts visible keys including the current token; ``window``
    <= 0 means an unbounded (full causal) window.
    """

    name: str
    doc_lens: Optional[tuple]          # fixed lengths, or None for drawn lengths
    total_tokens: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    window: int
    use_rope: bool
    rope_theta: float
    dtype: str                         # "fp32" or "bf16"
    sink_std: float = 1.0
    backward: bool = True
    drawn_len_range: Optional[tuple] = None   # (lo, hi) inclusive, for drawn lengths
    rms_eps: float = 1e-6
    seed: int = 0
    valid_range: Optional[tuple] = None       # (lo, hi): real tokens per document, rest padding


# The five synthetic Flint layers the library is measured and checked on.
TINY_SLIDING_FP32 = Workload(
    name="tiny_sliding_fp32_S256_H8x1_W64", doc_lens=(256,), total_tokens=256,
    num_q_heads=8, num_kv_heads=1, head_dim=128, window=64, use_rope=True,
    rope_theta=1e4, dtype="fp32")
SLIDING_BF16 = Workload(
    name="sliding_bf16_2x4096_H32x4_W512", doc_lens=(4096, 4096), total_tokens=8192,
    num_q_heads=32, num_kv_heads=4, head_dim=128, window=512, use_rope=True,
    rope_theta=1e6, dtype="bf16", backward=False)
FULL_BF16 = Workload(
    name="full_bf16_S32768_H32x4", doc_lens=(32768,), total_tokens=32768,
    num_q_heads=32, num_kv_heads=4, head_dim=128, window=0, use_rope=False,
    rope_theta=1e6, dtype="bf16", sink_std=2.0, backward=False)
PACKED_BF16 = Workload(
    name="packed_thd_bf16_T65536_H32x4_W1024", doc_lens=None, total_tokens=65536,
    num_q_heads=32, num_kv_heads=4, head_dim=128, window=1024, use_rope=True,
    rope_theta=1e6, dtype="bf16", drawn_len_range=(128, 8192))
LONG_FULL_BF16 = Workload(
    name="long_full_bf16_S131072_H32x4", doc_lens=(131072,), total_tokens=131072,
    num_q_heads=32, num_kv_heads=4, head_dim=128, window=0, use_rope=False,
    rope_theta=1e6, dtype="bf16")

# BSHD with trailing padding (the attention utils page's attention_mask, trailing
# as TE takes it): 8 sequences of 8192 slots, 4096-8192 real tokens each, on the
# sliding-layer shape of the packed workload.
BSHD_PADDED_BF16 = Workload(
    name="bshd_padded_bf16_B8_S8192_H32x4_W1024", doc_lens=(8192,) * 8, total_tokens=65536,
    num_q_heads=32, num_kv_heads=4, head_dim=128, window=1024, use_rope=True,
    rope_theta=1e6, dtype="bf16", valid_range=(4096, 8192))

# The full-causal layer with FP32 inputs (FP32 attention_compute_dtype, the Flint
# config page's default): the split tensor-core path at the headline layer's size.
FULL_FP32 = Workload(
    name="full_fp32_S32768_H32x4", doc_lens=(32768,), total_tokens=32768,
    num_q_heads=32, num_kv_heads=4, head_dim=128, window=0, use_rope=False,
    rope_theta=1e6, dtype="fp32", sink_std=2.0)

WORKLOADS = [TINY_SLIDING_FP32, SLIDING_BF16, FULL_BF16, PACKED_BF16, LONG_FULL_BF16,
             BSHD_PADDED_BF16, FULL_FP32]


def draw_doc_lens(w: Workload, gen: torch.Generator) -> List[int]:
    """Document lengths: fixed, or drawn uniformly until the total is reached.

    Drawn lengths are integers in [lo, hi]; the last document is truncated so
    the lengths sum to ``w.total_tokens`` exactly.
    """
    if w.doc_lens is not None:
        assert sum(w.doc_lens) == w.total_tokens
        return list(w.doc_lens)
    lo, hi = w.drawn_len_range
    lens: List[int] = []
    total = 0
    while total < w.total_tokens:
        n = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
        n = min(n, w.total_tokens - total)
        lens.append(n)
        total += n
    return lens


def cu_from_lens(lens: List[int]) -> torch.Tensor:
    """int32 [documents + 1] offsets of each document in the packed token axis."""
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def torch_dtype(name: str) -> torch.dtype:
    return {"fp32": torch.float32, "bf16": torch.bfloat16}[name]


def make_inputs(w: Workload, seed: Optional[int] = None, with_grad_out: Optional[bool] = None):
    """Draw one batch for workload ``w`` on the CPU.

    Returns a dict of CPU tensors: ``q`` [T,H,D], ``k``/``v`` [T,Hk,D], ``w_q``/``w_k``
    [D] (all in the workload dtype), ``sink`` [H] FP32, ``cu_doc_lens`` int32
    [N+1], and ``dout`` [T,H,D] when a backward pass is wanted. Padded workloads
    add ``valid_lens`` int32 [N] (drawn last, so the other draws are unchanged).
    """
    seed = w.seed if seed is None else seed
    with_grad_out = w.backward if with_grad_out is None else with_grad_out
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    lens = draw_doc_lens(w, gen)
    T, H, Hk, D = w.total_tokens, w.num_q_heads, w.num_kv_heads, w.head_dim
    dt = torch_dtype(w.dtype)
    out = {"cu_doc_lens": cu_from_lens(lens), "doc_lens": lens}
    out["q"] = torch.randn(T, H, D, generator=gen, dtype=torch.float32).to(dt)
    out["k"] = torch.randn(T, Hk, D, generator=gen, dtype=torch.float32).to(dt)
    out["v"] = torch.randn(T, Hk, D, generator=gen, dtype=torch.float32).to(dt)
    out["w_q"] = (1.0 + 0.1 * torch.randn(D, generator=gen, dtype=torch.float32)).to(dt)
    out["w_k"] = (1.0 + 0.1 * torch.randn(D, generator=gen, dtype=torch.float32)).to(dt)
    out["sink"] = w.sink_std * torch.randn(H, generator=gen, dtype=torch.float32)
    if with_grad_out:
        out["dout"] = torch.randn(T, H, D, generator=gen, dtype=torch.float32).to(dt)
    if w.valid_range is not None:
        lo, hi = w.valid_range
        v = torch.randint(lo, hi + 1, (len(lens),), generator=gen, dtype=torch.int64)
        out["valid_lens"] = torch.minimum(v, torch.tensor(lens)).to(torch.int32)
    return out


def make_custom(doc_lens, num_q_heads, num_kv_heads, head_dim=128, dtype="bf16",
                seed=0, sink_std=1.0, with_grad_out=True, qkv_std=1.0):
    """Draw inputs for arbitrary small shapes (parity sweeps), same draw order."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    lens = list(doc_lens)
    T = sum(lens)
    H, Hk, D = num_q_heads, num_kv_heads, head_dim
    dt = torch_dtype(dtype)
    out = {"cu_doc_lens": cu_from_lens(lens), "doc_lens": lens}
    out["q"] = (qkv_std * torch.randn(T, H, D, generator=gen, dtype=torch.float32)).to(dt)
    out["k"] = (qkv_std * torch.randn(T, Hk, D, generator=gen, dtype=torch.float32)).to(dt)
    out["v"] = torch.randn(T, Hk, D, generator=gen, dtype=torch.float32).to(dt)
    out["w_q"] = (1.0 + 0.1 * torch.randn(D, generator=gen, dtype=torch.float32)).to(dt)
    out["w_k"] = (1.0 + 0.1 * torch.randn(D, generator=gen, dtype=torch.float32)).to(dt)
    out["sink"] = sink_std * torch.randn(H, generator=gen, dtype=torch.float32)
    if with_grad_out:
        out["dout"] = torch.randn(T, H, D, generator=gen, dtype=torch.float32).to(dt)
    return out


# ----------------------------------------------------------------------------
# Decode over a KV cache (one new token per sequence)
# ----------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """B sequences, each with ``cache_lens[b]`` tokens cached and one new token.

    The caches are [B, Hk, C, D] (head-major per sequence). Cached keys are
    drawn as N(0, 1) rows: they stand for normalised keys, whose channels have
    unit mean square before the norm weight.
    """

    name: str
    batch: int
    cache_capacity: int
    num_q_heads: int
    num_kv_heads: int
    window: int
    use_rope: bool
    rope_theta: float
    lens_range: tuple                  # cache_lens drawn uniformly in [lo, hi] inclusive
    head_dim: int = 128
    sink_std: float = 1.0
    seed: int = 0


# Serving shape of a sliding layer: 64 sequences with 4096-8191 cached tokens,
# 4096-token window, 32/4 heads (the decode-step counterpart of the sliding
# configurations above).
DECODE_SLIDING_BF16 = DecodeWorkload(
    name="decode_bf16_B64_C8192_H32x4_W4096", batch=64, cache_capacity=8192,
    num_q_heads=32, num_kv_heads=4, window=4096, use_rope=True, rope_theta=1e6,
    lens_range=(4096, 8191))


def make_decode_inputs(w: DecodeWorkload, seed: Optional[int] = None, lens=None):
    """Draw one decode step: cache_lens, q, k, v (new tokens), w_q, w_k, sink, caches.

    Draw order: cache_lens (unless given), q, k, v, w_q, w_k, sink, k_cache,
    v_cache. All draws are FP32 from one CPU generator, cast to bf16 (sinks
    stay FP32, cache_lens int32).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed if seed is None else seed)
    B, C, H, Hk, D = w.batch, w.cache_capacity, w.num_q_heads, w.num_kv_heads, w.head_dim
    if lens is None:
        lo, hi = w.lens_range
        lens = torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64)
    cache_lens = torch.as_tensor(list(lens), dtype=torch.int32)
    bf = torch.bfloat16
    out = {"cache_lens": cache_lens}
    out["q"] = torch.randn(B, H, D, generator=gen, dtype=torch.float32).to(bf)
    out["k"] = torch.randn(B, Hk, D, generator=gen, dtype=torch.float32).to(bf)
    out["v"] = torch.randn(B, Hk, D, generator=gen, dtype=torch.float32).to(bf)
    out["w_q"] = (1.0 + 0.1 * torch.randn(D, generator=gen, dtype=torch.float32)).to(bf)
    out["w_k"] = (1.0 + 0.1 * torch.randn(D, generator=gen, dtype=torch.float32)).to(bf)
    out["sink"] = w.sink_std * torch.randn(H, generator=gen, dtype=torch.float32)
    out["k_cache"] = torch.randn(B, Hk, C, D, generator=gen, dtype=torch.float32).to(bf)
    out["v_cache"] = torch.randn(B, Hk, C, D, generator=gen, dtype=torch.float32).to(bf)
    return out
