"""GPU parity of flint_attn_decode (one new token per sequence over a KV cache)
against the FP64 decode oracle, through the C ABI.

The bar is the BF16 one (max-abs 2e-2, relative RMS 1e-2) on out (float32
output) and LSE. The cache append is checked exactly: the new value row
bit-for-bit, the new key row to within one bf16 ulp (the GPU rounds its fp32
k_hat, the oracle its fp64 one), and every other slot unchanged.
"""
import dataclasses

import numpy as np
import pytest
import torch

import flint_inputs as fi
from oracle import flint_oracle as fo
from parity_util import compare, f64, to_dev

pytestmark = pytest.mark.gpu


def bf16_store(x):
    return torch.as_tensor(np.asarray(x), dtype=torch.float64).to(torch.bfloat16).double().numpy()


def workload(H, Hk, C, W, rope, B):
    return dataclasses.replace(fi.DECODE_SLIDING_BF16, name="decode_case", batch=B,
                               cache_capacity=C, num_q_heads=H, num_kv_heads=Hk, window=W,
                               use_rope=rope, lens_range=(0, C - 1))


def run_gpu(cuda_lib, w, cpu, fp32_out=True, check=True):
    d = to_dev(cpu)
    kc, vc = d["k_cache"].clone(), d["v_cache"].clone()
    out, lse = cuda_lib.decode(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"],
                               d["cache_lens"], kc, vc, w.window, w.use_rope, w.rope_theta,
                               check_status=check, fp32_out=fp32_out)
    torch.cuda.synchronize()
    return out, lse, kc, vc


def run_oracle(w, cpu, rows=None):
    sel = slice(None) if rows is None else rows
    return fo.decode(cpu["q"][sel], cpu["k"][sel], cpu["v"][sel], cpu["w_q"], cpu["w_k"],
                     cpu["sink"], cpu["cache_lens"][sel], cpu["k_cache"][sel],
                     cpu["v_cache"][sel], w.window, w.use_rope, w.rope_theta, store=bf16_store)


def check_cache(cpu, kc, vc, KC, rows):
    lens = cpu["cache_lens"].tolist()
    for i, b in enumerate(rows):
        p = lens[b]
        g_k = f64(kc[b])
        g_v = f64(vc[b])
        ref_k = KC[i][:, p, :]
        assert np.all(np.abs(g_k[:, p, :] - ref_k) <= 2.0 ** -7 * np.abs(ref_k) + 1e-30), b
        assert np.array_equal(g_v[:, p, :], f64(cpu["v"][b])), b
        keep = np.ones(g_k.shape[1], bool)
        keep[p] = False
        assert np.array_equal(g_k[:, keep], f64(cpu["k_cache"][b])[:, keep]), b
        assert np.array_equal(g_v[:, keep], f64(cpu["v_cache"][b])[:, keep]), b


@pytest.mark.parametrize("H,Hk,C,W,rope,lens", [
    (32, 4, 600, 0, False, [0, 1, 17, 300, 599]),
    (32, 4, 600, 128, True, [0, 127, 128, 511, 599]),
    (32, 4, 600, 1, True, [0, 5, 599]),
    (32, 2, 300, 64, True, [5, 299, 150]),          # G = 16
    (4, 4, 200, 0, True, [0, 199, 77]),             # G = 1
    (8, 4, 300, 0, True, [0, 299, 100]),            # G = 2
    (16, 4, 400, 200, False, [399, 250, 0]),        # G = 4
    (6, 2, 250, 0, True, [249, 3, 130]),            # G = 3 (rows past G padded)
    (18, 2, 260, 100, True, [259, 40]),             # G = 9: heads on all 16 rows
    (32, 4, 1100, 1000, False, [1099, 513, 1024]),  # windows spanning several splits
])
def test_decode_matches_oracle(cuda_lib, H, Hk, C, W, rope, lens):
    w = workload(H, Hk, C, W, rope, len(lens))
    cpu = fi.make_decode_inputs(w, seed=7, lens=lens)
    out, lse, kc, vc = run_gpu(cuda_lib, w, cpu)
    O, L, KC, _ = run_oracle(w, cpu)
    compare(out, O, "bf16", "out")
    compare(lse, L, "bf16", "lse")
    check_cache(cpu, kc, vc, KC, list(range(len(lens))))


def test_decode_bf16_output(cuda_lib):
    w = workload(32, 4, 700, 256, True, 4)
    cpu = fi.make_decode_inputs(w, seed=3, lens=[0, 255, 400, 699])
    out, lse, _, _ = run_gpu(cuda_lib, w, cpu, fp32_out=False)
    assert out.dtype == torch.bfloat16
    O, L, _, _ = run_oracle(w, cpu)
    compare(out, O, "bf16", "out", out_bf16=True)
    compare(lse, L, "bf16", "lse")


def test_decode_full_size_sampled(cuda_lib):
    """The serving shape (64 sequences, 8192-slot caches, W = 4096): all outputs on
    the GPU, sampled sequences against the oracle (each depends only on its own
    cache)."""
    w = fi.DECODE_SLIDING_BF16
    cpu = fi.make_decode_inputs(w)
    out, lse, kc, vc = run_gpu(cuda_lib, w, cpu)
    rows = [0, 17, 40, 63]
    O, L, KC, _ = run_oracle(w, cpu, rows)
    compare(out[rows], O, "bf16", "out")
    compare(lse[rows], L, "bf16", "lse")
    check_cache(cpu, kc, vc, KC, rows)


def test_decode_out_of_range_slot_is_reported_and_skipped(cuda_lib):
    w = workload(32, 4, 64, 0, True, 3)
    cpu = fi.make_decode_inputs(w, seed=1, lens=[10, 64, 63])     # 64 is past the cache
    d = to_dev(cpu)
    kc, vc = d["k_cache"].clone(), d["v_cache"].clone()
    out = torch.full((3, 32, 128), 7.0, device="cuda")
    lse = torch.full((3, 32), 7.0, device="cuda")
    with pytest.raises(cuda_lib.FlintError) as e:
        cuda_lib.decode(d["q"], d["k"], d["v"], d["w_q"], d["w_k"], d["sink"], d["cache_lens"],
                        kc, vc, w.window, w.use_rope, w.rope_theta, out=out, lse=lse,
                        check_status=True, fp32_out=True)
    assert e.value.code == 1                                        # FLINT_ERR_INVALID_ARG
    assert torch.all(out[1] == 7.0) and torch.all(lse[1] == 7.0)
    assert torch.equal(kc[1], d["k_cache"][1]) and torch.equal(vc[1], d["v_cache"][1])
    good = [0, 2]
    O, L, KC, _ = run_oracle(w, cpu, good)
    compare(out[good], O, "bf16", "out")
    compare(lse[good], L, "bf16", "lse")
    check_cache(cpu, kc, vc, KC, good)


def test_decode_deterministic(cuda_lib):
    w = workload(32, 4, 900, 0, True, 3)
    cpu = fi.make_decode_inputs(w, seed=9, lens=[899, 450, 3])
    a = run_gpu(cuda_lib, w, cpu)
    b = run_gpu(cuda_lib, w, cpu)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
