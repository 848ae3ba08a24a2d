"""bench.py's work accounting, pinned on the CPU.

The headline metric counts masked FLOPs: 4·D·H per visible (query, key) pair in
the forward and 10·D·H in the backward (its five products, the recomputed QK^T
included); the decode metric counts the K/V bytes of every visible cache slot
once. Both counts are checked against brute-force counts over the oracle's own
visibility rule, and the pair counts of the measured layers against the closed
form L(L+1)/2 of an unwindowed document.
"""
import pytest

import bench
from oracle import flint_oracle as fo


def brute_pairs(lens, W):
    total = 0
    for L in lens:
        for i in range(L):
            lo, hi = fo.visible_keys(i, 0, W)
            total += hi - lo + 1
    return total


@pytest.mark.parametrize("lens,W", [([1], 0), ([1], 1), ([7, 0, 12], 3), ([50], 50),
                                    ([50], 51), ([64, 33], 1), ([100], 0), ([300, 5], 64),
                                    ([513], -1)])
def test_visible_pairs_equals_brute_force(lens, W):
    assert bench.visible_pairs(lens, W) == brute_pairs(lens, W)


def test_pair_counts_of_the_measured_layers():
    for L in (32768, 131072):
        assert bench.visible_pairs([L], 0) == L * (L + 1) // 2
    assert bench.visible_pairs([32768], 0) == 536_887_296
    assert bench.visible_pairs([4096, 4096], 512) == brute_pairs([4096, 4096], 512)
    assert bench.visible_pairs([256], 64) == brute_pairs([256], 64)


def test_flops_per_pair():
    pairs, fwd, bwd = bench.flops_of([32768], 0, 32)
    assert fwd == 4 * 128 * 32 * pairs
    assert bwd == 10 * 128 * 32 * pairs
    assert fwd + bwd == 30_787_265_101_824          # flops_per_step of the default line


@pytest.mark.parametrize("lens,W", [([0, 1, 4095, 4096, 8191], 4096), ([5, 0], 0), ([10, 3], 1)])
def test_decode_kv_bytes_equals_brute_force(lens, W):
    slots = sum(hi - lo + 1 for lo, hi in (fo.visible_keys(p, 0, W) for p in lens))
    assert bench.decode_kv_bytes(lens, W, 4) == slots * 4 * 128 * 2 * 2


def test_clock_sampler_starts_timing_after_its_first_sample(tmp_path, monkeypatch):
    """The clock sampler's start() returns only once nvidia-smi has written its
    first sample: a slow start-up (driver and NVML initialisation) must not fall
    inside a timed region. A stand-in nvidia-smi that needs 0.4 s before its first
    line checks that, and stop() parses the samples it wrote."""
    import os
    import stat
    import time
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\nsleep 0.4\n"
                    "while true; do\n"
                    "  echo '0, 1500, 1965, 700.5, Active, Not Active, Not Active, Not Active, Active'\n"
                    "  sleep 0.05\n"
                    "done\n")
    fake.chmod(fake.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ.get('PATH', '')}")
    sampler = bench.ClockSampler()
    t0 = time.time()
    sampler.start()
    waited = time.time() - t0
    assert waited >= 0.35, waited
    assert os.path.getsize(sampler.path) > 0
    time.sleep(0.1)
    clocks = sampler.stop()
    assert clocks["sm_mhz"] == 1500.0 and clocks["sm_max_mhz"] == 1965.0
    assert clocks["reasons"] == ["sw_power_cap"] and clocks["samples_under_load"] >= 1


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    """No nvidia-smi on PATH: start() returns at once and stop() reports nothing."""
    monkeypatch.setenv("PATH", str(tmp_path))
    sampler = bench.ClockSampler()
    sampler.start()
    assert sampler.stop() is None
