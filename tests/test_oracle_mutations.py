"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of ``oracle/flint_oracle.py`` (a dropped
term, a wrong sign or index, a transposed mapping) and runs the pin suite
(``tests/test_oracle_pins.py``) against the copy in a child process: the suite
must fail. An unmodified copy must pass, so a broken harness cannot make every
mutant look caught. Everything runs on the CPU; the real oracle is never
modified.
"""
import concurrent.futures
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, original text, replacement): each original occurs exactly once.
# Not listed, because they are equivalent mutations with unchanged outputs: a
# block's first key column moved one further left (the visibility mask hides
# it), and RoPE positions that run on across documents instead of restarting
# (the logits depend only on position differences within a document).
MUTANTS = [
    ("window_admits_one_extra_key",
     "vis &= (i - j) < window", "vis &= (i - j) <= window"),
    ("block_start_drops_a_visible_key",
     "lo = d0 if window <= 0 else max(d0, a - window + 1)\n            for kv in range(Hk):\n"
     "                hs = list(range(kv * G, (kv + 1) * G))\n"
     "                z = _block_logits(q_hat, k_hat, a, b, lo, window, hs, kv, scale)\n"
     "                p, _, l = ",
     "lo = d0 if window <= 0 else max(d0, a - window + 2)\n            for kv in range(Hk):\n"
     "                hs = list(range(kv * G, (kv + 1) * G))\n"
     "                z = _block_logits(q_hat, k_hat, a, b, lo, window, hs, kv, scale)\n"
     "                p, _, l = "),
    ("row_window_admits_one_extra_key",
     "max(d0, i - window + 1)", "max(d0, i - window)"),
    ("sink_logit_scaled",
     "s = sink_g[:, None]", "s = 0.5 * sink_g[:, None]"),
    ("sink_dropped_from_denominator",
     "Z = es + np.sum(e, axis=-1)", "Z = np.sum(e, axis=-1)"),
    ("softmax_scale_is_one_over_d",
     "    scale = 1.0 / np.sqrt(D) if scale is None else scale\n"
     "    sink = np.asarray(sink, dtype=np.float64)\n    O = ",
     "    scale = 1.0 / D if scale is None else scale\n"
     "    sink = np.asarray(sink, dtype=np.float64)\n    O = "),
    ("rope_rotation_sign",
     "x1 * c - x2 * s, x2 * c + x1 * s", "x1 * c + x2 * s, x2 * c - x1 * s"),
    ("rope_frequency_exponent",
     "float(theta) ** (-2.0 * j / head_dim)", "float(theta) ** (-1.0 * j / head_dim)"),
    ("rmsnorm_sum_instead_of_mean",
     "r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)\n    return",
     "r = 1.0 / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)\n    return"),
    ("rmsnorm_backward_sign",
     "dx = r * u - x * (r ** 3)", "dx = r * u + x * (r ** 3)"),
    ("softmax_backward_drops_D",
     "dz = p * (dp - Di[..., None])", "dz = p * dp"),
    ("dsink_sign",
     "dsink[hs] -= np.sum", "dsink[hs] += np.sum"),
    ("gqa_head_mapping_transposed",
     "return h // (H // Hk)", "return h % Hk"),
    ("padded_rows_lse_zero",
     "lse = np.repeat(sink[:, None], T, axis=1)", "lse = np.zeros((H, T))"),
    ("decode_new_key_not_cached",
     "kc[b, :, p, :] = keep(k_hat)", "kc[b, :, p, :] = 0.0 * keep(k_hat)"),
]


def _run_pins(work, name, mutation):
    """Copy the oracle and the pins to work/name, plant the mutation, run the pins."""
    d = os.path.join(work, name)
    shutil.copytree(os.path.join(ROOT, "oracle"), os.path.join(d, "oracle"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copytree(os.path.join(ROOT, "flint_inputs"), os.path.join(d, "flint_inputs"),
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.makedirs(os.path.join(d, "tests"))
    for f in ("conftest.py", "test_oracle_pins.py"):
        shutil.copy(os.path.join(ROOT, "tests", f), os.path.join(d, "tests", f))
    shutil.copytree(os.path.join(ROOT, "tests", "golden"), os.path.join(d, "tests", "golden"))
    path = os.path.join(d, "oracle", "flint_oracle.py")
    if mutation is not None:
        old, new = mutation
        with open(path) as f:
            src = f.read()
        if src.count(old) != 1:
            return "not applied", ""
        with open(path, "w") as f:
            f.write(src.replace(old, new))
    env = {k: v for k, v in os.environ.items() if k != "PYTHONPATH"}
    env["OMP_NUM_THREADS"] = "2"
    env["OPENBLAS_NUM_THREADS"] = "2"
    env["MKL_NUM_THREADS"] = "2"
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q",
                        "-p", "no:cacheprovider"], cwd=d, env=env, capture_output=True,
                       text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    work = str(tmp_path_factory.mktemp("mutants"))
    jobs = [("control", None)] + [(n, (o, r)) for n, o, r in MUTANTS]
    with concurrent.futures.ThreadPoolExecutor(max_workers=4) as ex:
        futs = {n: ex.submit(_run_pins, work, n, m) for n, m in jobs}
        return {n: f.result() for n, f in futs.items()}


def test_unmodified_copy_passes_the_pins(outcomes):
    rc, log = outcomes["control"]
    assert rc == 0, log


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(outcomes, name):
    rc, log = outcomes[name]
    assert rc != "not applied", f"{name}: the original text is not in the oracle"
    # 1 = tests failed (pytest's exit code); anything else would be a harness error
    assert rc == 1, f"{name}: the pins did not fail (exit {rc})\n{log}"
