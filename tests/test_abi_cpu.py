"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments before any CUDA call (these run without a GPU)."""
import ctypes
import os
import re

import pytest

from sink_aware_sliding_head_b200 import build as build_mod
from sink_aware_sliding_head_b200 import flint_attn as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return fa.load_library()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "flint_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(flint_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(fa.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n
    out = os.popen(f"nm -D --defined-only {fa.LIB_PATH}").read()
    for n in names:
        assert re.search(rf"\bT {n}\b", out), n


def test_version_and_status_strings(lib):
    assert "sm_100a" in fa.version()
    for code in range(6):
        assert lib.flint_status_string(code)


def params(**kw):
    d = dict(total_tokens=256, num_docs=1, num_q_heads=32, num_kv_heads=4, window=0,
             use_rope=False, rope_theta=1e6, dtype=fa.FLINT_BF16)
    d.update(kw)
    return fa.make_params(**d)


def test_workspace_bytes(lib):
    n_fwd = fa.workspace_bytes(params(), False)
    n_bwd = fa.workspace_bytes(params(), True)
    # q_hat + k_hat at least, backward adds fp32 gradient accumulators
    assert n_fwd >= 256 * (32 + 4) * 128 * 2
    assert n_bwd >= n_fwd + 256 * (32 + 4) * 128 * 4
    assert fa.workspace_bytes(params(head_dim=64), False) == 0
    assert fa.workspace_bytes(params(num_q_heads=30), False) == 0


def _fwd(lib, p, ptr=0x1000, ws=0x100000, ws_bytes=1 << 40):
    P = ctypes.c_void_p
    return lib.flint_attn_fwd(ctypes.byref(p), P(ptr), P(ptr), P(ptr), P(ptr), P(ptr), P(ptr),
                              P(ptr), P(ptr), P(ptr), P(ws), ws_bytes, None)


def test_argument_errors_return_before_any_launch(lib):
    assert _fwd(lib, params(head_dim=64)) == 2              # FLINT_ERR_UNSUPPORTED
    assert _fwd(lib, params(num_q_heads=12, num_kv_heads=1)) == 2   # G = 12
    assert _fwd(lib, params(num_q_heads=30)) == 1           # H % Hk != 0
    assert _fwd(lib, params(num_docs=0)) == 1
    assert _fwd(lib, params(total_tokens=-1)) == 1
    assert _fwd(lib, params(use_rope=True, rope_theta=0.0)) == 1
    assert _fwd(lib, params(dtype=7)) == 1
    assert _fwd(lib, params(), ptr=0) == 1                  # null pointers
    assert _fwd(lib, params(), ptr=0x1008) == 1             # not 16-byte aligned
    assert _fwd(lib, params(), ws=0x100010) == 1            # workspace not 256-byte aligned
    assert _fwd(lib, params(), ws_bytes=16) == 3            # FLINT_ERR_WORKSPACE
    assert lib.flint_attn_fwd(None, *([None] * 9), None, 0, None) == 1


def test_fp32_any_group_size_is_accepted_by_validation(lib):
    # FP32 inputs take any H/Hk (group sizes other than 1, 2, 4, 8, 16 run on CUDA
    # cores); only workspace sizing is checked here
    assert fa.workspace_bytes(params(num_q_heads=12, num_kv_heads=1, dtype=fa.FLINT_FP32),
                              False) > 0


def test_decode_validation(lib):
    """flint_attn_decode's workspace size and argument errors, without a GPU."""
    ok = fa.decode_params(64, 8192, 32, 4, 4096, True, 1e6)
    n = lib.flint_attn_decode_workspace_bytes(ctypes.byref(ok))
    # status, split counters and per-split partials (4 splits of 1024 keys for W = 4096)
    assert n >= 64 * 32 * (128 + 2) * 4 * 4 and n % 256 == 0
    bad = [fa.decode_params(64, 8192, 32, 4, 4096, True, 1e6, head_dim=64),   # D != 128
           fa.decode_params(4, 64, 34, 1, 0, False, 1e4),                       # G = 34
           fa.decode_params(4, 64, 32, 5, 0, False, 1e4),                       # H % Hk
           fa.decode_params(0, 64, 32, 4, 0, False, 1e4)]                       # B = 0
    for p in bad:
        assert lib.flint_attn_decode_workspace_bytes(ctypes.byref(p)) == 0
    p32 = fa.decode_params(4, 64, 32, 4, 0, False, 1e4)
    p32.dtype = fa.FLINT_FP32
    assert lib.flint_attn_decode_workspace_bytes(ctypes.byref(p32)) == 0
    nul = ctypes.c_void_p(0)
    code = lib.flint_attn_decode(ctypes.byref(p32), *([nul] * 11), nul, 0, nul)
    assert code == 2                                     # FLINT_ERR_UNSUPPORTED
    code = lib.flint_attn_decode(ctypes.byref(ok), *([nul] * 11), nul, 0, nul)
    assert code == 1                                     # null pointers, before any launch


def test_header_is_c99_and_links(lib, tmp_path):
    """A C99 program that includes the public header and links the library."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(fa.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_check.c"), "-o", str(exe),
                    "-L", libdir, "-lflint_attn", f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "c abi ok" in r.stdout


def test_compute_f16_validation(lib):
    """The fp16 attention boundary is for FP32 inputs and the tensor-core group sizes."""
    assert fa.workspace_bytes(params(compute_f16=True), False) == 0          # BF16 inputs
    assert fa.workspace_bytes(params(dtype=fa.FLINT_FP32, compute_f16=True, num_q_heads=12,
                                     num_kv_heads=1), False) == 0            # G = 12
    split = fa.workspace_bytes(params(dtype=fa.FLINT_FP32), True)
    f16 = fa.workspace_bytes(params(dtype=fa.FLINT_FP32, compute_f16=True), True)
    # the split path keeps a lo part next to each fp16 copy of dO and v
    assert split >= f16 + 256 * (32 + 4) * 128 * 2


def test_selftest_wait_validation(lib):
    """flint_attn_selftest_wait rejects bad arguments before any launch."""
    P = ctypes.c_void_p
    f = lib.flint_attn_selftest_wait
    assert f(1000, 0, P(0), None) == 1                   # null status
    assert f(1000, 0, P(0x100010), None) == 1            # not 256-byte aligned
    assert f(0, 0, P(0x100000), None) == 1               # limit below 1 cycle
    assert f(4_000_000_001, 0, P(0x100000), None) == 1   # above the kernels' own limit


def test_empty_batch_accepts_null_token_tensors(lib):
    """With T = 0 the [T, ...] tensors may be null; validation passes them and stops
    at the workspace size check (which comes before any CUDA call). With T > 0 the
    same null pointers are an argument error."""
    P = ctypes.c_void_p
    w, ws = P(0x1000), P(0x100000)
    for T, want in ((0, 3), (256, 1)):
        p = params(total_tokens=T, num_docs=2)
        assert lib.flint_attn_fwd(ctypes.byref(p), None, None, None, w, w, w, w, None, None,
                                  ws, 16, None) == want
        assert lib.flint_attn_bwd(ctypes.byref(p), None, None, None, w, w, w, w, None, None,
                                  None, None, None, None, w, w, w, ws, 16, None) == want
    p = params(total_tokens=0, num_docs=2)
    # the parameter-sized tensors stay required
    assert lib.flint_attn_fwd(ctypes.byref(p), None, None, None, None, w, w, w, None, None,
                              ws, 16, None) == 1
    assert lib.flint_attn_bwd(ctypes.byref(p), None, None, None, w, w, w, w, None, None,
                              None, None, None, None, w, w, None, ws, 16, None) == 1


def test_per_device_setup_flags(tmp_path):
    """The launchers' per-device set-up flags (device_once.h), compiled and run on
    the CPU: one set-up per device, independent devices, retry after a failure,
    no caching outside the table, one set-up under concurrent first calls."""
    import shutil
    import subprocess
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no C++ compiler")
    exe = tmp_path / "device_once_check"
    subprocess.run([gxx, "-std=c++17", "-O1", "-Wall", "-Werror", "-pthread",
                    "-I", os.path.join(ROOT, "sink_aware_sliding_head_b200", "csrc"),
                    os.path.join(ROOT, "tests", "c", "device_once_check.cpp"), "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "device once ok" in r.stdout


def test_static_preprocess_validation(lib):
    """flint_attn_bwd_preprocess_static's argument rules, checked before any launch."""
    P = ctypes.c_void_p
    f = lib.flint_attn_bwd_preprocess_static
    w = P(0x1000)

    def call(p, tok=w):
        return f(ctypes.byref(p), tok, tok, tok, w, tok, w, None)

    assert call(params(compute_f16=True)) == 1                    # fp16 boundary needs FP32
    assert call(params(num_q_heads=256, num_kv_heads=4)) == 3     # above the static limit
    assert call(params(head_dim=64)) == 2
    assert call(params(), tok=P(0)) == 1                          # null token tensors, T > 0
    assert call(params(), tok=P(0x1008)) == 1                     # misaligned
    # T = 0: null token tensors pass validation (the call then needs a device)
    assert call(params(total_tokens=0), tok=P(0)) in (0, 4)
    assert f(ctypes.byref(params()), w, w, w, P(0), w, w, None) == 1   # null sink
