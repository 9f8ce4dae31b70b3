"""The C ABI boundary on the host: the library loads, exports every function that
include/moe.h declares, and rejects bad arguments before touching a device.

Nothing here launches work: every call is made with arguments that host-side
validation rejects, or is a pure host function (workspace sizing, status text).
The calls pass made-up "device" addresses, so the tests run in a child process
that sees no GPU (CUDA_VISIBLE_DEVICES empty): should host validation ever let
one through, the call fails with a CUDA error instead of reaching a real device.
"""
import ctypes
import os
import re
import subprocess
import sys

import pytest

import mixture_experts_layer_logits_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")
NO_DEVICE = os.environ.get("CUDA_VISIBLE_DEVICES") == ""

# a fake, 16-byte aligned "device" address: validation never dereferences it
A = ctypes.c_void_p(0x7f0000001000)
MIS = ctypes.c_void_p(0x7f0000001004)
NUL = None


@pytest.mark.skipif(NO_DEVICE, reason="this is the child process")
def test_boundary_checks_in_a_process_without_a_device():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        "-m", "not gpu", os.path.abspath(__file__)],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout and " failed" not in r.stdout, r.stdout[-2000:]


@pytest.fixture(scope="module")
def lib():
    if not NO_DEVICE:
        pytest.skip("runs in the child process without a device")
    from mixture_experts_layer_logits_b200 import build

    build.build()
    return moe.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ["moe_workspace_size", "moe_route", "moe_permute", "moe_grouped_ffn",
                 "moe_combine", "moe_forward", "moe_device_status", "moe_status_string",
                 "moe_last_cuda_error"]:
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} is declared in include/moe.h but not exported"


def S(T=8, E=128, k=8, H=2048, I=768):
    return moe.Shape(T, E, k, H, I)


def test_workspace_size(lib):
    assert lib.moe_workspace_size(S()) > 0
    assert lib.moe_workspace_size(S(H=0, I=0)) > 0            # routing-only
    assert lib.moe_workspace_size(S(H=100)) == 0              # not a multiple of 128
    assert lib.moe_workspace_size(S(I=64)) == 0
    assert lib.moe_workspace_size(S(E=0)) == 0
    assert lib.moe_workspace_size(S(E=1025)) == 0
    assert lib.moe_workspace_size(S(k=17, E=64)) == 0
    assert lib.moe_workspace_size(S(k=9, E=8)) == 0           # k > E
    assert lib.moe_workspace_size(S(T=0)) == 0
    # grows with T and is a multiple of 256
    a = lib.moe_workspace_size(S(T=8))
    b = lib.moe_workspace_size(S(T=8192))
    assert b > a and a % 256 == 0 and b % 256 == 0
    # the FFN workspace covers the routing-only one
    assert lib.moe_workspace_size(S()) >= lib.moe_workspace_size(S(H=0, I=0))


def test_route_validation(lib):
    st = None
    assert lib.moe_route(NUL, S(), A, A, st) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_route(A, S(), NUL, A, st) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_route(A, S(E=0), A, A, st) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_route(A, S(E=2000), A, A, st) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_route(A, S(k=0), A, A, st) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_route(A, S(E=4, k=5), A, A, st) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_route(A, S(T=-1), A, A, st) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_route(MIS, S(), A, A, st) == moe.MOE_ERR_MISALIGNED


def test_permute_validation(lib):
    n = lib.moe_workspace_size(S(H=0, I=0))
    assert lib.moe_permute(NUL, S(), A, A, A, n, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(A, S(), A, A, NUL, n, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(A, S(E=0), A, A, A, n, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_permute(A, S(), MIS, A, A, n, None) == moe.MOE_ERR_MISALIGNED
    assert lib.moe_permute(A, S(), A, A, A, n - 1, None) == moe.MOE_ERR_WORKSPACE_TOO_SMALL


def test_grouped_ffn_validation(lib):
    n = lib.moe_workspace_size(S())
    ok = [A, A, A, A, A, S(), A, A, n, None]
    for i in (0, 1, 2, 3, 4, 6, 7):
        args = list(ok)
        args[i] = NUL
        assert lib.moe_grouped_ffn(*args) == moe.MOE_ERR_INVALID_ARG
    for bad in (S(H=200), S(I=100), S(H=0), S(E=0)):
        args = list(ok)
        args[5] = bad
        assert lib.moe_grouped_ffn(*args) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    args = list(ok)
    args[1] = MIS
    assert lib.moe_grouped_ffn(*args) == moe.MOE_ERR_MISALIGNED
    args = list(ok)
    args[8] = n - 256
    assert lib.moe_grouped_ffn(*args) == moe.MOE_ERR_WORKSPACE_TOO_SMALL


def test_combine_validation(lib):
    assert lib.moe_combine(NUL, A, S(), A, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_combine(A, A, S(H=96), A, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_combine(A, A, S(k=0), A, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert lib.moe_combine(A, MIS, S(), A, None) == moe.MOE_ERR_MISALIGNED


def test_forward_validation(lib):
    n = lib.moe_workspace_size(S())
    ok = [A, A, A, A, S(), A, NUL, NUL, NUL, NUL, A, n, None]
    for i in (0, 1, 2, 3, 5, 10):
        args = list(ok)
        args[i] = NUL
        assert lib.moe_forward(*args) == moe.MOE_ERR_INVALID_ARG
    args = list(ok)
    args[4] = S(H=130)
    assert lib.moe_forward(*args) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    for i in (0, 1, 2, 3, 5, 10, 6, 7, 8, 9):       # optional outputs are checked when given
        args = list(ok)
        args[i] = MIS
        assert lib.moe_forward(*args) == moe.MOE_ERR_MISALIGNED
    args = list(ok)
    args[11] = 0
    assert lib.moe_forward(*args) == moe.MOE_ERR_WORKSPACE_TOO_SMALL


def test_forward_w8_validation(lib):
    n = lib.moe_workspace_size(S())
    ok = [A, A, A, A, A, A, S(), A, NUL, NUL, NUL, NUL, A, n, None]
    for i in (0, 1, 2, 3, 4, 5, 7, 12):
        args = list(ok)
        args[i] = NUL
        assert lib.moe_forward_w8(*args) == moe.MOE_ERR_INVALID_ARG
    for i in (0, 1, 2, 3, 4, 5, 7, 12, 8, 9, 10, 11):
        args = list(ok)
        args[i] = MIS
        assert lib.moe_forward_w8(*args) == moe.MOE_ERR_MISALIGNED
    args = list(ok)
    args[6] = S(H=130)
    assert lib.moe_forward_w8(*args) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    args = list(ok)
    args[13] = 0
    assert lib.moe_forward_w8(*args) == moe.MOE_ERR_WORKSPACE_TOO_SMALL
    # FP8 weights run only as the one-launch FFN: T = 65 is refused before any launch
    args = list(ok)
    args[6] = S(T=65)
    args[13] = lib.moe_workspace_size(S(T=65))
    assert lib.moe_forward_w8(*args) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    ev = (ctypes.c_void_p * 5)(*([A] * 5))
    assert lib.moe_forward_w8_timed(*ok, ev, 4) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_w8_timed(*ok, None, 5) == moe.MOE_ERR_INVALID_ARG


def test_forward_w8_supported(lib):
    f = lib.moe_forward_w8_supported
    assert f(S()) == 1                              # decode
    assert f(S(T=64, E=256, H=7168, I=2048)) == 1   # skewed decode
    assert f(S(T=16, E=8, k=2, H=256, I=512)) == 1  # tiny
    assert f(S(T=65)) == 0
    assert f(S(T=8192, H=4096, I=1536)) == 0        # prefill
    assert f(S(H=100)) == 0


def test_device_status_validation(lib):
    assert lib.moe_device_status(NUL, 1024, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_device_status(A, 0, None) == moe.MOE_ERR_WORKSPACE_TOO_SMALL


def test_status_strings(lib):
    seen = set()
    for code in range(8):
        s = lib.moe_status_string(code).decode()
        assert s and s not in seen
        seen.add(s)
    assert lib.moe_status_string(99).decode() == "unknown status"


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "library_path", str(tmp_path / "missing.so"))
    with pytest.raises(OSError):
        moe.load_library()


def test_product_package_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "mixture_experts_layer_logits_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "moe_oracle" not in text and "libmoe_oracle" not in text, f


def test_fused_forward_selection(lib):
    """moe_forward runs FFN + combine as one launch exactly for T <= 64 shapes."""
    if os.environ.get("MOE_DISABLE_FUSED", "0") not in ("", "0"):
        pytest.skip("MOE_DISABLE_FUSED is set")
    assert lib.moe_forward_fused(S()) == 1                              # decode, T = 8
    assert lib.moe_forward_fused(S(T=64, E=256, H=7168, I=2048)) == 1   # skewed decode
    assert lib.moe_forward_fused(S(T=65)) == 0
    assert lib.moe_forward_fused(S(T=8192, H=4096, I=1536)) == 0        # prefill
    assert lib.moe_forward_fused(S(H=100)) == 0                         # unsupported shape
    assert lib.moe_forward_kernel_count(S()) == 1                       # one launch
    assert lib.moe_forward_kernel_count(S(T=65)) >= 4


def test_selftest_wait_timeout_validation(lib):
    f = lib.moe_selftest_wait_timeout
    assert f(NUL, 64, 1000, NUL) == moe.MOE_ERR_INVALID_ARG
    assert f(A, 64, 0, NUL) == moe.MOE_ERR_INVALID_ARG             # limit out of range
    assert f(A, 64, 2000001, NUL) == moe.MOE_ERR_INVALID_ARG
    assert f(MIS, 64, 1000, NUL) == moe.MOE_ERR_MISALIGNED
    assert f(A, 4, 1000, NUL) == moe.MOE_ERR_WORKSPACE_TOO_SMALL   # needs the error word + a flag


def test_permute_noalloc_rejects_sizes_beyond_its_scratch(lib):
    fn = lib.moe_permute_noalloc
    fn.argtypes = [ctypes.c_void_p, moe.Shape, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    k = 8
    T = (1 << 20) // k + 1                       # one row past the scratch's limit
    assert fn(A, moe.Shape(T, 64, k, 0, 0), A, A, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert fn(NUL, moe.Shape(8, 64, k, 0, 0), A, A, None) == moe.MOE_ERR_INVALID_ARG
    assert fn(A, moe.Shape(8, 2000, k, 0, 0), A, A, None) == moe.MOE_ERR_UNSUPPORTED_SHAPE
    assert fn(A, moe.Shape(8, 64, k, 0, 0), MIS, A, None) == moe.MOE_ERR_MISALIGNED
