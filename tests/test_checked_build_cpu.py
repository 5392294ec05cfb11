"""The checked build and the tuning switches, on the host (no kernel runs):
libcskv_check.so exports the same entry points as libcskv.so and says which
build it is; the package loads it under CSKV_CHECK=1 and its host-side
argument checks are the regular build's; CSKV_SPLITS changes the attention's
split count and with it the workspace it asks for."""
import ctypes
import os
import subprocess
import sys

from test_abi_cpu import _declared

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "compressed_sparse_kv_softmax_b200")


def test_checked_library_exports_the_header_and_says_so():
    regular = ctypes.CDLL(os.path.join(PKG, "libcskv.so"))
    checked = ctypes.CDLL(os.path.join(PKG, "libcskv_check.so"))
    for name in _declared():
        assert hasattr(checked, name), f"{name} declared in cskv.h but not exported"
    assert regular.cskv_build_checked() == 0
    assert checked.cskv_build_checked() == 1
    assert checked.cskv_version() == regular.cskv_version()


def _python(code, **env):
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       env=dict(os.environ, **env), timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return r.stdout.strip()


def test_package_loads_the_checked_build_under_CSKV_CHECK():
    code = ("import compressed_sparse_kv_softmax_b200 as C; "
            "print(C.build_checked(), C.LIB_PATH.endswith('libcskv_check.so'))")
    assert _python(code, CSKV_CHECK="1") == "True True"
    assert _python(code, CSKV_CHECK="0") == "False False"


def test_host_checks_are_the_same_in_the_checked_build():
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_abi_cpu.py"), "-m", "not gpu"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, CSKV_CHECK="1"))
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]


def test_splits_override_sets_the_workspace():
    # one decode row over 8,192 entries and the window: the planned split count
    # writes partials (64 heads x (512 + 1) floats per split); with one split the
    # row writes its output directly and needs no workspace; with four, four
    # partials (+ 512 bytes of alignment room)
    code = ("import compressed_sparse_kv_softmax_b200 as C; "
            "print(C.attn_workspace_size(1, 1, 64, 512, 8192, 128))")
    planned = int(_python(code))
    assert planned >= 64 * 513 * 4 * 8
    assert int(_python(code, CSKV_SPLITS="1")) == 0
    assert int(_python(code, CSKV_SPLITS="4")) == 4 * 64 * 513 * 4 + 512
    assert int(_python(code, CSKV_SPLITS="junk")) == planned
