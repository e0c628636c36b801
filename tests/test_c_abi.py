"""include/ss2d.h from plain C: the header compiles as C99 with -pedantic and -Werror, a C
program links against libss2d.so, and its host-side answers (version, status strings, the
struct layouts, argument checks and workspace queries) match what the Python binding sees."""
import ctypes
import os
import shutil
import subprocess

import pytest

import selective_scan_02_b200 as ss
from selective_scan_02_b200 import BlockArgs, CoreArgs, CoreGrads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def c_results(tmp_path_factory):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no host C compiler")
    lib = ss.LIB_PATH
    if not os.path.exists(lib):
        pytest.fail("libss2d.so is not built")
    exe = str(tmp_path_factory.mktemp("c_abi") / "c_abi_check")
    cmd = [gcc, "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi", "c_abi_check.c"), "-o", exe, lib,
           "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-3000:]
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-3000:]
    out = {}
    for line in r.stdout.splitlines():
        k, _, v = line.partition(" ")
        out[k] = v
    return out


def test_header_and_library_from_c(c_results):
    lib = ss.load_library()
    assert int(c_results["version"]) == lib.ss2d_version()
    assert c_results["status_ok"] == "SS2D_OK" and c_results["status_device"] == "SS2D_ERR_DEVICE"
    # the ctypes mirrors have the C layout
    assert int(c_results["sizeof_args"]) == ctypes.sizeof(CoreArgs)
    assert int(c_results["sizeof_grads"]) == ctypes.sizeof(CoreGrads)
    assert int(c_results["offset_ckpt"]) == CoreArgs.ckpt.offset
    assert int(c_results["offset_layout"]) == CoreArgs.layout.offset
    assert int(c_results["offset_merge_order"]) == CoreArgs.merge_order.offset
    assert int(c_results["sizeof_block"]) == ctypes.sizeof(BlockArgs)
    assert int(c_results["offset_block_eps"]) == BlockArgs.out_norm_eps.offset
    assert int(c_results["offset_block_out_dtype"]) == BlockArgs.out_dtype.offset


def test_checks_and_queries_from_c(c_results):
    assert int(c_results["bad_n"]) == 2 and "N=5" in c_results["bad_n_msg"]     # SS2D_ERR_UNSUPPORTED
    assert int(c_results["misaligned"]) == 3                                     # SS2D_ERR_MISALIGNED
    assert int(c_results["device_status_direct"]) == 0
    # B1 D16 8x8 bf16: the transposed copy of x (1*16*64 bf16) and no segmentation
    assert int(c_results["fwd_ws"]) == 16 * 64 * 2
    assert int(c_results["bwd_ws"]) not in (0, 2 ** 64 - 1)
