"""Builds a host emulator of CUDA kernel source for the CPU tests (see tests/emu/)."""
import os
import shutil
import subprocess

import pytest

EMU = os.path.join(os.path.dirname(os.path.abspath(__file__)), "emu")
FLAGS = ["-std=c++20", "-O1", "-g", "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined"]


def build_emulator(d, kernel_header: str, main_cpp: str) -> str:
    """Writes kernel_header as kernel_emu.h next to the emulation headers and main_cpp (a file
    of tests/emu/) in directory d, and compiles them with AddressSanitizer and UBSan.

    Skips the test when the host has no C++ compiler or no sanitizer runtime; fails it when
    the kernel source does not build."""
    d = str(d)
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no host C++ compiler")
    probe = os.path.join(d, "probe.cpp")
    with open(probe, "w") as f:
        f.write("int main() { return 0; }\n")
    if subprocess.run([gxx, *FLAGS, "-o", os.path.join(d, "probe"), probe], capture_output=True).returncode != 0:
        pytest.skip("the host compiler has no AddressSanitizer / UBSan runtime")
    with open(os.path.join(d, "kernel_emu.h"), "w") as f:
        f.write(kernel_header)
    for name in ("cuda_emu.h", "common_emu.h", main_cpp):
        shutil.copy(os.path.join(EMU, name), d)
    exe = os.path.join(d, "emu")
    r = subprocess.run([gxx, *FLAGS, "-I", d, "-o", exe, os.path.join(d, main_cpp), "-lpthread"],
                       capture_output=True, text=True)
    if r.returncode != 0:
        pytest.fail("host emulation does not build: " + r.stderr[-3000:])
    return exe
