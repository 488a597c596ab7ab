"""The C ABI from plain C: include/svdq.h compiles as strict C99 and C++11,
and tests/c_abi_host.c (built with gcc, linked against the in-tree
libsvdq.so, no Python on its path) prepares a host-only layer, reads its
description and tensors, round-trips a checkpoint and checks the documented
status codes of bad calls.  No GPU work."""
import os
import shutil
import subprocess

import pytest

import w4a4_diffusion_transformer_b200 as lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")


@pytest.fixture(scope="module", autouse=True)
def built():
    from w4a4_diffusion_transformer_b200 import build
    build.build()
    lib.load()


def _compiler(name):
    path = shutil.which(name)
    if path is None:
        pytest.fail(f"{name} is needed to build the C check")
    return path


@pytest.mark.parametrize("std,lang,cc", [("c99", "c", "gcc"), ("c11", "c", "gcc"), ("c++11", "c++", "g++")])
def test_header_is_strict_c_and_cpp(tmp_path, std, lang, cc):
    src = tmp_path / "hdr.c"
    src.write_text('#include "svdq.h"\nint main(void) { return svdq_status_string(SVDQ_OK) == 0; }\n')
    r = subprocess.run([_compiler(cc), f"-std={std}", "-x", lang, "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", INCLUDE, "-c", str(src), "-o", str(tmp_path / "hdr.o")],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr


def test_c_program_against_the_library(tmp_path):
    exe = tmp_path / "c_abi_host"
    libdir = os.path.dirname(lib.LIB_PATH)
    r = subprocess.run([_compiler("gcc"), "-std=c99", "-O1", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                        os.path.join(ROOT, "tests", "c_abi_host.c"), "-o", str(exe), "-L", libdir, "-lsvdq",
                        f"-Wl,-rpath,{libdir}", "-lm"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"
