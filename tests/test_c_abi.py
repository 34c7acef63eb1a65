"""The C ABI from plain C and from C++, without Python in between: the header
compiles as C99 and as C++17, a program links against the in-tree library,
and its host-side checks (tests/c/abi_host.c) give the documented statuses.
CPU only: no call in the program reaches the device."""

import os
import shutil
import subprocess

import pytest

from newton_schulz_msign_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "abi_host.c")
INCLUDE = os.path.join(ROOT, "include")


@pytest.mark.parametrize("compiler,flags", [("gcc", ["-std=c99", "-pedantic"]), ("g++", ["-x", "c++", "-std=c++17"])])
def test_c_program_links_and_checks(tmp_path, compiler, flags):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    lib = build.build()
    libdir = os.path.dirname(lib)
    exe = str(tmp_path / "abi_host")
    subprocess.run([compiler, *flags, "-Wall", "-Wextra", "-Werror", "-I", INCLUDE, SRC, "-x", "none",
                    "-L", libdir, "-lmsign_b200", f"-Wl,-rpath,{libdir}", "-o", exe], check=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    assert run.stdout.strip() == "ok"
