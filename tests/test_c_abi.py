"""include/dmu.h is a plain C header: a C99 program (tests/c/abi_check.c)
compiles against it with -std=c99 -pedantic -Werror, links against
libdmu.so and passes its host-side argument checks. No GPU is needed: every
call in the program returns before any device work."""
import os
import shutil
import subprocess

import pytest

from gram_newton_schulz_b200 import dmu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c99_program_builds_and_passes(tmp_path):
    dmu.load()  # the library must exist (built by __graft_entry__.build())
    libdir = os.path.dirname(dmu.LIB_PATH)
    exe = str(tmp_path / "abi_check")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I" + os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_check.c"),
           "-L" + libdir, "-ldmu", "-Wl,-rpath," + libdir, "-o", exe]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    assert "abi_check ok" in run.stdout
