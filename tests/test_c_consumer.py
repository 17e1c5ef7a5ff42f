"""include/kda.h is a plain C interface: a C99 program and a C++ program that
include it build with warnings as errors, link against the shared library and
run its host-side calls (sizes, version, argument checks; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_consumer", "host_calls.c")


@pytest.fixture(scope="module")
def libdir():
    from gated_delta_rule_108_b200 import build, kda
    build.build()
    path = kda.lib()._name
    return os.path.dirname(os.path.abspath(path)), os.path.basename(path)


@pytest.mark.parametrize("compiler,flags", [
    ("gcc", ["-x", "c", "-std=c99", "-pedantic"]),
    ("g++", ["-x", "c++", "-std=c++17", "-pedantic"]),
])
def test_header_builds_links_and_runs(libdir, tmp_path, compiler, flags):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not available")
    d, name = libdir
    exe = tmp_path / f"host_calls_{compiler.replace('+', 'x')}"
    cmd = [compiler, *flags, "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), SRC,
           "-x", "none", "-L", d, f"-l:{name}", f"-Wl,-rpath,{d}", "-o", str(exe)]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert "host calls ok" in run.stdout
