"""The float64 oracle's C library under AddressSanitizer and UBSan: it is
built with -fsanitize=address,undefined into a temporary directory and the
oracle's pin tests run against it in a child process (sanitizer runtimes
preloaded, any report aborts the run).  The in-tree build is not touched."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _runtime(name):
    out = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True,
                         text=True).stdout.strip()
    return out if os.path.isabs(out) and os.path.exists(out) else None


def test_oracle_pins_pass_under_asan_and_ubsan(tmp_path):
    if not shutil.which("gcc"):
        pytest.skip("gcc not available")
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("sanitizer runtimes not available")
    lib = str(tmp_path / "liboracle_sanitized.so")
    subprocess.run(["gcc", "-O1", "-g", "-fopenmp", "-fPIC", "-shared",
                    "-fsanitize=address,undefined", "-fno-sanitize-recover=undefined",
                    "-fno-omit-frame-pointer", "-o", lib,
                    os.path.join(ROOT, "oracle", "llama_oracle.c"), "-lm"], check=True)
    env = dict(os.environ, LLM_ORACLE_LIB=lib, LD_PRELOAD=f"{asan}:{ubsan}",
               ASAN_OPTIONS="detect_leaks=0:verify_asan_link_order=0", OMP_NUM_THREADS="4")
    # the child loads the instrumented build, not the in-tree one
    who = subprocess.run([sys.executable, "-c", "import oracle.oracle as o; print(o._lib._name)"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert who.returncode == 0 and who.stdout.strip() == lib, who.stdout + who.stderr
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py"),
                        os.path.join(ROOT, "tests", "test_oracle_decode.py"),
                        os.path.join(ROOT, "tests", "test_oracle_dropout.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert "ERROR: AddressSanitizer" not in tail and "runtime error" not in tail, tail
