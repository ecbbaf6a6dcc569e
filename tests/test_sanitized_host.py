"""The library's host code under AddressSanitizer and UBSan (CPU only, no
device work): every source is compiled with the sanitizers on its host side
into a temporary library; the C consumer program and the ABI tests
(configuration checks, argument refusals, null contexts, layout, workspace
size, schedule, plateau, gradient buckets) run against it, and any sanitizer
report fails.  The in-tree build is not touched."""
import glob
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
SAN = "-fsanitize=address,-fsanitize=undefined,-fno-omit-frame-pointer"
ASAN_OPTIONS = "protect_shadow_gap=0:detect_leaks=0:verify_asan_link_order=0"


def _runtime(name):
    out = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True,
                         text=True).stdout.strip()
    return out if os.path.isabs(out) and os.path.exists(out) else None


def _clean(text):
    return "AddressSanitizer" not in text and "runtime error" not in text


@pytest.fixture(scope="module")
def sanlib(tmp_path_factory):
    if not (shutil.which("gcc") and os.path.exists(NVCC)):
        pytest.skip("gcc or nvcc not available")
    d = tmp_path_factory.mktemp("llm_san")
    procs = []
    for src in sorted(glob.glob(os.path.join(ROOT, "scratch_llama_decoder_b200", "csrc", "*.cu"))):
        obj = str(d / (os.path.basename(src)[:-3] + ".o"))
        procs.append((obj, subprocess.Popen(
            [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O1", "-std=c++17",
             "-Xcompiler", "-fPIC," + SAN, "--expt-relaxed-constexpr",
             "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj],
            stdout=subprocess.PIPE, stderr=subprocess.STDOUT)))
    for obj, p in procs:
        out = p.communicate(timeout=900)[0]
        assert p.returncode == 0, out.decode()[-2000:]
    lib = str(d / "libllm.so")
    subprocess.run([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-Xcompiler", "-fsanitize=address,-fsanitize=undefined", "-o", lib] +
                   [o for o, _ in procs] + ["-lcudart"], check=True)
    return d, lib


def test_c_consumer_under_sanitizers(sanlib):
    d, lib = sanlib
    exe = str(d / "host_calls")
    subprocess.run(["gcc", "-std=c11", "-g", "-fsanitize=address,undefined", "-o", exe,
                    os.path.join(ROOT, "tests", "c_abi", "host_calls.c"),
                    "-I", os.path.join(ROOT, "include"), "-L", str(d), "-lllm",
                    "-Wl,-rpath," + str(d)], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120,
                       env=dict(os.environ, ASAN_OPTIONS=ASAN_OPTIONS))
    assert r.returncode == 0 and _clean(r.stdout + r.stderr), r.stderr[-3000:]
    assert any(ln.startswith("bucket") for ln in r.stdout.splitlines())


def test_abi_tests_under_sanitizers(sanlib):
    _, lib = sanlib
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("sanitizer runtimes not available")
    env = dict(os.environ, LLM_LIB=lib, LD_PRELOAD=f"{asan}:{ubsan}", ASAN_OPTIONS=ASAN_OPTIONS)
    who = subprocess.run([sys.executable, "-c",
                          "import scratch_llama_decoder_b200 as P; print(P._lib.LIB_PATH)"],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert who.returncode == 0 and who.stdout.strip() == lib, who.stdout + who.stderr
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_abi.py"),
                        os.path.join(ROOT, "tests", "test_lr_schedule_abi.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0 and _clean(r.stdout + r.stderr), tail
