"""A training step through the C ABI from plain C on the GPU (no Python or
torch in that process): tests/c_abi/step_on_gpu.c allocates with the CUDA
runtime, draws the parameters with llm_init and runs llm_step; its dump of
the parameters before and after, the ids and the loss is checked against the
float64 oracle's step on the same parameters and ids."""
import os
import subprocess

import numpy as np
import pytest

import oracle as O
from synth import get_config
from tests.gpu_util import TOL, rel

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "scratch_llama_decoder_b200")


def _cudart():
    out = subprocess.run(["ldd", os.path.join(LIBDIR, "libllm.so")], check=True,
                         capture_output=True, text=True).stdout
    return next(ln.split()[2] for ln in out.splitlines() if "libcudart" in ln)


def test_c_program_step_matches_oracle(tmp_path):
    exe, dump = str(tmp_path / "step_on_gpu"), str(tmp_path / "step.bin")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-o", exe,
                    os.path.join(ROOT, "tests", "c_abi", "step_on_gpu.c"),
                    "-I", os.path.join(ROOT, "include"), "-I", "/usr/local/cuda/include",
                    "-L", LIBDIR, "-lllm", "-Wl,-rpath," + LIBDIR, _cudart()], check=True)
    r = subprocess.run([exe, dump], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    raw = open(dump, "rb").read()
    n, nt = np.frombuffer(raw[:16], np.int64)
    o = 16
    tok = np.frombuffer(raw[o:o + 4 * nt], np.int32); o += 4 * nt
    tgt = np.frombuffer(raw[o:o + 4 * nt], np.int32); o += 4 * nt
    loss = float(np.frombuffer(raw[o:o + 4], np.float32)[0]); o += 4
    before = np.frombuffer(raw[o:o + 4 * n], np.float32).astype(np.float64); o += 4 * n
    after = np.frombuffer(raw[o:o + 4 * n], np.float32).astype(np.float64)
    cfg = get_config("c1", vocab=27, d_model=16, n_layer=1, n_head=4, n_kv_head=2, d_ff=42,
                     ctx=16, batch=2)
    assert O.n_params(cfg) == n
    lref, _, g = O.forward_backward(cfg, before, tok.reshape(2, 16), tgt.reshape(2, 16),
                                    want_logits=False)
    f32 = lambda x: float(np.float32(x))
    pref, _, _ = O.adamw(before, g, np.zeros(n), np.zeros(n), 1, f32(1e-2), f32(0.1))
    tol = TOL["fp32"]
    assert abs(loss - lref) <= tol["loss"] * abs(lref), (loss, lref)
    assert rel(after - before, pref - before) <= tol["params"]
    assert rel(after, pref) <= tol["params"]
    # llm_init: gains 1, matrices ~ N(0, 0.08)
    lay = {nm: (off, rr * cc) for nm, off, rr, cc in O.param_layout(cfg)}
    off, cnt = lay["l0.g1"]
    assert np.all(before[off:off + cnt] == 1.0)
    off, cnt = lay["wte"]
    assert abs(before[off:off + cnt].std() - 0.08) < 0.02
