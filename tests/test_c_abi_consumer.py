"""The C ABI from plain C (gcc, no Python in the loop): a program linked
against libllm.so calls the host-only entry points, and its output agrees with
the float64 oracle (layout, parameter count, schedule, plateau rule) and with
the gradient buckets' definition.  No GPU is used."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle as O
from oracle import train_terms as TT
from synth import get_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "scratch_llama_decoder_b200")


@pytest.fixture(scope="module")
def output(tmp_path_factory):
    if not shutil.which("gcc"):
        pytest.skip("gcc not available")
    exe = str(tmp_path_factory.mktemp("c_abi") / "host_calls")
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-o", exe,
                    os.path.join(ROOT, "tests", "c_abi", "host_calls.c"),
                    "-I", os.path.join(ROOT, "include"), "-L", LIBDIR, "-lllm",
                    "-Wl,-rpath," + LIBDIR], check=True)
    r = subprocess.run([exe], check=True, capture_output=True, text=True, timeout=60)
    return [ln.split() for ln in r.stdout.splitlines()]


def _cfg():
    return get_config("c1", vocab=27, d_model=16, n_layer=2, n_head=4, n_kv_head=2, d_ff=42,
                      ctx=16, batch=2)


def test_layout_and_count_match_the_oracle(output):
    cfg = _cfg()
    rows = [r for r in output if r[0] == "tensor"]
    want = O.param_layout(cfg)
    assert [(r[1], int(r[2]), int(r[3]), int(r[4])) for r in rows] == \
        [(nm, off, rr, cc) for nm, off, rr, cc in want]
    assert int(next(r for r in output if r[0] == "params")[1]) == O.n_params(cfg)
    assert int(next(r for r in output if r[0] == "workspace")[1]) > 0


def test_schedule_and_plateau_match_the_oracle(output):
    f32 = lambda x: float(np.float32(x))
    for _, t, lr in (r for r in output if r[0] == "lr"):
        want = TT.lr_at(int(t), f32(3e-4), f32(3e-5), 10, 10, 110)
        assert float(lr) == pytest.approx(want, rel=1e-6, abs=1e-12), t
    pl = TT.Plateau(0.5, 2, 3, 0.0)
    metric = [3.0, 2.5, 2.6, 2.6, 2.6, 2.4, 2.4, 2.4, 2.4, 2.4]
    got = [float(r[2]) for r in output if r[0] == "plateau"]
    assert got == [pl.update(m) for m in metric]


def test_buckets_and_errors(output):
    cfg = _cfg()
    lay = {nm: (off, rr * cc) for nm, off, rr, cc in O.param_layout(cfg)}
    b = [(int(r[2]), int(r[3])) for r in output if r[0] == "bucket"]
    assert b[0] == (lay["gf"][0], O.n_params(cfg) - lay["gf"][0])
    assert b[1][0] == lay["l1.g1"][0] and b[2][0] == lay["l0.g1"][0]
    assert b[3] == (0, lay["wte"][1])
    assert output[-1] and "token" in " ".join(output[-1]).lower()
