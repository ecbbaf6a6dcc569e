"""The benchmark's step options (host logic, no GPU): the defaults are the
step as benchmarked (no overrides, no options, the workload's own name, so
the captured GEMM traffic still applies); any option renames the workload,
which withholds that traffic figure; the oracle sample runs with every option
on the tiny workload."""
import bench
from synth import get_config


def test_defaults_are_the_benchmarked_step():
    over, opts, suffix = bench.step_options(bench.parse([]))
    assert over == {} and opts == {} and suffix == ""
    cfg = get_config("c5", **over)
    assert cfg["name"] + suffix == bench.GEMM_TRAFFIC["workload"]


def test_options_rename_the_workload_and_withhold_traffic():
    args = bench.parse(["--clip", "1.0", "--clip-mode", "linf", "--dropout", "0.1",
                        "--rope-scale", "2", "--ctx", "4096", "--batch", "4", "--recompute"])
    over, opts, suffix = bench.step_options(args)
    assert over == {"ctx": 4096, "batch": 4, "recompute": 1}
    assert opts == {"clip": (1.0, "linf"), "dropout": 0.1, "rope_scale": 2.0}
    for part in ("ctx4096", "batch4", "recompute1", "clip-linf1", "dropout0.1", "rope_scale2"):
        assert part in suffix
    for one in (["--dropout", "0.1"], ["--clip", "0.5"], ["--rope-scale", "4"], ["--recompute"]):
        _, _, sfx = bench.step_options(bench.parse(one))
        assert sfx and bench.gemm_traffic(get_config("c5")["name"] + sfx) is None


def test_oracle_sample_runs_with_every_option():
    cfg = get_config("c1")
    opts = bench.step_options(bench.parse(["--clip", "0.01", "--clip-mode", "linf",
                                           "--dropout", "0.2", "--rope-scale", "2"]))[1]
    rate, t, cores, S = bench.oracle_sample_rate(cfg, 8, reps=2, warmup=1, opts=opts)
    assert rate > 0 and S == 8 and cores >= 1


def test_data_parallel_modes_parse():
    assert bench.parse([]).dp == "none"
    for mode in ("allreduce", "overlap", "sharded", "sharded-overlap"):
        assert bench.parse(["--dp", mode]).dp == mode


def test_kernel_rates_skip_empty_classes_and_scale_peaks():
    """A class with no launches in the timed steps (the forward SwiGLU pass once
    the W13 GEMM's epilogue takes it over) is left out; the tensor-core GEMM is
    rated against the sustained bf16 peak, the split-precision float32 GEMM
    against a third of the tf32 rate, the memory-bound passes against HBM."""
    pk = {"hbm_gbs": 6000.0, "bf16_tflops_sustained": 1200.0}
    classes = {"gemm": (20.0, 2.4e13, 100), "swiglu_fwd": (0.0, 1e9, 0),
               "gemm_tf32": (10.0, 1.2e12, 10), "adamw": (3.0, 1.5e10, 2)}
    out = bench.kernel_rates(classes, 2, pk, "test")
    assert "swiglu_fwd" not in out
    g = out["gemm"]
    assert abs(g["ms_per_step"] - 10.0) < 1e-9 and abs(g["achieved"] - 1200.0) < 1e-6
    assert abs(g["frac"] - 1.0) < 1e-9
    t = out["gemm_tf32"]
    assert abs(t["peak"] - 1200.0 * bench.TF32_OF_BF16 / 3) < 1e-6
    a = out["adamw"]
    assert a["unit"] == "GB/s" and abs(a["achieved"] - 5000.0) < 1e-6


def test_gemm_traffic_needs_the_captured_sources():
    """The captured GEMM traffic is reported only for the captured workload and
    while both GEMM sources hash to the recorded values."""
    import hashlib
    import os
    name = bench.GEMM_TRAFFIC["workload"]
    root = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "scratch_llama_decoder_b200", "csrc")
    same = all(hashlib.sha256(open(os.path.join(root, f), "rb").read()).hexdigest() == h
               for f, h in bench.GEMM_TRAFFIC["sha256"].items())
    assert bench.gemm_traffic(name) == (bench.GEMM_TRAFFIC["bytes_per_launch"] if same else None)
    assert bench.gemm_traffic(name + "-other") is None

