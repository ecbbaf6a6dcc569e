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
