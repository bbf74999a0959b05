"""Host-side pieces of bench.py (no GPU): defaults, the clock-log summary and the rule that
the reported DRAM traffic is dropped once the kernel sources differ from the captured ones."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_defaults_are_one_gpu_and_a_few_steps():
    a = bench.parse_args([])
    assert (a.gpus, a.steps, a.warmup, a.config, a.impl, a.split) == (
        1, 3, 3, "wan14b_720p", "ours", "problems")
    assert a.warmup >= 3


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler_over(tmp_path, lines):
    path = tmp_path / "clocks.csv"
    path.write_text("".join(lines))
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.path = str(path)
    cs.proc = _Done()
    cs.f = open(os.devnull, "w")
    return cs.stop()


def test_clock_summary_takes_the_median_under_load_and_the_reasons_seen(tmp_path):
    row = "0, {sm}, 1965, {w}, 0x0, Not Active, Not Active, Not Active, {cap}\n"
    lines = [row.format(sm=1965, w=120.0, cap="Not Active"),      # idle: left out
             row.format(sm=1740, w=998.0, cap="Active"),
             row.format(sm=1762, w=995.0, cap="Active"),
             row.format(sm=1800, w=960.0, cap="Not Active"),
             "garbage line\n"]
    got = _sampler_over(tmp_path, lines)
    assert got == {"sm_mhz": 1762.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                   "samples": 4, "samples_under_load": 3}


def test_clock_summary_reports_slowdowns(tmp_path):
    lines = ["0, 1500, 1965, 900, 0x8, Active, Not Active, Active, Not Active\n"]
    got = _sampler_over(tmp_path, lines)
    assert got["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    fake = tmp_path / "repo"
    shutil.copytree(os.path.join(ROOT, "profiles"), fake / "profiles")
    csrc = fake / "block_sparse_attention_25_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("attn_fwd.cu", "bsa_common.cuh"):
        shutil.copy(os.path.join(ROOT, "block_sparse_attention_25_b200", "csrc", name), csrc / name)
    monkeypatch.setattr(bench, "ROOT", str(fake))
    recorded = bench.measured_traffic(False, False)
    if recorded is None:  # the committed summary predates the current sources
        return
    assert recorded > 0 and bench.measured_traffic(True, False) > 0
    with open(csrc / "attn_fwd.cu", "a") as f:
        f.write("\n// edited\n")
    assert bench.measured_traffic(False, False) is None
    assert bench.measured_traffic(True, False) is None


def test_reference_arm_sizes_its_rows_to_the_budget(monkeypatch):
    """The reference arm draws its inputs once and takes between 16 and --cpu-sample-rows
    rows a step, fewer when the steps would otherwise exceed the oracle budget."""
    calls = []
    real_rows = bench.oracle_rows

    def counting_rows(inp, n_rows, seed=0):
        calls.append(n_rows)
        return real_rows(inp, n_rows, seed)

    drawn = []
    real_inputs = bench.oracle_inputs

    def counting_inputs(wl):
        drawn.append(wl.name)
        return real_inputs(wl)

    monkeypatch.setattr(bench, "oracle_rows", counting_rows)
    monkeypatch.setattr(bench, "oracle_inputs", counting_inputs)
    args = bench.parse_args(["--impl", "reference", "--config", "tiny", "--steps", "3",
                             "--warmup", "3", "--cpu-sample-rows", "40"])
    res = bench.run_reference(args, 1, 0, None)
    assert len(drawn) == 1
    step_rows = calls[2:]                       # after the warm-up and the 8-row probe
    assert calls[:2] == [4, 8] and len(step_rows) == 3
    assert all(r == 40 for r in step_rows)      # tiny rows are cheap: the cap applies
    assert res["value"] > 0 and res["steps"] == 3 and "40 sampled query rows" in res["cpu_baseline"]["sample"]
    # a budget far below one row's cost gives the floor of 16 rows a step
    calls.clear()
    monkeypatch.setattr(bench, "REF_BUDGET_S", 1e-9)
    bench.run_reference(args, 1, 0, None)
    assert calls[2:] == [16, 16, 16]
    # ranks other than 0 do no work
    assert bench.run_reference(args, 2, 1, None) is None
