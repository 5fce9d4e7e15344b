"""Host logic of bench.py that needs no GPU: the reference arm sizes each
timed step's oracle sample from the costs its first warm-up step measures,
so that all timed steps fit the budget, and prints one JSON line with the
contract's keys; the clock record of a timed region is summarised and a
slowdown voids its number."""
import argparse
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _args(steps, warmup=2, groups=16):
    return argparse.Namespace(steps=steps, warmup=warmup, cpu_sample_groups=groups)


def _run(monkeypatch, capsys, steps, t_pre, t_group, groups=16):
    calls = []

    def fake_sample(cfg, inp, g):
        calls.append(g)
        return {"value": 1e-3, "unit": bench.UNIT, "cores": 1, "kind": "oracle", "sample": f"{g} groups",
                "sample_seconds": t_pre + g * t_group, "extrapolated_ms": 1e6,
                "t_pre_s": t_pre, "t_att_per_group_s": t_group}

    monkeypatch.setattr(bench, "cpu_sample", fake_sample)
    monkeypatch.setattr(synth, "make_inputs", lambda cfg, seed=0: None)
    bench.run_reference(_args(steps, groups=groups), synth.CONFIGS["small"], 0, 1)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    return calls, line


def test_reference_step_size_follows_the_budget(monkeypatch, capsys):
    # 50 steps in 120 s leave 2.4 s a step: 2.4 - 1.0 s of prepass = 1.4 s of
    # 0.5 s groups -> 2 groups per timed step
    calls, line = _run(monkeypatch, capsys, steps=50, t_pre=1.0, t_group=0.5)
    assert calls[:2] == [1, 1]                 # the warm-up steps take one group
    assert set(calls[2:]) == {2} and len(calls) == 52
    assert line["impl"] == "reference" and line["steps"] == 50
    for key in ("metric", "value", "unit", "ms_per_step", "cpu_baseline", "e2e", "higher_is_better"):
        assert key in line
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    # the same workload keys as the GPU arm's line, the host named, the step extrapolated
    cfg = synth.CONFIGS["small"]
    assert {k: line["config"][k] for k in "BNHD"} == {"B": cfg.B, "N": cfg.N, "H": cfg.H, "D": cfg.D}
    assert line["extrapolated"] is True and line["cpu_baseline"]["extrapolated"] is True
    assert line["cpu_baseline"]["nproc"] == os.cpu_count() and "cpu_model" in line["cpu_baseline"]


def test_reference_step_size_is_bounded(monkeypatch, capsys):
    # few steps: capped at half of --cpu-sample-groups; a prepass longer than
    # the per-step budget: still one group
    calls, _ = _run(monkeypatch, capsys, steps=2, t_pre=0.1, t_group=0.01, groups=16)
    assert set(calls[2:]) == {8}
    calls, _ = _run(monkeypatch, capsys, steps=50, t_pre=30.0, t_group=1.0)
    assert set(calls[2:]) == {1}


def test_reference_arm_prints_nothing_on_other_ranks(monkeypatch, capsys):
    monkeypatch.setattr(bench, "cpu_sample", lambda *a: pytest.fail("rank 1 must not sample"))
    bench.run_reference(_args(3), synth.CONFIGS["small"], 1, 2)
    assert capsys.readouterr().out == ""


def _smi(mhz, reasons=()):
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    flags = ["Active" if n in reasons else "Not Active" for n in names]
    return f"0, {mhz}, 1965, 900.00, 0x0000000000000000, " + ", ".join(flags) + "\n"


def test_clock_summary_and_rejection():
    # an idle sample before the load is left out of the median; reasons seen anywhere count
    s = bench.summarize_clocks([_smi(345), _smi(1965), _smi(1950), _smi(1965)])
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "samples": 4, "reasons": []}
    assert bench.clocks_rejection(s) is None
    # a power cap alone is kept, even at lower clocks
    s = bench.summarize_clocks([_smi(1310, ["sw_power_cap"])] * 3)
    assert s["reasons"] == ["sw_power_cap"] and bench.clocks_rejection(s) is None
    # any hardware or thermal slowdown voids the number
    s = bench.summarize_clocks([_smi(1965), _smi(1800, ["hw_thermal_slowdown"])])
    assert bench.clocks_rejection(s) == "hw_thermal_slowdown"
    # clocks held low with no reason: a leftover clock lock
    s = bench.summarize_clocks([_smi(1200)] * 5)
    assert bench.clocks_rejection(s) == "sm clock held low with no reason"
    # no samples (sampling off or nvidia-smi missing): nothing to judge
    assert bench.summarize_clocks(["garbage\n"]) is None and bench.clocks_rejection(None) is None


def test_defaults_follow_the_contract(monkeypatch):
    # no flags: one GPU, the long-context workload, at least 3 warm-up steps,
    # every mainloop and workload name accepted
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    a = bench.parse()
    assert (a.gpus, a.config, a.impl, a.mainloop) == (1, "long_fused", "ours", "default")
    assert a.warmup >= 3 and a.steps >= 1
    monkeypatch.setattr(sys, "argv", ["bench.py", "--config", "nonesuch"])
    with pytest.raises(SystemExit):
        bench.parse()
    import synth
    for name in synth.CONFIG_ORDER:
        monkeypatch.setattr(sys, "argv", ["bench.py", "--config", name])
        assert bench.parse().config == name
