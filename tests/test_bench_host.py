"""Host logic of bench.py's reference arm (the fp64 oracle timed on the host
cores), on CPU: the JSON line it prints, its token accounting and its rank
handling.  The workload is shrunk so that each test takes seconds."""
import argparse
import json

import pytest

import bench
import rehyat_inputs
from rehyat_inputs import make_problem

TINY = dict(batch=1, heads=3, T=5, Hs=3, Ws=4, D=32, Dp=32, Tc=2, To=1, causal=False,
            dtype="bf16")


@pytest.fixture
def small_workload(monkeypatch):
    orig = rehyat_inputs.config_problem
    monkeypatch.setattr(rehyat_inputs, "config_problem",
                        lambda name, **kw: orig(name, **dict(kw, batch=1, heads=2, T=4, Hs=3,
                                                             Ws=5, Tc=2, To=1)))


def test_reference_line_keys_and_arithmetic(monkeypatch, capsys, small_workload):
    seen = []

    def fake_run(p, plan, start_head=0):
        seen.append(start_head)
        return dict(seconds=0.5, token_equiv=1000.0, sample="stub sample")

    monkeypatch.setattr(bench, "plan_oracle_sample", lambda p, budget: dict(heads=1, chunks=1))
    monkeypatch.setattr(bench, "run_oracle_sample", fake_run)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    assert bench.main(["--impl", "reference", "--steps", "4", "--warmup", "0"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert seen == list(range(7))          # 3 warm-up samples (the minimum), then 4 timed
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["steps"] == 4 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] == pytest.approx(2000.0)              # 4000 tokens in 2 s
    assert line["ms_per_step"] == pytest.approx(500.0)
    assert line["dtype"] == "f64" and line["data"] == "synthetic"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert "stub sample" in cb["sample"]
    assert isinstance(cb["host"], dict) and "cpu" in cb["host"]   # the CPU model is recorded
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["config"]["workload"].startswith(bench.WORKLOAD)


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    def boom(*a, **k):
        raise AssertionError("a non-zero rank ran the oracle")

    monkeypatch.setattr(bench, "plan_oracle_sample", boom)
    monkeypatch.setattr(bench, "run_oracle_sample", boom)
    args = argparse.Namespace(steps=2, warmup=3, gpus=2)
    assert bench.run_reference(args, 2, 1) == 0
    assert capsys.readouterr().out == ""


def test_oracle_sample_accounting_and_head_rotation():
    p = make_problem(seed=5, **TINY)
    BH = p.batch * p.heads
    r = bench.run_oracle_sample(p, dict(heads=2, chunks=2), start_head=BH - 1)
    rows = 2 * p.Tc * p.HW                 # chunks 0 and 1 hold T_c slices each
    assert r["token_equiv"] == pytest.approx(rows * 2 / p.heads)
    assert r["seconds"] > 0
    assert r["sample"].startswith(f"2 of {BH} (batch, head) pairs x chunks 0..1 of 3")
    # The ragged last chunk (one slice) counts its own rows.
    r = bench.run_oracle_sample(p, dict(heads=1, chunks=3))
    assert r["token_equiv"] == pytest.approx(p.T * p.HW / p.heads)


def test_oracle_sample_plan_stays_in_budget():
    p = make_problem(seed=6, **TINY)
    tight = bench.plan_oracle_sample(p, 0.0)
    assert tight["heads"] == 1 and tight["chunks"] >= 1
    roomy = bench.plan_oracle_sample(p, 1e6)
    assert roomy == dict(heads=p.batch * p.heads, chunks=3)


# Independent counts of the method's work per configuration, from the planning
# analysis (computed by a separate script, printed to a few digits):
# (B, h, T, HW, D, D', T_c, T_o, causal) -> total FLOP, softmax FLOP, exps,
# full-softmax FLOP.
WORK = [
    ((1, 2, 4, 16, 32, 32, 2, 1, False), "1.7e6", "0.66e6", "5.1e3", "1.0e6"),      # tiny fp32
    ((1, 12, 21, 600, 128, 128, 3, 1, True), "199e9", "179e9", "0.35e9", "975e9"),  # 21x20x30
    ((2, 12, 21, 1560, 128, 128, 3, 1, False), "2.525e12", "2.422e12", "4.73e9", "13.19e12"),
    ((1, 12, 81, 1560, 128, 128, 3, 1, True), "5.0e12", "4.8e12", "9.4e9", "98e12"),  # stream
]


def _matches(value, printed):
    """value agrees with a number printed as ``printed`` to within one unit
    of its last printed digit."""
    mant, exp = printed.lower().split("e")
    decimals = len(mant.split(".")[1]) if "." in mant else 0
    return abs(value - float(printed)) <= 10.0 ** (int(exp) - decimals)


@pytest.mark.parametrize("cfg,total,soft,exps,full", WORK, ids=["tiny", "320x480", "480x832",
                                                               "stream81"])
def test_algorithmic_work_matches_independent_counts(cfg, total, soft, exps, full):
    """The roofline numerator (bench.algorithmic_work) agrees with counts made
    independently, to the digits those were printed with."""
    B, h, T, HW, D, Dp, Tc, To, causal = cfg
    w = bench.algorithmic_work(*cfg)
    N = T * HW
    phi_q_and_readout = (2.0 * N * D * Dp + 2.0 * N * Dp * D + 2.0 * N * Dp) * B * h
    assert _matches(w["total_flops"], total), (w["total_flops"], total)
    assert _matches(w["attn_flops"] - phi_q_and_readout, soft)
    assert _matches(w["exps"], exps), (w["exps"], exps)
    assert _matches(w["full_softmax_flops"], full)


def _smi_line(t, sm, reasons=("Not Active",) * 4, sm_max=1965):
    stamp = __import__("datetime").datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")
    return ", ".join([stamp[:-3], str(sm), str(sm_max), "812.40", "0x0000000000000000",
                      *reasons])


def test_clock_summary_keeps_the_timed_window_and_its_reasons():
    """The clock record of the bench line: median SM clock, max clock and the
    throttle reasons seen inside the timed window only."""
    cs = bench.ClockSampler.__new__(bench.ClockSampler)   # no nvidia-smi process
    t0 = 1_000_000.0
    cs.lines = [
        _smi_line(t0 - 5.0, 900, ("Active", "Not Active", "Not Active", "Not Active")),  # before
        _smi_line(t0 + 0.1, 1950),
        _smi_line(t0 + 0.2, 1965, ("Not Active", "Not Active", "Not Active", "Active")),
        _smi_line(t0 + 0.3, 1800),
        "garbage, line",
        _smi_line(t0 + 9.0, 700, ("Not Active", "Active", "Not Active", "Not Active")),    # after
    ]
    s = cs.summary(t0, t0 + 0.5)
    assert s == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 3}
    # A hardware slowdown inside the window is reported by name.
    cs.lines.append(_smi_line(t0 + 0.4, 1200, ("Active", "Not Active", "Not Active",
                                               "Not Active")))
    assert cs.summary(t0, t0 + 0.5)["reasons"] == ["hw_slowdown", "sw_power_cap"]
    # No sample inside the window: the last three samples stand in.
    assert cs.summary(t0 + 100, t0 + 101)["samples"] == 3
    cs.lines = []
    assert cs.summary(t0, t0 + 1) is None


def test_traffic_is_reported_only_for_the_captured_source():
    """`roofline.traffic` comes from the committed ncu summary only while the
    kernel source hashes to the value recorded with the capture."""
    import os
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    assert "attn" in d
    for key in d:
        sha = d[key]["source_sha"]
        assert bench.load_traffic(key, sha) == float(d[key]["dram_bytes_per_launch"])
        assert bench.load_traffic(key, "0" * 16) is None
    assert bench.load_traffic("no_such_kernel", d["attn"]["source_sha"]) is None
    assert len(bench.kernel_source_sha(["bench.py"])) == 16
