"""bench.py host logic that needs no GPU: the clock report covers only the
timed region, and every reason NVML can flag is named."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _sampler_with(samples, begin, end):
    c = bench.ClockSampler("0")
    c.samples = samples
    c.sm_max = 1965.0
    c.source = "test"
    c.t_begin, c.t_end = begin, end
    return c


def test_clock_report_keeps_only_the_timed_region():
    rows = [(0.0, 300.0, 90.0, []), (1.0, 1965.0, 700.0, []), (1.5, 1800.0, 990.0, ["sw_power_cap"]),
            (2.0, 1900.0, 800.0, []), (3.0, 500.0, 100.0, ["hw_slowdown"])]
    r = _sampler_with(rows, 0.9, 2.1).stop()
    assert r["samples"] == 5 and r["samples_in_timed_region"] == 3
    assert r["sm_mhz"] == 1900.0
    assert r["sm_mhz_min_in_timed_region"] == 1800.0
    assert r["reasons"] == ["sw_power_cap"]   # the slowdown after the region is not reported
    assert r["sm_max_mhz"] == 1965.0


def test_clock_report_without_samples():
    r = _sampler_with([], 0.0, 1.0).stop()
    assert r["sm_mhz"] is None and r["samples"] == 0


def test_a_timed_region_shorter_than_the_period_still_holds_a_sample():
    """sample_now(), called while the timed launches run, puts a sample inside
    the region even when the sampling thread never woke up there; a sample
    without a power reading still counts."""
    import time
    c = bench.ClockSampler("0")
    c.sm_max, c.source = 1965.0, "test"
    c._read = lambda: (time.monotonic(), 1950.0, None, [])
    c.samples = [(time.monotonic() - 10.0, 1965.0, 120.0, [])]   # before the region
    c.mark_begin()
    c.sample_now()
    c.mark_end()
    r = c.stop()
    assert r["samples_in_timed_region"] == 1 and r["sm_mhz"] == 1950.0
    assert r["power_w_max"] == 120.0


def test_reason_bits_are_distinct():
    bits = [b for _, b in bench.ClockSampler.REASONS]
    assert len(set(bits)) == len(bits)
    names = {n for n, _ in bench.ClockSampler.REASONS}
    assert {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"} <= names


def test_reference_arm_prints_a_complete_line(monkeypatch):
    """The reference arm (the oracle on the host cores) runs end to end on a
    small budget and reports the contract's keys; rank 0 alone works."""
    import argparse

    monkeypatch.setattr(bench, "REFERENCE_SECONDS", 1.0)
    args = argparse.Namespace(steps=2, warmup=1)
    assert bench.run_reference(args, 1, 2) is None          # other ranks do no work
    r = bench.run_reference(args, 0, 1)
    assert r["impl"] == "reference" and r["steps"] == 2 and r["warmup"] == 1
    assert r["value"] > 0 and r["unit"] == "TFLOP/s" and r["higher_is_better"] is True
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == r["value"] and cb["cores"] >= 1 and cb["sample"]
    assert r["e2e"] == {"value": r["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert r["config"]["M"] == 4096 and r["config"]["N"] == 9216 and r["config"]["K"] == 3072


def test_cpu_baseline_legs_run_on_the_host():
    """The main arm's CPU-baseline legs (the oracle on a bounded sample of the
    headline workload, and the single-core runs) need no GPU: run them on a
    small budget and check what they report."""
    tflops, spent, desc, rows, runs = bench.cpu_oracle_sample(0.5)
    assert tflops > 0 and spent > 0 and 16 <= rows <= 4096 and "extrapolated" in desc
    assert len(runs) == 3 and tflops == sorted(runs)[1]
    assert bench.cpu_model()
    single = bench.cpu_oracle_single_core()
    assert set(single) == {"0:tiny", "3:tern_m1"}
    assert all(v["seconds"] > 0 and v["gflops"] > 0 for v in single.values())


def test_an_optional_section_that_fails_is_recorded_not_fatal():
    res = {"value": 1.0}
    assert bench.report_section(res, "ok", lambda: 3) == 3 and "errors" not in res

    def boom():
        raise RuntimeError("out of memory")
    assert bench.report_section(res, "sweep", boom) is None
    assert res["errors"] == {"sweep": "RuntimeError: out of memory"} and res["value"] == 1.0


def test_policy_module_report_agrees_with_direct_cosines():
    """The bench's policy report from per-layer terms, on synthetic outputs:
    its cosines equal the ones computed directly, and its front and cheapest
    policy are those of the enumeration."""
    import itertools

    import numpy as np
    g = np.random.default_rng(3)
    names = ["a", "b", "c"]
    dense, quant, nbytes = {}, {}, {}
    for n in names:
        d = g.standard_normal(200)
        dense[n] = d
        for bits, amp in ((4, 0.1), (8, 0.006)):
            quant[(n, bits)] = d + amp * g.standard_normal(200)
            nbytes[(n, bits)] = 100 * bits + len(n)
    terms = []
    for n in names:
        d = dense[n]
        opts = {b: (nbytes[(n, b)], float((quant[(n, b)] - d) @ d), float((quant[(n, b)] - d) @ (quant[(n, b)] - d)))
                for b in (4, 8)}
        terms.append((n, float(d @ d), opts))
    rows = []
    dcat = np.concatenate([dense[n] for n in names])
    for combo in itertools.product((4, 8), repeat=3):
        q = np.concatenate([quant[(n, b)] for n, b in zip(names, combo)])
        rows.append({"bits": dict(zip(names, combo)),
                     "cosine_vs_dense_bf16": float(q @ dcat / np.sqrt((q @ q) * (dcat @ dcat)))})
    r = bench.policy_module_report(terms, 10_000, rows, min_cosine=0.9999)
    assert r["max_abs_cosine_difference_vs_direct"] < 1e-12
    assert r["front"][0]["bits"] == {"a": 4, "b": 4, "c": 4} and r["front"][-1]["bits"] == {"a": 8, "b": 8, "c": 8}
    best = r["cheapest_with_cosine_at_least_0.9999"]
    ok = [row for row in rows if row["cosine_vs_dense_bf16"] >= 0.9999]
    cheapest = min(ok, key=lambda row: sum(nbytes[(n, b)] for n, b in row["bits"].items()))
    assert best == cheapest["bits"]


def test_headline_parity_accepts_the_oracle_and_rejects_a_corrupt_output():
    """The parity check of the timed run's output, given an output built on
    the host: the oracle's own result rounded to bf16 passes, the same with a
    corrupted row does not."""
    import numpy as np
    import torch

    import oracle as O
    import workloads as WL
    lin = WL.workload(bench.HEADLINE_CID).linears[bench.HEADLINE_LIN]
    X, W, bias = WL.make_inputs(lin, bench.HEADLINE_CID, bench.HEADLINE_LIN)
    p, s, b = O.pack_ref(W, lin.bits, lin.group)
    rows = np.unique(np.concatenate([np.arange(32), np.linspace(0, lin.M - 1, 32).astype(np.int64)]))
    y = np.zeros((lin.M, lin.N), dtype=np.float32)
    y[rows] = O.qgemm_ref_rows(rows, X, p, s, b, lin.bits, lin.group, lin.K, bias)
    out = torch.from_numpy(y).to(torch.bfloat16)
    r = bench.headline_parity(out)
    assert r["rows_checked"] == rows.size and r["within_tolerance"] and r["rel_frobenius"] < 3e-3
    out[rows[5]] = -out[rows[5]]
    r = bench.headline_parity(out)
    assert not r["within_tolerance"]


def test_main_arm_prints_one_compact_headline_line(monkeypatch, capsys):
    """The main arm end to end with its GPU measurements stubbed: stdout
    holds exactly one line, valid JSON within HEADLINE_MAX_BYTES carrying the
    contract's keys, even when the detailed sections are large; those go to
    stderr (and the --report file) as lines of their own."""
    import json

    import torch

    import workloads as WL
    lin = WL.workload(bench.HEADLINE_CID).linears[bench.HEADLINE_LIN]
    peaks = {"hbm_gbs": 6553.9, "bf16_tflops": 1638.3, "bf16_tflops_sustained": 1379.1, "source": "test"}
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 40}
    e2e = {"value": 160.0, "unit": "TFLOP/s", "h2d_bytes_per_step": lin.M * lin.K * 2,
           "d2h_bytes_per_step": lin.M * lin.N * 2}

    def fake_run_ours(args, rank, world, local_rank):
        job = bench.replica_throughput(2 * lin.M * lin.N * lin.K, args.steps, args.steps * 180e-6, world)
        res = bench.assemble_ours(args, world, lin, 4, job, 178e-6, e2e, clk, peaks)
        return res, peaks, None

    big_rows = [{"workload": 4, "linear": f"lin{i}", "us": 100.0 + i, "frac_of_roofline": 0.8, "pad": "x" * 400}
                for i in range(40)]
    block = {"us_total": 1184.0, "cosine_vs_dense_bf16_all_five": 0.998}
    monkeypatch.setattr(torch.cuda, "set_device", lambda *_: None)
    monkeypatch.setattr(bench, "run_ours", fake_run_ours)
    monkeypatch.setattr(bench, "sweep", lambda peaks: (big_rows, block))
    monkeypatch.setattr(bench, "fused_sweep", lambda: [{"pad": "z" * 500}] * 10)
    monkeypatch.setattr(bench, "policy_sweep", lambda: {"assignments": [{"pad": "w" * 200}] * 32})
    monkeypatch.setattr(bench, "cpu_baseline", lambda s: {"value": 0.4, "unit": "TFLOP/s", "cores": 16,
                                                          "kind": "oracle", "sample": "stub", "cpu_model": "cpu"})
    monkeypatch.setattr(bench, "cpu_oracle_single_core", lambda: {"0:tiny": {"seconds": 0.1}})
    monkeypatch.setattr(bench, "headline_parity", lambda out: {"within_tolerance": True})
    assert bench.main(["--steps", "20", "--warmup", "5"]) == 0
    cap = capsys.readouterr()
    lines = cap.out.strip().splitlines()
    assert len(lines) == 1
    assert len(lines[0]) <= bench.HEADLINE_MAX_BYTES
    r = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "config", "dtype",
              "roofline", "cpu_baseline", "e2e", "clocks", "parity", "peaks", "gpu_launches", "higher_is_better"):
        assert k in r, k
    assert r["value"] > 0 and r["steps"] == 20 and r["warmup"] == 5 and r["n_gpus"] == 1
    assert abs(r["ms_per_step"] - 0.18) < 1e-9
    assert r["roofline"]["bound"] == "tensor" and 0 < r["roofline"]["frac"] < 1.2
    assert r["e2e"]["h2d_bytes_per_step"] > 0 and r["e2e"]["d2h_bytes_per_step"] > 0
    assert r["sweep_summary"]["4:lin0"] == [100.0, 0.8]
    assert "sweep" not in r and "policy_sweep" not in r and "clocks_detail" not in r
    sections = [json.loads(x)["report"] for x in cap.err.splitlines() if x.startswith('{"report"')]
    assert {"sweep", "fused_epilogues", "policy_sweep", "workload4_block", "clocks_detail"} <= set(sections)


def test_headline_line_drops_summaries_before_exceeding_its_size():
    import json
    res = {"metric": "m", "value": 1.0, "sweep_summary": {f"k{i}": [1.0, 0.5] for i in range(2000)}}
    line = bench.headline_line(res)
    assert len(line) <= bench.HEADLINE_MAX_BYTES
    assert json.loads(line) == {"metric": "m", "value": 1.0}
