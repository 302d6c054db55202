"""The benchmark's JSON contract, on the CPU: the reference arm (the oracle timed on
the host cores) prints one line with the keys the measurement contract requires,
for the same metric and workload as the GPU arm; the clock sampler summarises to
the `clocks` object even where no GPU or NVML is present."""
import contextlib
import io
import json

import bench
import synthetic_inputs as si

REQUIRED = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config"}


def test_reference_arm_prints_one_contract_line():
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        rc = bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0", "--cpu-tokens", "32"])
    assert rc == 0
    lines = [line for line in out.getvalue().splitlines() if line.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert REQUIRED <= set(d)
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True and d["value"] > 0
    # the default workload is the largest single-GPU configuration: the GPT-2 1.5B FFN
    assert d["config"]["workload"] == si.GPT2_1P5B.name
    assert d["config"]["d_model"] == 1600 and d["config"]["d_ff"] == 6400 and d["config"]["tokens_per_gpu"] == 32768
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and "32 of 32768" in cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_clock_sampler_summary_without_a_gpu():
    c = bench.ClockSampler(0, period_s=0.01)
    with c:
        pass
    s = c.summary()
    assert set(s) >= {"sm_mhz", "sm_max_mhz", "reasons"}
    if not c.samples:
        assert s["sm_mhz"] is None and s["reasons"]


def test_clock_sampler_splits_samples_by_phase():
    """Samples are attributed to the phase whose mark precedes them; the last phase runs on."""
    c = bench.ClockSampler(0, period_s=0.01)
    c.source = "nvml"
    c.marks = [("a", 0.0), ("b", 10.0)]
    c.samples = [(1.0, 1900.0, 1965.0, set()), (2.0, 1800.0, 1965.0, {"sw_power_cap"}),
                 (11.0, 1500.0, 1965.0, set()), (-1.0, 1000.0, 1965.0, set())]
    s = c.summary()
    assert s["phases"]["a"] == {"sm_mhz_median": 1850.0, "sm_mhz_min": 1800.0, "samples": 2}
    assert s["phases"]["b"] == {"sm_mhz_median": 1500.0, "sm_mhz_min": 1500.0, "samples": 1}
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 4 and s["sm_min_mhz"] == 1000.0


def test_headline_flops_are_the_four_ffn_gemms():
    wl = si.GPT2_355M
    assert wl.gemm_flops() == 4 * 2 * 8192 * 1024 * 4096


def test_weight_sequence_is_cumulative_and_seeded():
    wl = si.FFNWorkload("tiny", d=16, ff=32, tokens=16, dtype="f16", steps=3)
    W1, W2 = wl.weights()
    seq = wl.weight_sequence(W1, W2)
    assert [len(x) for x in seq] == [4, 4]
    for li in range(2):
        for t in range(3):
            assert seq[li][t + 1].equal(si.perturb(seq[li][t], wl.perturb_seed(t, li)))
    assert not seq[0][1].equal(seq[0][2])
