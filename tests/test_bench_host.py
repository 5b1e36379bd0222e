"""Host-side parts of bench.py that need no GPU: the clock sampler's
in-process polling and summary (with a fake NVML), the bounded reference
arm's per-step budget, the `--gpus` launcher, and the inputs of the roofline
object (peak source, traffic record validity, algorithmic bytes and FLOPs)."""
import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    try:
        sys.argv = ["bench.py"]
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


class FakeNvml:
    NVML_CLOCK_SM = 1

    def __init__(self, mhz=1700, reasons=0x4, fail=False):
        self.mhz, self.reasons, self.fail = mhz, reasons, fail

    def nvmlInit(self):
        if self.fail:
            raise RuntimeError("NVML unavailable")

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.mhz

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.reasons


def test_clock_polling_until_the_timing_event_completes():
    b = _bench()
    clk = b.ClockSampler(0)
    calls = []
    clk.poll_until(lambda: len(calls.append(1) or calls) > 4, nvml=FakeNvml())
    s = clk.summary()
    assert s["samples"] == 4 and s["sm_mhz"] == 1700 and s["sm_min_mhz"] == 1700
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_polling_never_raises():
    b = _bench()
    clk = b.ClockSampler(0)
    clk.poll_until(lambda: False, nvml=FakeNvml(fail=True))
    assert clk.summary() is None


def test_reference_budget_is_bounded():
    b = _bench()
    src = open(os.path.join(ROOT, "bench.py")).read()
    assert "90.0 / max(1, args.steps + args.warmup)" in src
    assert hasattr(b, "OracleSampler")


def test_reference_arm_json_line_on_cpu(monkeypatch):
    """The reference arm runs the oracle on host cores only: on the tiny
    workload, with each step's oracle budget cut to a few milliseconds, it
    prints the contract's keys with its own metric in e2e and cpu_baseline."""
    import argparse
    import json

    b = _bench()
    real_run = b.OracleSampler.run
    monkeypatch.setattr(b.OracleSampler, "run", lambda self, budget: real_run(self, 0.002))
    args = argparse.Namespace(workload="tiny_f32", steps=2, warmup=3)
    res = b.run_reference(args, rank=0, world=1)
    line = json.loads(json.dumps(res))
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["metric"] == b.METRIC
    assert line["value"] > 0 and line["unit"] == "tokens/s"
    assert abs(line["ms_per_step"] - 1e3 / line["value"]) < 1e-9 * line["ms_per_step"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert "tiny_f32" in line["config"]["workload"]
    # Ranks other than 0 do no work and print nothing.
    assert b.run_reference(args, rank=1, world=2) is None


def _json_lines(out):
    import json
    return [json.loads(ln) for ln in out.splitlines() if ln.startswith("{")]


def test_gpus_flag_launches_one_rank_per_gpu():
    """`bench.py --gpus 2` without a launcher re-runs itself as two ranks under
    torch.distributed.run; in the host-only dry run (gloo, no GPU) rank 0
    reports two ranks and the slowest rank's time (rank 1 steps 2 ms, rank 0
    1 ms), never a one-rank result."""
    import subprocess

    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--dry-run", "--steps", "5", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["dry_run"] is True and line["n_gpus"] == 2
    assert line["ms_per_step"] >= 2.0 and line["ms_per_step"] >= line["rank0_ms_per_step"]


def test_gpus_flag_must_match_the_launcher():
    import subprocess

    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--dry-run", "--steps", "2", "--warmup", "3"],
                       capture_output=True, text=True, timeout=120, env=env, cwd=ROOT)
    assert r.returncode != 0 and "launcher started 1 rank" in r.stderr
    assert not _json_lines(r.stdout)


def test_peaks_measured_file_else_fallback(tmp_path, monkeypatch):
    """The roofline denominators come from MEASURED_PEAKS.json when it is
    present and are labelled as the fallback otherwise."""
    b = _bench()
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    hbm, tf, tf_sus, src = b._peaks()
    assert (hbm, tf, src) == (b.FALLBACK_HBM_GBS, b.FALLBACK_BF16_TFLOPS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        '{"hbm_gbs": 6552.0, "bf16_tflops": 1638.5, "bf16_tflops_sustained": 1368.2}')
    assert b._peaks() == (6552.0, 1638.5, 1368.2, "measured")


def test_traffic_record_only_for_the_kernel_it_was_taken_on(tmp_path, monkeypatch):
    """A DRAM-traffic record is reported only while the decode kernel's
    sources hash to the value stored beside it."""
    import json
    import shutil
    b = _bench()
    csrc = tmp_path / "mla_latent_kv_nope_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("k_decode_tc.cu", "tile_deal.cuh", "common.cuh", "sm100.cuh"):
        shutil.copy(os.path.join(ROOT, "mla_latent_kv_nope_b200", "csrc", name), csrc / name)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    rec = {"v3_bf16": {"source_hash": b._decode_source_hash(), "traffic_bytes_per_launch": 123.0}}
    (tmp_path / "profiles" / "decode_traffic.json").write_text(json.dumps(rec))
    assert b._ncu_traffic("v3_bf16") == 123.0
    assert b._ncu_traffic("longctx_bf16") is None
    with open(csrc / "k_decode_tc.cu", "a") as f:
        f.write("\n")
    assert b._ncu_traffic("v3_bf16") is None


def test_algorithmic_counts_are_the_closed_forms():
    """Per cached row the decode reads one latent row (576 bf16 = 1152 B, or
    512 E4M3 codes + 64 bf16 RoPE keys + a 4-byte scale = 644 B) and does
    2 H (576 + 512) FLOPs (QK^T over d_c + d_r, P.c over d_c)."""
    import numpy as np
    sys.path.insert(0, ROOT)
    from mla_latent_kv_nope_b200 import inputs
    b = _bench()
    w = inputs.WORKLOADS["v3_bf16"]
    lens = np.full(32, 8193)
    byts, flops, rows = b._algorithmic(w, lens)
    assert rows == 32 * 8193
    assert byts == rows * 1152
    assert flops == 2 * 128 * rows * (576 + 512)
    byts8, flops8, _ = b._algorithmic(w, lens, fp8=True)
    assert byts8 == rows * 644 and flops8 == flops


def test_clock_summary_of_a_second_window():
    """The decode-only pass gets its own clock summary from the separate
    sampler's lines inside its window; the in-process samples belong to the
    timed steps only."""
    b = _bench()
    clk = b.ClockSampler(0)
    clk.poll_until(lambda: len(clk.inproc) >= 3, nvml=FakeNvml(mhz=1965, reasons=0))
    clk.start(); clk.t_start, clk.t_stop = 10.0, 20.0
    clk.lines = ["12.0 1965 0", "25.0 1800 4", "26.0 1812 4", "40.0 1500 8", "bad line"]
    main = clk.summary()
    assert main["samples"] == 4 and main["reasons"] == []
    dec = clk.summary((24.0, 30.0))
    assert dec["samples"] == 2 and dec["sm_min_mhz"] == 1800 and dec["reasons"] == ["sw_power_cap"]
    assert clk.summary((50.0, 60.0)) is None
