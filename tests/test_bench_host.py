"""Host-side logic of the benchmark that needs no GPU: the clock record is
built only from samples inside the timed window, and says so when none fell
there."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _FakeProc:
    def __init__(self, text):
        self.text = text

    def kill(self):
        pass

    def communicate(self, timeout=None):
        return self.text, ""


def _sampler(lines, t0, t1, tmp_path=None):
    import tempfile
    s = bench.ClockSampler(device=None)
    fd, s.path = tempfile.mkstemp(suffix=".clk")
    with os.fdopen(fd, "w") as f:
        f.write("\n".join(lines))
    s.proc = _FakeProc("")
    s.smax = 1965.0
    s.t0, s.t1 = t0, t1
    return s


def test_clock_record_uses_only_the_timed_window():
    lines = ["99.0 600 0",          # before the window: idle clock, ignored
             "100.001 1965 0", "100.003 1950 4", "100.005 1965 0",
             "100.2 300 8"]          # after the window: ignored
    rec = _sampler(lines, 100.0, 100.01).stop()
    assert rec["samples"] == 3
    assert rec["sm_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["sm_max_mhz"] == 1965.0
    assert "note" not in rec


def test_clock_record_without_samples_says_so():
    rec = _sampler(["50.0 1965 0", "garbage"], 100.0, 100.005).stop()
    assert rec["samples"] == 0 and rec["sm_mhz"] is None
    assert "no sample" in rec["note"]


def test_clock_record_maps_slowdown_bits():
    rec = _sampler(["1.0 1500 104"], 0.0, 2.0).stop()  # 0x40 | 0x20 | 0x8
    assert rec["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_reference_arm_names_the_same_workload_config(capsys, monkeypatch):
    """Both arms print the same `config` object: the reference arm builds it
    with the same function, from the same seeded host inputs, that the
    CUDA arm uses (sizes and the L2 note only; no device needed)."""
    import json
    from dual_flow_transformer_b200 import synth
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.delenv("RANK", raising=False)
    args = bench.parse_args(["--impl", "reference", "--workload", "tiny", "--steps", "2",
                             "--warmup", "3"])
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    w = synth.WORKLOADS["tiny"]
    host = synth.make_attn_inputs(w, seed=bench.synth_seed("tiny"))
    assert line["config"] == bench.workload_config("tiny", w, host)
    assert line["impl"] == "reference" and line["config"]["parallelism"] == "single GPU"
