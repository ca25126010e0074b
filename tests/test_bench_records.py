"""Host-side records of bench.py on the CPU: the ncu traffic figures are reported only
while the captured sources are unchanged, the peak denominators carry their source,
and stage times are averaged per step, not per launch."""
import hashlib
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

CSRC = os.path.join(ROOT, "gated_delta_rule_transitions_b200", "csrc")


def _tag(name):
    with open(os.path.join(CSRC, name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def test_traffic_records_name_existing_sources_and_plausible_bytes():
    for kernel, (nbytes, files) in bench.NCU_TRAFFIC.items():
        assert nbytes > 0, kernel
        for name in files:
            assert os.path.exists(os.path.join(CSRC, name)), (kernel, name)


def test_traffic_reported_only_for_the_captured_source(monkeypatch):
    name = "tc_common.cuh"
    monkeypatch.setitem(bench.NCU_TRAFFIC, "probe", (123.0, {name: _tag(name)}))
    assert bench.ncu_traffic("probe") == 123.0
    monkeypatch.setitem(bench.NCU_TRAFFIC, "probe", (123.0, {name: "0" * 16}))
    assert bench.ncu_traffic("probe") is None
    monkeypatch.setitem(bench.NCU_TRAFFIC, "probe", (123.0, {"no_such_file.cu": "0" * 16}))
    assert bench.ncu_traffic("probe") is None
    assert bench.ncu_traffic("not_recorded") is None


def test_peaks_are_labelled_by_source(monkeypatch, tmp_path, capsys):
    hbm, burst, sustained, src = bench._peaks()
    assert src in ("measured", "fallback")
    assert hbm > 0 and burst > 0 and sustained > 0
    # without the measurement file the fallback figures are used, labelled and announced
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    hbm, burst, sustained, src = bench._peaks()
    assert src == "fallback" and (hbm, burst, sustained) == (6650.0, 1590.0, 1400.0)
    assert "fallback" in capsys.readouterr().err


def test_stage_times_are_per_step():
    # a stage that launched 2 kernels per step for 5 steps, 10 ms in all: 2 ms per step
    assert bench._stage_avg({"decode": (10.0, 10)}, "decode", 5) == 2.0
    assert bench._stage_avg({}, "decode", 5) is None
    assert bench._stage_avg({"decode": (0.0, 0)}, "decode", 5) is None
