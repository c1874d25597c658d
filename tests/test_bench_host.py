"""Host logic of bench.py, on the CPU: the byte models behind the roofline
figures, the clock-sample summary, and the reference arm's JSON line (the
float64 oracle timed on host cores)."""
import json
import types

import pytest

import bench


def _wl(batch, seqlen, dim, dstate, dtype, gate=True, D=True, bias=True,
        h0=False):
    present = object()
    return types.SimpleNamespace(
        batch=batch, seqlen=seqlen, dim=dim, dstate=dstate, dtype=dtype,
        dev={"z": present if gate else None, "D": present if D else None,
             "delta_bias": present if bias else None,
             "h0": present if h0 else None})


def test_scan_bytes_of_the_2p8b_layer():
    # x, raw step, z read and y written once (bf16, 4 x 8192 x 5120 each),
    # B and C once (4 x 8192 x 16 bf16), A_log, D, step bias, and h_last
    # (float32 [4, 5120, 16]); no h0. 1.346 GB per call.
    act = 4 * 8192 * 5120 * 2
    want = 4 * act + 2 * (4 * 8192 * 16 * 2) + (5120 * 16 * 4 + 2 * 5120 * 4) \
        + 4 * 5120 * 16 * 4
    assert bench.algorithmic_bytes(_wl(4, 8192, 5120, 16, "bf16")) == want
    assert round(want / 1e9, 3) == 1.346


def test_scan_bytes_options():
    base = bench.algorithmic_bytes(_wl(1, 64, 16, 4, "f32", gate=False,
                                       D=False, bias=False))
    # x, raw step, y; B, C; A_log; h_last
    assert base == 3 * 64 * 16 * 4 + 2 * 64 * 4 * 4 + 16 * 4 * 4 + 16 * 4 * 4
    gated = bench.algorithmic_bytes(_wl(1, 64, 16, 4, "f32", gate=True,
                                        D=False, bias=False))
    assert gated - base == 64 * 16 * 4
    with_h0 = bench.algorithmic_bytes(_wl(1, 64, 16, 4, "f32", gate=False,
                                          D=False, bias=False, h0=True))
    assert with_h0 - base == 16 * 4 * 4
    conv = bench.algorithmic_bytes(_wl(1, 64, 16, 4, "f32", gate=False,
                                       D=False, bias=False), op="conv")
    assert conv - base == 16 * bench.CONV_WIDTH * 4 + 16 * 4


def test_decode_bytes_of_the_batched_step():
    # 1024 sequences of the 2.8B layer, one token, width-4 conv buffer:
    # 797 MB per launch
    n = bench.decode_bytes(_wl(1024, 1, 5120, 16, "bf16"))
    want = (2 * 1024 * 5120 * 16 * 4          # state in and out
            + 2 * 1024 * 5120 * 4 * 2         # conv buffer in and out
            + 4 * 1024 * 5120 * 2             # x_new, raw step, z, y
            + 2 * 1024 * 16 * 2               # B, C
            + 5120 * 16 * 4 + 5120 * 4 * 4 + 3 * 5120 * 4)
    assert n == want
    assert round(n / 1e6) == 797


def test_clock_summary():
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 880.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = c.summary()
    assert s == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0,
                 "reasons": ["sw_power_cap"], "samples": 3}
    empty = bench.ClockSampler(0)
    assert empty.summary()["samples"] == 0


def test_warmup_below_three_is_refused():
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--warmup", "2"])


def test_reference_arm_line(capsys):
    rc = bench.main(["--impl", "reference", "--shape", "0", "--steps", "2",
                     "--warmup", "3", "--reference-budget", "1"])
    assert rc == 0
    lines = [ln for ln in capsys.readouterr().out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["dtype"] == "f64" and d["data"] == "synthetic"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1
    assert cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"],
                        "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "b=1" in d["config"]["workload"]


def test_every_op_has_kernel_sources_and_a_config():
    """Each --op choice names the sources its traffic figure is tied to, and
    its config record names the operation."""
    ops = ("scan", "conv", "step", "bwd", "train")
    wl = _wl(4, 8192, 5120, 16, "bf16")
    for op in ops:
        assert op in bench.KERNEL_SOURCES
        assert len(bench.kernel_source_hash(op)) == 16
        cfg = bench.workload_config(wl, op, 1, 3)
        assert cfg["op"] == op and cfg["parallelism"] == "dp1"
    assert "backward" in bench.workload_config(wl, "bwd", 1, 3)["workload"]
    assert "training step" in bench.workload_config(wl, "train", 1,
                                                    3)["workload"]
    # a world of 2 doubles the global batch (weak scaling)
    assert bench.workload_config(wl, "scan", 2, 3)["global_batch"] == 8


def test_traffic_record_goes_stale_with_its_sources(monkeypatch):
    """A recorded ncu traffic figure is reported only while the sources it
    was captured from are unchanged; otherwise the line carries null and
    says why."""
    now = bench.kernel_source_hash("scan")
    monkeypatch.setattr(bench, "NCU_TRAFFIC", {("scan", 3): (1.5e9, now)})
    value, why = bench.traffic_record("scan", 3)
    assert value == 1.5e9 and now in why
    monkeypatch.setattr(bench, "NCU_TRAFFIC",
                        {("scan", 3): (1.5e9, "0" * 16)})
    value, why = bench.traffic_record("scan", 3)
    assert value is None and "stale" in why
    value, why = bench.traffic_record("bwd", 3)
    assert value is None and "no ncu capture" in why


@pytest.mark.parametrize("op", ["step", "bwd", "train", "conv"])
def test_reference_arm_times_the_forward_only(capsys, op):
    rc = bench.main(["--impl", "reference", "--op", op, "--steps", "2",
                     "--warmup", "3"])
    assert rc == 0
    d = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert d["impl"] == "reference" and "unavailable" in d


def test_clock_summary_keeps_the_timed_region():
    """Samples taken before the timed region started are left out; the
    first sample after it (which covers its last moments) is kept."""
    c = bench.ClockSampler(0)
    idle = "0, 600, 1965, 90.0, 0x0, Not Active, Not Active, Not Active, " \
           "Not Active"
    busy = "0, 1965, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, " \
           "Not Active"
    c.lines = [idle, idle]
    c.mark()
    c.lines += [busy, busy]
    c.mark(end=True)
    c.lines += [idle]
    s = c.summary()
    assert s["sm_mhz"] == 1965.0 and s["samples"] == 2
