"""bench.py's nvidia-smi clock summary (parsed on the CPU from a recorded sample)."""
import bench


def test_clock_summary_parses_rows(tmp_path):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    s.proc = object()  # as if nvidia-smi had run
    rows = ["0, 1965, 1965, 650.1, 0x0, Not Active, Not Active, Not Active, Active, 3996, 61",
            "0, 1950, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Active, 3996, 63",
            "0, 300, 1965, 90.0, 0x0, Not Active, Not Active, Not Active, Not Active, 3996, [N/A]",
            "0, 1965, 1965, 640.0, 0x0, Not Active, Not Active, Not Active, Not Active"]
    open(s.path, "w").write("\n".join(rows) + "\n")
    out = s.summary()
    assert out["samples"] == 4 and out["sm_max_mhz"] == 1965.0
    assert out["sm_mhz"] == 1965.0            # median of the samples under load (> half of max)
    assert out["reasons"] == ["sw_power_cap"]
    assert out["mem_mhz"] == 3996.0 and out["mem_temp_c"] == 63.0
