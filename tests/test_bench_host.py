"""Host-side pieces of bench.py that need no GPU: the clock sampler's parsing and window
filter, and the lookup of the DRAM traffic recorded by an ncu capture."""
import datetime
import os
import time

import bench


class _DoneProcess:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        pass


def test_clock_sampler_keeps_only_samples_inside_the_timed_window(tmp_path):
    cs = bench.ClockSampler(0)
    cs.path = str(tmp_path / "clocks.csv")
    now = time.time()
    with open(cs.path, "w") as f:
        for i in range(6):
            t = datetime.datetime.fromtimestamp(now + 0.1 * i).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
            reason = "Active" if i in (0, 5) else "Not Active"   # only outside the window
            f.write(f"{t}, 0, {1800 + i}, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, {reason}\n")
    cs.proc = _DoneProcess()
    clk = cs.stop((now + 0.05, now + 0.45))
    assert clk["samples"] == 4
    assert clk["sm_mhz"] == 1802.5
    assert clk["sm_max_mhz"] == 1965.0
    assert clk["reasons"] == []          # the sw_power_cap samples fell outside the window
    assert not os.path.exists(cs.path)


def test_recorded_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    src_dir = tmp_path / "swin3d_window_attention_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    src = src_dir / "attn_tcgen05.cu"
    src.write_text("int a = 1;  // kernel v1\n")
    sha = bench.kernel_code_sha256(src.read_text())
    (tmp_path / "profiles" / "window_attn_tc_stage1_full.md").write_text(
        f"- kernel source: `x`, code sha256 `{sha}`\n- dram_bytes_per_launch: 1234567  (algorithmic: 1)\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic() == 1234567
    src.write_text("// a new comment\nint a = 1;  /* edited */\n\n")   # comments only: same code
    assert bench.recorded_traffic() == 1234567
    src.write_text("int a = 2;\n")             # the code changed since the capture
    assert bench.recorded_traffic() is None
