"""Host-side pieces of bench.py that need no GPU: the clock sampler's parsing and window
filter, and the lookup of the DRAM traffic recorded by an ncu capture."""
import datetime
import json
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


def test_recorded_traffic_follows_the_kernel_source(tmp_path):
    src_dir = tmp_path / "swin3d_window_attention_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    files = {"attn_tcgen05.cu": "int a = 1;  // kernel v1\n", "attn_common.cuh": "int d = 1;\n",
             "sm100_ptx.cuh": "int b = 1;\n", "s3w_common.cuh": "int c = 1;\n"}
    for name, text in files.items():
        (src_dir / name).write_text(text)
    sha = bench.kernel_code_sha256(str(tmp_path))
    (tmp_path / "profiles" / "window_attn_tc_stage1.json").write_text(json.dumps(
        {"code_sha256": sha, "dram_bytes_read": 1000000, "dram_bytes_write": 234567}))
    assert bench.recorded_traffic(str(tmp_path)) == 1234567
    (src_dir / "attn_tcgen05.cu").write_text("// a new comment\nint a = 1;  /* edited */\n\n")   # comments only
    assert bench.recorded_traffic(str(tmp_path)) == 1234567
    (src_dir / "sm100_ptx.cuh").write_text("int b = 2;\n")    # a header the kernel includes changed
    assert bench.recorded_traffic(str(tmp_path)) is None


def test_roofline_picks_the_binding_bound():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0}
    r = bench.roofline(1e9, 1e9, 2.0, peaks)          # 1 ms of bytes, 0.01 ms of FLOPs
    assert r["bound"] == "hbm" and abs(r["frac"] - 0.5) < 1e-12 and abs(r["achieved"] - 500.0) < 1e-9
    r = bench.roofline(1e6, 1e12, 20.0, peaks)        # 0.001 ms of bytes, 10 ms of FLOPs
    assert r["bound"] == "tensor" and abs(r["frac"] - 0.5) < 1e-12 and r["unit"] == "TFLOP/s"


def test_algorithmic_sizes_of_the_workloads():
    s1 = bench.WORKLOADS["stage1"]
    assert bench.attn_bytes(s1) == 4 * 259200 * 512 * 2 == 1061683200
    assert bench.attn_flops(s1) == 1800 * 8 * 4 * 144 * 144 * 64
    s3 = bench.WORKLOADS["stage3_padded"]
    assert bench.geometry(s3)[2] == 2 * 2 * 8 * 8          # 4x48x96 padded -> 2x8x8 windows per sample
    assert bench.attn_bytes(s3) == 4 * 2 * 4 * 45 * 90 * 2048 * 2   # real tokens only
    stack = bench.WORKLOADS["stack_b4"]
    per_block = bench.attn_bytes(stack) + bench.adaln_bytes(stack)
    assert abs(6 * per_block / 57.3e9 - 1) < 1e-3
