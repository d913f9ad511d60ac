"""Host-side logic of bench.py, including the multi-rank path on CPU (gloo, 2 ranks).

The decode path has no data exchange: ranks run independent replicas and only
the timing is reduced (max over ranks).  These tests run that reduction and the
throughput arithmetic without a GPU.
"""
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [12.5, 30.0]
        mx = bench.reduce_max(times[rank], torch.device("cpu"))
        rate = bench.whole_job_tokens_per_s(world, 512, 10, mx)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"max": mx, "rate": rate}, f)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_reduction_and_weak_scaling_rate(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn")
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    assert res[0] == res[1]
    assert res[0]["max"] == 30.0
    assert res[0]["rate"] == pytest.approx(2 * 512 * 10 / 0.030)


def test_single_process_reduction_is_identity():
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    assert bench.whole_job_tokens_per_s(1, 512, 256, 1000.0) == pytest.approx(512 * 256)


def test_algorithmic_bytes_follow_the_pending_fill():
    # one sequence, fill 255: step 0 reads 256 pending rows, then the block empties
    b0 = bench.algorithmic_read_bytes([255], 0, 1)
    b1 = bench.algorithmic_read_bytes([255], 1, 1)
    per_group_fixed = 2 * 4 * 512 + 2 * 4 * 1024
    assert b0 == 4 * ((2048 + 256) * 1024 + per_group_fixed)
    assert b1 == 4 * ((2048 + 1) * 1024 + per_group_fixed)


def _run_reference(env_extra=None):
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **(env_extra or {}))
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                           "--warmup", "0"], cwd=root, env=env, capture_output=True, text=True,
                          timeout=600)


def test_reference_arm_prints_one_contract_line():
    """The reference arm is the oracle on the host cores: one JSON line with the
    base contract's keys, the impl tag, a cpu_baseline describing the run and an
    e2e block that moves no bytes."""
    r = _run_reference()
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tok/s"
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == bench.WORKLOAD
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tok/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    """Under torchrun only rank 0 runs and prints the reference line."""
    r = _run_reference({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not any(l.startswith("{") for l in r.stdout.splitlines())


class _FakeNvml:
    """Read-only NVML stand-in: a scripted SM clock and clock-event-reason bits."""
    NVML_CLOCK_SM = 1

    def __init__(self, script):
        self.script = list(script)  # (sm MHz, reason bits) per query
        self.i = 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByUUID(self, uuid):
        return "h"

    def nvmlDeviceGetHandleByIndex(self, i):
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.script[min(self.i, len(self.script) - 1)][0]

    def nvmlDeviceGetCurrentClocksThrottleReasons(self, h):
        v = self.script[min(self.i, len(self.script) - 1)][1]
        self.i += 1
        return v


def test_clock_sampler_keeps_only_timed_samples_and_names_reasons():
    """The bench's clock record: samples outside begin/end are dropped, the median
    SM clock and the union of the reasons seen inside are reported (0x4 is
    sw_power_cap, 0x8 hw_slowdown, 0x20 sw_thermal_slowdown, 0x40
    hw_thermal_slowdown)."""
    import time
    fake = _FakeNvml([(1965, 0x0), (1800, 0x4), (1700, 0x4 | 0x40)])
    cs = bench.ClockSampler(0)
    cs.nvml = (fake, "h")
    t = time.monotonic()
    cs.windows = [[t, t + 1.0]]
    cs.samples = [(t - 0.5, 1200.0, 1965.0, {"hw_slowdown"}),  # before the window
                  (t + 0.1, 1965.0, 1965.0, set()),
                  (t + 0.2, 1800.0, 1965.0, {"sw_power_cap"}),
                  (t + 0.3, 1700.0, 1965.0, {"sw_power_cap", "hw_thermal_slowdown"}),
                  (t + 2.0, 900.0, 1965.0, {"sw_thermal_slowdown"})]  # after it
    cs.stop_flag = False

    class _Done:
        def join(self, timeout=None):
            pass
    cs.th = _Done()
    rec = cs.stop()
    assert rec["samples"] == 3
    assert rec["sm_mhz"] == 1800.0
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_clock_sampler_polls_nvml_only_inside_a_window():
    """The polling thread reads NVML while a window is open and not after."""
    import time
    fake = _FakeNvml([(1900, 0x4)])
    cs = bench.ClockSampler(0)
    cs.nvml = (fake, "h")
    import threading
    cs.th = threading.Thread(target=cs._poll_nvml, daemon=True)
    cs.th.start()
    time.sleep(0.05)
    assert not cs.samples          # no window yet
    cs.begin()
    time.sleep(0.1)
    cs.end()
    n = len(cs.samples)
    time.sleep(0.05)
    rec = cs.stop()
    assert n >= 3 and len(cs.samples) == n
    assert rec["sm_mhz"] == 1900.0 and rec["reasons"] == ["sw_power_cap"]
