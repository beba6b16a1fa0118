"""Host-side logic of bench.py, including its multi-process path on CPU.

bench.py runs one process per GPU; every rank processes its own batch (weak
scaling, no data-path collective) and the step time is the maximum over
ranks.  The rank plumbing is exercised here with world_size 2 over gloo.
"""
import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def test_parse_args_defaults_and_checks():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.steps >= 1 and a.impl == "muir"
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])
    with pytest.raises(SystemExit):
        bench.parse_args(["--steps", "0"])


def test_flop_count_matches_formula():
    # 9Cd + C^2/3 + 8d^2 at C = d = 128
    assert abs(bench.flops_fwd_per_token_head(128, 128) - 283989.333) < 1e-2
    assert bench.BYTES_FWD == 2048 and bench.BYTES_BWD == 3840


def test_summarize_clocks():
    rows = [["1800", "1965", "900", "0x4", "Not Active", "Not Active", "Not Active", "Active"],
            ["1900", "1965", "950", "0x0", "Not Active", "Not Active", "Not Active", "Not Active"],
            ["garbage"]]
    c = bench.summarize_clocks(rows)
    assert c["sm_mhz"] == 1850 and c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]
    assert bench.summarize_clocks([])["samples"] == 0


class _FakeNvml:
    """Stands in for pynvml: answers the read-only queries the sampler makes."""
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, mask):
        self.clocks, self.mask, self.calls, self.shut = list(clocks), mask, 0, False

    def nvmlInit(self):
        pass

    def nvmlShutdown(self):
        self.shut = True

    def nvmlDeviceGetHandleByUUID(self, uuid):
        assert uuid.startswith("GPU-")
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.calls += 1
        return self.clocks[min(self.calls - 1, len(self.clocks) - 1)]

    def nvmlDeviceGetPowerUsage(self, h):
        return 950000

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.mask


def test_nvml_clock_sampler_reads_clocks_and_reasons():
    import time
    fake = _FakeNvml([1000, 1965, 1965, 1965, 1965], mask=0x4)
    s = bench.NvmlClockSampler("GPU-0000", nvml=fake, period=0.002)
    time.sleep(0.05)
    c = s.stop()
    assert fake.shut and c["samples"] >= 3
    assert c["sm_mhz"] == 1965 and c["sm_max_mhz"] == 1965  # the pre-region sample is dropped
    assert c["reasons"] == ["sw_power_cap"] and c["sampler"].startswith("nvml")
    fake = _FakeNvml([1965], mask=0x8 | 0x40)
    s = bench.NvmlClockSampler("GPU-0000", nvml=fake, period=0.002)
    time.sleep(0.02)
    assert s.stop()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]


def test_clock_sampler_falls_back_without_nvml(monkeypatch):
    class NoNvml:
        def __init__(self, *a, **k):
            raise RuntimeError("NVML not readable")
    monkeypatch.setattr(bench, "NvmlClockSampler", NoNvml)
    s = bench.clock_sampler("")
    assert isinstance(s, bench.ClockSampler)
    c = s.stop()  # nvidia-smi may be absent here: then no samples, and no error
    assert c["sampler"].startswith("nvidia-smi") and c["samples"] >= 0


def test_roofline_picks_the_binding_bound():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0,
             "source": "measured"}
    r = bench.kernel_roofline("k_bwd", 1.0, 524288, 128, 128, peaks)
    assert r["bound"] in ("hbm", "tensor") and 0 < r["frac"] < 1
    assert r["unit"] == ("GB/s" if r["bound"] == "hbm" else "TFLOP/s")
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12


def test_rank_seeds_are_distinct_and_rank0_is_canonical():
    assert bench.rank_seed(0) == 1002
    assert len({bench.rank_seed(r) for r in range(8)}) == 8


def test_reference_arm_only_rank0_reports():
    a = bench.parse_args(["--impl", "reference"])
    assert bench.reference_arm(a, rank=1, world=2) is None


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, lr = bench.dist_env()
    # each rank times its own batch; the job time is the slowest rank
    mine = 10.0 + 5.0 * rank
    worst = bench.max_over_ranks(mine, w, device="cpu")
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"rank": r, "world": w, "local": lr, "worst": worst,
                   "seed": bench.rank_seed(r)}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2(tmp_path):
    port = _free_port()
    mp.spawn(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert [x["rank"] for x in res] == [0, 1]
    assert all(x["world"] == 2 for x in res)
    assert all(x["worst"] == 15.0 for x in res)
    assert res[0]["seed"] != res[1]["seed"]


def _rank_step_main(rank, world, port, out_dir):
    """One rank of the bench's per-rank step logic on a CPU stand-in: its own
    seeded batch, the oracle's chunked forward as the step, the bench's timing
    protocol (warm-up, barrier, timed steps, barrier, max over ranks)."""
    import time

    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, _ = bench.dist_env()
    T = 32
    x = bench.rank_batch(r, B=1, H=1, T=T, dk=8, dv=8)
    calls = []

    def step():
        calls.append(1)
        oracle.chunk_fwd(*[x[n] for n in bench.NAMES], S0=x["S0"], chunk=8, threads=1)
        if r == 1:
            time.sleep(0.01)  # the slower rank sets the job time

    own = {}

    def timer():
        t = {}

        def start():
            t["0"] = time.perf_counter()

        def stop():
            own["ms"] = (time.perf_counter() - t["0"]) * 1e3
            return own["ms"]
        return start, stop

    ms = bench.timed_steps(step, 3, 2, w, timer, dist.barrier, device="cpu")
    value = bench.job_tokens_per_s(ms, T, w)
    with open(os.path.join(out_dir, f"step{rank}.json"), "w") as f:
        json.dump({"ms": ms, "own_ms": own["ms"] / 3, "value": value, "calls": len(calls),
                   "q0": float(x["q"].float().flatten()[0])}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_per_rank_step_gloo_world2(tmp_path):
    port = _free_port()
    mp.spawn(_rank_step_main, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    res = [json.load(open(tmp_path / f"step{r}.json")) for r in range(2)]
    assert all(x["calls"] == 5 for x in res)          # 2 warm-up + 3 timed steps
    assert res[0]["ms"] == res[1]["ms"]               # one job time: the max over ranks
    assert res[0]["ms"] >= max(x["own_ms"] for x in res) - 1e-9
    assert res[1]["own_ms"] >= 10.0                   # the slow rank's own time ...
    assert res[0]["ms"] >= 10.0                       # ... is the job's
    assert res[0]["value"] == pytest.approx(32 * 2 / (res[0]["ms"] / 1e3))
    assert res[0]["q0"] != res[1]["q0"]               # each rank has its own batch


def test_gpus_flag_spawns_one_rank_per_gpu(monkeypatch):
    """bench.py --gpus N started as one process relaunches itself under
    torch.distributed.run with N ranks on 127.0.0.1, forwarding its arguments."""
    seen = {}

    def fake_call(cmd):
        seen["cmd"] = cmd
        return 0

    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench.subprocess, "call", fake_call)
    assert bench.main(["--gpus", "4", "--steps", "3", "--warmup", "3"]) == 0
    cmd = seen["cmd"]
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--nnodes=1" in cmd
    assert cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-7].endswith("bench.py")
    assert cmd[-6:] == ["--gpus", "4", "--steps", "3", "--warmup", "3"]
