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
