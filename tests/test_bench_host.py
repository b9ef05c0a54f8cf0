"""Host logic of bench.py on CPU: the multi-rank path (world size 2 over gloo),
clock parsing and the roofline arithmetic.  No GPU is used."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, local = bench.rank_env()
    # each rank times a different amount of work; the job time is the slowest rank's
    t = bench.max_over_ranks(10.0 + r * 5.0, w)
    W, act, x = bench.make_inputs(bench.rank_seed(r))
    q.put((r, w, local, t, float(W[0, :8].sum()), float(act[:8].sum())))
    dist.barrier()
    dist.destroy_process_group()


def test_two_ranks_gloo_max_and_distinct_shards():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 for r in res)
    assert all(r[3] == 15.0 for r in res)          # max over ranks on every rank
    assert res[0][4] != res[1][4] and res[0][5] != res[1][5]  # each rank its own matrix


def test_world_one_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5


CSV = """index, clocks.current.sm [MHz], clocks.max.sm [MHz], power.draw [W], clocks_event_reasons.active, clocks_event_reasons.hw_slowdown, clocks_event_reasons.hw_thermal_slowdown, clocks_event_reasons.sw_thermal_slowdown, clocks_event_reasons.sw_power_cap
0, 1965 MHz, 1965 MHz, 500.1 W, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active
0, 1800 MHz, 1965 MHz, 990.0 W, 0x0000000000000004, Not Active, Not Active, Not Active, Active
0, 1700 MHz, 1965 MHz, 995.0 W, 0x0000000000000004, Not Active, Not Active, Not Active, Active
0, 345 MHz, 1965 MHz, 120.0 W, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active
"""


def test_parse_clocks():
    c = bench.parse_clocks(CSV)
    assert c["samples"] == 4
    assert c["sm_max_mhz"] == 1965.0
    assert c["sm_mhz"] == 1800.0        # median of the loaded samples (idle 345 dropped)
    assert c["reasons"] == ["sw_power_cap"]
    assert bench.parse_clocks("")["sm_mhz"] is None


def test_roofline_arithmetic():
    ab = bench.algorithmic_bytes(4096, 4096, 11, 1)
    packed = 4096 * 2816
    side = 2 * 4096 + 2 * 2048 + 2 * 4096 + 8 * 2048
    assert ab["decode"] == packed + side + 2 * 4096 * 4096
    assert ab["gemv"] == packed + side + 2 * 4096 + 2 * 4096
    # 16.7M weights at 5.5 bpw: ~11.5 MB of indices
    assert abs(packed / 4096 / 4096 * 8 - 5.5) < 1e-9
    assert bench.fp32_peak_tflops(1965.0) == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)
    pairs = 4096 * 2048
    assert bench.encode_flops(4096, 4096, 128, 5 * pairs) == pytest.approx(pairs * (28 + 20))


def test_bench_cli_rejects_short_warmup():
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])
