"""bench.py's multi-rank logic on the CPU with gloo, world size 2: the timed
figure is the slowest rank's, the value is every rank's work over that time,
and the reference arm runs on rank 0 only."""

import datetime
import io
import os
import socket
import sys
import contextlib

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"), world)
        q.put((rank, ms, bench.whole_job_value(world, 2e12, ms)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [15.0, 15.0]
    want = 2 * 2e12 / 15e-3 / 1e12  # both ranks' work over the slower rank's time
    assert all(abs(r[2] - want) < 1e-9 * want for r in res)


def test_single_rank_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu"), 1) == 3.5


def test_reference_arm_is_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    from mixed_precision_block_b200.synth import WORKLOADS
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(None, WORKLOADS["video"])  # returns before touching its arguments
    assert buf.getvalue() == ""


def test_roofline_follows_the_phase_floors_and_prep_bytes():
    sys.path.insert(0, ROOT)
    import bench
    from types import SimpleNamespace
    from mixed_precision_block_b200.synth import WORKLOADS
    pk = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    wl = WORKLOADS["video"]  # 24 heads, d = 128, 118,800 tokens, 1980 regions
    # the survey's worked figure for the headline budget: 3.46 GB of prep traffic
    info = SimpleNamespace(n16=294030, n8=294030, n4=0, nb=1980)
    assert abs(bench.prep_bytes(wl, info) / 1e9 - 3.46) < 0.01
    # phase floors: 16-bit at the burst bf16 peak, INT8 at twice it, NVFP4 at four times
    info = SimpleNamespace(n16=1000, n8=2000, n4=4000, nb=1980)
    r = bench.roofline(wl, info, 2.0, 4.0, pk, "measured", 1965.0)
    per_pair = 4 * 64 * 64 * 128 * 24
    t_tensor = (1000 * per_pair / 1.6e15 + 2000 * per_pair / 3.2e15 + 4000 * per_pair / 6.4e15) * 1e3
    assert abs(r["floor_ms"]["tensor"] - t_tensor) < 1e-12
    assert abs(r["frac"] - t_tensor / 2.0) < 1e-12  # achieved / phase-weighted peak = floor / time
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-12
    t_prep = bench.prep_bytes(wl, info) / 6.5e12 * 1e3
    assert abs(r["whole_call"]["frac"] - (t_tensor + t_prep) / 4.0) < 1e-12
    # the XU floor is reported beside it, not as the bound
    t_xu = 24 * (1000 * 6144 + 2000 * 4096 + 4000 * 4096 * (1.5 + 1 / 16)) / (16 * 148 * 1965e6) * 1e3
    assert r["bound"] == "tensor" and abs(r["xu_floor_ms"] - t_xu) < 1e-9
