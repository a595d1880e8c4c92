"""CPU checks of bench.py: the data-parallel plumbing (gradient all-reduce,
max-over-ranks timing, barrier) on two gloo ranks, and the JSON contract of
the oracle arm (--impl reference) on a small workload."""
import datetime
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    flat = torch.full((17,), float(rank + 1))
    bench.allreduce_grads(flat)
    # overlapped form: several tensors started back to back, then waited for
    parts = [torch.full((5,), float(rank + 1)), torch.full((3,), 10.0 * (rank + 1))]
    bench.allreduce_finish([bench.allreduce_start(t) for t in parts])
    assert parts[0].tolist() == [3.0] * 5 and parts[1].tolist() == [30.0] * 3
    slowest = bench.reduce_max(10.0 * rank + 1.5, torch.device("cpu"))
    bench.barrier(torch.device("cpu"))
    out.put((rank, flat.tolist(), slowest))
    dist.destroy_process_group()


def test_two_rank_gradient_allreduce_and_max_timing():
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
    for rank, flat, slowest in res:
        assert flat == [3.0] * 17          # sum of 1 and 2 on every rank
        assert slowest == 11.5            # max over ranks of the per-rank times


def _dp_worker(rank, world, port, out):
    """Rank `rank` holds token rows rank::world of one small layer: it takes
    the oracle's dG of its rows, sums dG across ranks with the bench's
    overlapped all-reduce, and turns the sum into dq with the oracle's CNP
    backward."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import oracle
    import poetx_inputs as pi
    inp = pi.layer_inputs(pi.CONFIGS["attn3b"], 0, T=50, m=128, n=192, b=64, sigma_q=0.03)
    rows = np.arange(rank, inp.T, world)
    GR, GP = oracle.cnp_blocks(inp.qR, inp.b), oracle.cnp_blocks(inp.qP, inp.b)
    _, dGR, dGP = oracle.backward(inp.x64[rows], inp.W0lin64.T, inp.permR, GR, inp.permP, GP, inp.dz64[rows])
    flat = torch.from_numpy(np.concatenate([dGR.ravel(), dGP.ravel()]))
    half = dGR.size
    parts = [flat[:half], flat[half:]]          # one exchange per side, started back to back
    bench.allreduce_finish([bench.allreduce_start(t) for t in parts])
    dG = flat.numpy()
    dqR = oracle.cnp_backward(inp.qR, inp.b, dG[:half].reshape(dGR.shape))
    dqP = oracle.cnp_backward(inp.qP, inp.b, dG[half:].reshape(dGP.shape))
    out.put((rank, dqR, dqP))
    dist.destroy_process_group()


def test_data_parallel_dG_sum_gives_the_all_token_dq():
    """The data-parallel exchange of the bench: the CNP backward is linear in
    dG and dG is a sum over tokens, so summing the per-rank dG (token rows
    split across two ranks) and then running the CNP backward gives the dq of
    all tokens on one rank."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    import poetx_inputs as pi
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dp_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = pi.layer_inputs(pi.CONFIGS["attn3b"], 0, T=50, m=128, n=192, b=64, sigma_q=0.03)
    _, dqR, dqP = oracle.layer_backward(inp.x64, inp.W0lin64.T, inp.permR, inp.qR, inp.permP, inp.qP, inp.b,
                                        inp.dz64)
    for _, gR, gP in res:
        np.testing.assert_allclose(gR, dqR, rtol=1e-11, atol=1e-12 * np.abs(dqR).max())
        np.testing.assert_allclose(gP, dqP, rtol=1e-11, atol=1e-12 * np.abs(dqP).max())


def test_reference_arm_json_contract():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny", "--steps", "2", "--warmup", "3", "--ref-tokens", "16"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["value"] > 0 and line["higher_is_better"] is True
    assert line["steps"] == 2 and line["warmup"] == 3
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    import poetx_inputs as pi
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        ref_tokens, warmup, steps = 4, 3, 1

    assert bench.bench_reference(A, pi.CONFIGS["tiny"]) is None


def test_bench_rejects_short_warmup():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--warmup", "2"],
                         capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0


def test_clock_samples_inside_timed_region():
    # only samples stamped inside [t_begin, t_end] count as under load
    import datetime
    import bench

    def line(sec, mhz, power, cap="Not Active"):
        ts = datetime.datetime(2026, 1, 1, 12, 0, 0) + datetime.timedelta(seconds=sec)
        stamp = ts.strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{stamp}, 0, {mhz}, 1965, {power}, 0x0, Not Active, Not Active, Not Active, {cap}"

    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0).timestamp()
    lines = [line(0.0, 1965, 150.0), line(0.1, 1965, 160.0), line(0.5, 1300, 990.0, "Active"),
             line(0.55, 1320, 1000.0, "Active"), line(0.6, 1310, 980.0), line(1.5, 1965, 200.0)]
    rec = bench.ClockSampler.parse(lines, t0 + 0.45, t0 + 0.65)
    assert rec["samples"] == 3 and rec["samples_total"] == 6
    assert rec["sm_mhz"] == 1310 and rec["sm_mhz_min"] == 1300
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["power_w_max"] == 1000.0
    # no window given: every sample counts
    rec = bench.ClockSampler.parse(lines)
    assert rec["samples"] == 6 and rec["window"] == "all samples"
    # malformed lines are skipped
    assert bench.ClockSampler.parse(["garbage", ""])["samples"] == 0
