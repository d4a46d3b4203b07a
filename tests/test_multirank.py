"""The bench's multi-rank plumbing on CPU: two gloo ranks.

`bench.py --gpus N` runs one independent replica per GPU (weak scaling, no
collective on the data path). The ranks meet only to take the slowest rank's
time. These tests run that reduction, the whole-job throughput and the
per-rank seeding with two gloo processes on 127.0.0.1, plus the reference
arm's rule that only rank 0 runs.
"""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import kv_synth  # noqa: E402


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench._max_over_ranks(dist, torch.device("cpu"), times[rank])
        data_seed, sign_seed = bench.rank_seeds(rank)
        w = kv_synth.WORKLOADS["tiny_d64"]
        signs = kv_synth.rademacher_signs(1, w.H, w.d, seed=sign_seed)
        t = torch.from_numpy(signs.astype("float32")).reshape(-1)
        gathered = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(gathered, t)
        out.put((rank, ms, data_seed, [g.tolist() for g in gathered]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_code_their_own_caches():
    world, port = 2, _free_port()
    times = [3.25, 7.5]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the max over ranks
    assert [r[1] for r in res] == [max(times)] * world
    # distinct data and sign seeds per replica
    assert res[0][2] != res[1][2]
    assert res[0][3][0] != res[0][3][1]
    # whole-job throughput counts every rank's bytes over the slowest time
    gbps = bench.job_gbps(1e9, 10, world, max(times))
    assert gbps == pytest.approx(1e9 * 10 * world / (max(times) / 1e3) / 1e9)
    assert gbps < bench.job_gbps(1e9, 10, world, min(times))


def test_single_rank_reduction_is_the_identity():
    assert bench._max_over_ranks(None, torch.device("cpu"), 4.5) == 4.5


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = bench.parse_args(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_end_to_end_chunks_cover_every_slice_once():
    for target in (1, 8, 28, 56, 200):
        for n in (1, 2, 3, 4, 7, 8, 9, 28, 56, 64, 100):
            chunks = bench.e2e_chunks(n, target)
            assert len(chunks) == min(target, n)
            covered = [s for a, b in chunks for s in range(a, b)]
            assert covered == list(range(n))
            assert all(b > a for a, b in chunks)
            sizes = [b - a for a, b in chunks]
            assert max(sizes) - min(sizes) <= 1   # balanced
    # the Qwen-shaped cache (56 slices) at the default: 28 chunks of 2 slices
    assert bench.e2e_chunks(56, 28) == [(2 * i, 2 * i + 2) for i in range(28)]
