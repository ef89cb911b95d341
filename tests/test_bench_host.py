"""Host-side logic of bench.py without a GPU: algorithmic work formulas and
the multi-rank aggregation (world size 2 over gloo)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def test_algorithmic_work_matches_the_stated_figures():
    # 6.7B-class layer at 8k, chunk 512, no state in or out
    F = bench.chunkwise_flops(8, 16, 8192, 256, 512, 512)
    assert abs(F - 9.285e11) / 9.285e11 < 1e-3
    # exact count: no inter term in chunk 0, no state update after the last chunk
    assert F / (8 * 16 * 8192) == 885504          # per token-head
    assert bench.chunkwise_bytes(8, 16, 8192, 256, 512) == 3 * 2 ** 30
    # 1.3B-class layer: chunkwise C=128 and the parallel form
    assert abs(bench.chunkwise_flops(8, 8, 2048, 256, 256, 128) - 4.09e10) / 4.09e10 < 2e-3
    assert abs(bench.parallel_flops(8, 8, 2048, 256, 256) - 1.375e11) / 1.375e11 < 1e-3
    # 64k, state returned
    F5 = bench.chunkwise_flops(1, 16, 65536, 256, 512, 512, state_out=True)
    assert abs(F5 - 9.607e11) / 9.607e11 < 1e-3
    # decode step: fp32 state read + write dominates
    assert abs(bench.step_bytes(8, 16, 256, 512) - 134.6e6) / 134.6e6 < 1e-3


def test_ragged_chunks_count_exact_lengths():
    Ls = bench.chunk_lengths(1000, 512)
    assert Ls == [512, 488]
    F = bench.chunkwise_flops(1, 1, 1000, 2, 3, 512, state_in=True, state_out=True)
    assert F == (512 * 513 + 488 * 489) * 5 + 2 * (2 * 2 * 3 * 1000)


def test_phase_split_and_single_chunk_agree_with_the_whole():
    """The two phases' flops add up to the whole call, and one chunk covering
    the sequence (no state in or out) is the parallel form's causal count."""
    for args in ((8, 16, 8192, 256, 512, 512, False, False), (1, 2, 1000, 64, 96, 128, True, True),
                 (2, 3, 77, 8, 16, 37, True, False)):
        st, out = bench.chunkwise_phase_flops(*args)
        assert st + out == bench.chunkwise_flops(*args)
    assert bench.chunkwise_flops(8, 8, 2048, 256, 256, 2048) == \
        bench.parallel_flops(8, 8, 2048, 256, 256)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w = bench.init_dist("gloo")
    try:
        t_local = 0.5 + r          # rank 1 is slower
        bench.barrier()
        t_max = bench.max_over_ranks(t_local)
        out[r] = (t_max, bench.global_throughput(65536, 10, w, t_max))
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


def test_two_ranks_take_the_max_time_and_sum_the_tokens():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1]
    t_max, value = out[0]
    assert t_max == pytest.approx(1.5)
    assert value == pytest.approx(65536 * 10 * 2 / 1.5)


def test_gpus_flag_launches_that_many_ranks_and_sums_their_tokens():
    """`bench.py --gpus 2` outside torchrun re-runs itself as two ranks; rank 0
    prints n_gpus = 2, the max time over the ranks and both ranks' tokens."""
    import json
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items()
           if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2",
                        "--steps", "10", "--warmup", "3", "--plumbing-check"],
                       capture_output=True, text=True, timeout=240, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout          # rank 0 alone prints
    line = lines[0]
    assert line["n_gpus"] == 2 and line["gpus_requested"] == 2
    assert line["t_max_s"] == pytest.approx(1.5)
    assert line["value"] == pytest.approx(8 * 8192 * 10 * 2 / 1.5)


def test_rank_launch_command_uses_torchrun_on_loopback():
    cmd = bench.rank_launch_command(4, ["--gpus", "4", "--steps", "5"], 29555)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert "--master-port=29555" in cmd and cmd[-4:] == ["--gpus", "4", "--steps", "5"]
