"""The bench's multi-rank orchestration on CPU ranks (no GPU).

* `--gpus 2` without WORLD_SIZE starts two ranks through torch.distributed.run
  (the reference arm, which needs no GPU): rank 0 prints the one JSON line,
  rank 1 exits 0 without output.
* A launch whose WORLD_SIZE differs from --gpus exits non-zero.
* gloo, world size 2: each rank draws its own batch (seed + rank), calibrates
  its calibration rows with the oracle standing in for the GPU kernel, the
  scales are all-reduced with the product helper (MAX), and the step times are
  combined with the bench's max-over-ranks; the scales must equal the oracle's
  calibration over both ranks' rows, the time the slower rank's, and the
  whole-job rate the two ranks' work over that time.
"""
import json
import os
import socket
import subprocess
import sys
import time

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _clean_env(**extra):
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    env.update(OMP_NUM_THREADS="1", **extra)
    return env


def test_two_gpus_flag_starts_two_ranks_and_rank0_prints_one_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--gpus", "2", "--workload", "tiny_w8a8", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, env=_clean_env(), cwd=ROOT)
    assert res.returncode == 0, res.stderr[-3000:]
    lines = [l for l in res.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["config"]["parallelism"] == "dp2"


def test_world_size_mismatch_exits_nonzero():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                          "--impl", "reference", "--workload", "tiny_w8a8", "--steps", "1"],
                         capture_output=True, text=True, timeout=120,
                         env=_clean_env(WORLD_SIZE="3", RANK="0", LOCAL_RANK="0"), cwd=ROOT)
    assert res.returncode == 2
    assert "WORLD_SIZE=3" in res.stderr


def test_relaunch_command_names_the_launcher():
    cmd = bench.relaunch_command(["--gpus", "4", "--steps", "3"], 4, 12345)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "--master-addr=127.0.0.1" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle as O
        from post_quantized_linear_b200.parallel import allreduce_scales_
        from synth import workloads as W
        w_, r_, l_ = bench.rank_env()
        assert (w_, r_, l_) == (world, rank, rank)
        wl = W.small_case(96, 256, 64, seed=3, kseg=[0, 128, 256], x_sigmas=[1.0, 6.0])
        wl_r = bench.rank_workload(wl, rank)
        x, _, _ = W.generate(wl_r)
        xn = W.to_numpy_x(x)
        t0 = time.perf_counter()
        sp, sn = O.calibrate(xn, wl.kseg)              # stands in for the GPU calibration
        tp, tn = torch.from_numpy(sp.copy()), torch.from_numpy(sn.copy())
        allreduce_scales_(tp, tn)
        local_ms = (time.perf_counter() - t0) * 1e3 + 10.0 * rank   # rank 1 is the slower one
        got = bench.max_over_ranks([local_ms, float(rank)], world, torch.device("cpu"))
        np.save(os.path.join(out_dir, f"r{rank}.npy"),
                np.concatenate([tp.numpy(), tn.numpy(), np.float32([local_ms]),
                                np.float32(got)]).astype(np.float64))
    finally:
        dist.destroy_process_group()


def test_ranks_draw_own_batches_share_scales_and_time_by_the_slowest(tmp_path):
    import oracle as O
    from synth import workloads as W
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    wl = W.small_case(96, 256, 64, seed=3, kseg=[0, 128, 256], x_sigmas=[1.0, 6.0])
    xs = [W.to_numpy_x(W.generate(bench.rank_workload(wl, r))[0]) for r in range(world)]
    assert not np.array_equal(xs[0], xs[1])                 # independent batches
    sp, sn = O.calibrate(np.concatenate(xs), wl.kseg)       # the union of the ranks' rows
    res = [np.load(tmp_path / f"r{r}.npy") for r in range(world)]
    J = len(wl.kseg) - 1
    for r in range(world):
        np.testing.assert_array_equal(res[r][:J].astype(np.float32), sp)
        np.testing.assert_array_equal(res[r][J:2 * J].astype(np.float32), sn)
    slowest = max(res[r][2 * J] for r in range(world))
    for r in range(world):
        assert res[r][2 * J + 1] == slowest and res[r][2 * J + 2] == world - 1
    ops = wl.exec_ops
    assert bench.whole_job_tops(world, 5, ops, slowest) == world * 5 * ops / (slowest * 1e-3) / 1e12
