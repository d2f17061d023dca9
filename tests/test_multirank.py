"""Token-sharded calibration across ranks (gloo, world size 2, CPU).

Each rank calibrates its own rows (with the oracle, on the CPU), the scales are
all-reduced with MAX by the product helper, and the result must equal the
oracle's calibration over all rows bit for bit (fp32 rounding is monotone);
the same for the scales of the block-Hadamard-transformed rows."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle as O
        from post_quantized_linear_b200.parallel import allreduce_scales_, shard_rows
        from synth import workloads as W
        wl = W.small_case(203, 512, 64, seed=5, kseg=[0, 256, 512], x_sigmas=[1.0, 7.0],
                          x_dtype="bf16")
        x, _, _ = W.generate(wl)
        xn = W.to_numpy_x(x)
        r0, r1 = shard_rows(wl.M, rank, world)
        sp, sn = O.calibrate(np.ascontiguousarray(xn[r0:r1]), wl.kseg)
        tp, tn = torch.from_numpy(sp.copy()), torch.from_numpy(sn.copy())
        allreduce_scales_(tp, tn)
        np.save(os.path.join(result_dir, f"r{rank}.npy"), np.stack([tp.numpy(), tn.numpy()]))
        # the block-Hadamard variant: scales of this rank's rows of XH
        hp, hn = O.calibrate_hadamard(np.ascontiguousarray(xn[r0:r1]), wl.kseg)
        tp, tn = torch.from_numpy(hp.copy()), torch.from_numpy(hn.copy())
        allreduce_scales_(tp, tn)
        np.save(os.path.join(result_dir, f"h{rank}.npy"), np.stack([tp.numpy(), tn.numpy()]))
    finally:
        dist.destroy_process_group()


def test_sharded_calibration_equals_full_calibration(tmp_path):
    world = 2
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    import oracle as O
    from synth import workloads as W
    wl = W.small_case(203, 512, 64, seed=5, kseg=[0, 256, 512], x_sigmas=[1.0, 7.0],
                      x_dtype="bf16")
    x, _, _ = W.generate(wl)
    sp, sn = O.calibrate(W.to_numpy_x(x), wl.kseg)
    hp, hn = O.calibrate_hadamard(W.to_numpy_x(x), wl.kseg)
    for r in range(world):
        got = np.load(tmp_path / f"r{r}.npy")
        np.testing.assert_array_equal(got[0], sp)
        np.testing.assert_array_equal(got[1], sn)
        goth = np.load(tmp_path / f"h{r}.npy")
        np.testing.assert_array_equal(goth[0], hp)
        np.testing.assert_array_equal(goth[1], hn)


@pytest.mark.parametrize("M,world", [(10, 3), (8192, 8), (5, 8), (1, 2)])
def test_shard_rows_partition(M, world):
    from post_quantized_linear_b200.parallel import shard_rows
    spans = [shard_rows(M, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == M
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0 and a1 >= a0
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1
