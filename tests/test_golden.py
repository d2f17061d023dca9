"""Regression fixtures (tests/golden/, written from the oracle by
tests/golden/make_golden.py): the oracle must still reproduce them bit for bit
(no GPU), and the CUDA path must match them (GPU: scales, codes, rotated
weight codes and int32 accumulators exactly; fp32 outputs bit for bit, the
epilogue's order being fixed)."""
import os
import sys

import numpy as np
import pytest
import torch

sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden"))
import make_golden as G  # noqa: E402

NAMES = sorted(G.CASES)


@pytest.mark.parametrize("name", NAMES)
def test_oracle_reproduces_fixture(name):
    stored = G.read(name)
    fresh = G.compute(name)
    assert sorted(stored) == sorted(fresh)
    for key in stored:
        got = np.asarray(fresh[key])
        want = stored[key]
        if got.dtype == np.float32:
            np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32), err_msg=key)
        else:
            np.testing.assert_array_equal(got.astype(np.int64), want, err_msg=key)


@pytest.mark.gpu
@pytest.mark.parametrize("name", NAMES)
def test_gpu_matches_fixture(name):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_quantized_linear_b200 as pq
    from synth import workloads as W
    stored = G.read(name)
    wl = G.case_workload(name)
    x, w, b = W.generate(wl)
    xd, wd, bd = x.cuda(), w.cuda(), b.cuda()
    if name == "hadamard_w4":
        sp, sn = pq.calibrate_hadamard(xd, wl.kseg)
        qw = pq.quantize_weights(wd, wl.kseg, wl.nseg, bits=4)
        qp, qn = pq.quantize_activations_hadamard(xd, wl.kseg, sp, sn)
        rot = pq.rotate_weights_hadamard(qw)
        y = pq.linear_from_codes_hadamard(qp, qn, qw, rot, sp, sn, bd, out_dtype=torch.float32)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(rot.cpu().numpy(), stored["w_rot"])
    else:
        sp, sn = pq.calibrate(xd, wl.kseg)
        qw = pq.quantize_weights(wd, wl.kseg, wl.nseg, bits=8)
        qp, qn = pq.quantize_activations(xd, wl.kseg, sp, sn)
        y = pq.linear(xd, qw, sp, sn, bd, out_dtype=torch.float32)
        y2 = pq.linear_from_codes(qp, qn, qw, sp, sn, bd, out_dtype=torch.float32)
        acc = pq.linear_accumulators(xd, qw, sp, sn)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(qw.codes.cpu().numpy(), stored["w_codes"])
        np.testing.assert_array_equal(qw.scales.cpu().numpy().view(np.uint32),
                                      stored["w_scales"].view(np.uint32))
        np.testing.assert_array_equal(acc.cpu().numpy(), stored["acc"])
        np.testing.assert_array_equal(y2.cpu().numpy().view(np.uint32), stored["y"].view(np.uint32))
    assert pq.stream_status() == 0
    np.testing.assert_array_equal(sp.cpu().numpy().view(np.uint32), stored["s_pos"].view(np.uint32))
    np.testing.assert_array_equal(sn.cpu().numpy().view(np.uint32), stored["s_neg"].view(np.uint32))
    np.testing.assert_array_equal(qp.cpu().numpy(), stored["q_pos"])
    np.testing.assert_array_equal(qn.cpu().numpy(), stored["q_neg"])
    np.testing.assert_array_equal(y.cpu().numpy().view(np.uint32), stored["y"].view(np.uint32))
