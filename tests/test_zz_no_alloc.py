"""The allocation-free split-K entry point (library-owned static scratch),
called through the C ABI.  It serves callers that cannot allocate device
memory while they run: an inference loop that forbids allocation after
start-up, or a process whose device memory is held by another allocator.

Checks, on two calls in a row: the same bits as the split-K entry point with a
caller workspace and as the one-pass GEMM from codes; the oracle's result
(fp32 bit-exact, bf16 within one ulp); and no device memory allocated by the
call (torch's allocator and the device's free memory unchanged across it).
Collected last; passes alone in a fresh process and after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from synth import workloads as W

from parity_util import assert_bf16_within_1ulp, bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield


def _bits(y):
    return y.view(torch.int16) if y.dtype == torch.bfloat16 else y.view(torch.int32)


def _static_call(qp, qn, qw, sp, sn, bias, y):
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    cw, keep = qw.c_struct()
    st = _lib.load().sq_linear_forward_codes_splitk_static(
        ctypes.c_void_p(qp.data_ptr()), ctypes.c_void_p(qn.data_ptr()), qp.stride(0), qp.shape[0],
        qp.shape[1], ctypes.byref(cw), ctypes.c_void_p(sp.data_ptr()), ctypes.c_void_p(sn.data_ptr()),
        None if bias is None else ctypes.c_void_p(bias.data_ptr()), ctypes.c_void_p(y.data_ptr()),
        _lib.SQ_BF16 if y.dtype == torch.bfloat16 else _lib.SQ_F32, y.stride(0), None)
    return st


@pytest.mark.parametrize("M,K,N,out", [(64, 3072, 4096, "bf16"), (100, 1024, 400, "f32"),
                                       (1, 256, 128, "bf16")])
def test_static_scratch_splitk_matches_existing_entry_points(M, K, N, out):
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    wl = W.small_case(M, K, N, seed=170 + M, out=out)
    x, w, b = W.generate(wl)
    dev = torch.device("cuda", 0)
    xd, wd, bd = x.to(dev), w.to(dev), b.to(dev)
    sp, sn = pq.calibrate(xd, wl.kseg)
    qw = pq.quantize_weights(wd, wl.kseg, wl.nseg, bits=8)
    qp, qn = pq.quantize_activations(xd, wl.kseg, sp, sn)
    odt = torch.float32 if out == "f32" else torch.bfloat16
    ws = pq.splitk_workspace(M, N, K, device=dev)
    ref_ws = pq.linear_from_codes_splitk(qp, qn, qw, sp, sn, ws, bd, out_dtype=odt)
    ref = pq.linear_from_codes(qp, qn, qw, sp, sn, bd, out_dtype=odt)
    O.build()
    xn = W.to_numpy_x(x)
    o_sp, o_sn = O.calibrate(xn, wl.kseg)
    o_wc, o_ws = O.quantize_weights_w8(w.numpy(), wl.kseg)
    y_ref = O.linear_forward(xn, wl.kseg, o_sp, o_sn, 8, o_wc, o_ws, b.numpy(), out=out)
    for call in range(2):                   # two calls in a row share the scratch
        y = torch.full((M, N), 3.0, dtype=odt, device=dev)
        torch.cuda.synchronize()
        torch_before = torch.cuda.memory_allocated(dev)
        free_before = torch.cuda.mem_get_info(dev)[0]
        assert _static_call(qp, qn, qw, sp, sn, bd, y) == _lib.SQ_OK
        torch.cuda.synchronize()
        if call == 1:                       # the first call may load the library's module
            assert torch.cuda.memory_allocated(dev) == torch_before
            assert torch.cuda.mem_get_info(dev)[0] == free_before
        assert pq.stream_status() == _lib.SQ_OK
        assert torch.equal(_bits(y), _bits(ref_ws))
        assert torch.equal(_bits(y), _bits(ref))
        if out == "f32":
            np.testing.assert_array_equal(y.cpu().numpy(), y_ref)
        else:
            assert_bf16_within_1ulp(bf16_bits(y), y_ref)


def test_static_scratch_rejects_sizes_beyond_the_maximum():
    """8 * M * N bytes of partial sums (one K split) above 16 MiB: SQ_ERR_RANGE,
    reported before any launch."""
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    M, K, N = 128, 256, 17408              # 128 * 17408 * 8 = 17.8 MB > 16 MiB
    dev = torch.device("cuda", 0)
    qp = torch.zeros((M, K), dtype=torch.int8, device=dev)
    w = torch.zeros((N, K), dtype=torch.float32, device=dev)
    qw = pq.quantize_weights(w, [0, K], bits=8)
    s = torch.ones(1, dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    assert _static_call(qp, qp, qw, s, s, None, y) == _lib.SQ_ERR_RANGE
    torch.cuda.synchronize()
