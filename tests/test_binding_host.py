"""Host-side behaviour of the Python binding (no GPU): the C view of a
quantized weight is built once and rebuilt when a field it is made of
changes (a call at small M pays for marshalling, not for the kernel)."""
import torch

import post_quantized_linear_b200 as pq


def _qw(N=64, K=256, kseg=(0, 256)):
    return pq.QuantizedWeight(bits=8, N=N, K=K, kseg=tuple(kseg), nseg=(0, N),
                              codes=torch.zeros((N, K), dtype=torch.int8),
                              scales=torch.ones((len(kseg) - 1, N), dtype=torch.float32))


def test_c_struct_is_reused_while_the_weight_is_unchanged():
    qw = _qw()
    c1, _ = qw.c_struct()
    c2, _ = qw.c_struct()
    assert c1 is c2
    assert (c1.bits, c1.N, c1.K) == (8, 64, 256)
    assert c1.codes == qw.codes.data_ptr() and c1.scales == qw.scales.data_ptr()


def test_c_struct_follows_replaced_tensors_and_segments():
    qw = _qw()
    c1, _ = qw.c_struct()
    qw.codes = torch.zeros((64, 256), dtype=torch.int8)
    c2, _ = qw.c_struct()
    assert c2 is not c1 and c2.codes == qw.codes.data_ptr()
    qw.kseg = (0, 128, 256)
    qw.scales = torch.ones((2, 64), dtype=torch.float32)
    c3, _ = qw.c_struct()
    assert c3 is not c2
    assert c3.kseg.count == 2 and [c3.kseg.bounds[i] for i in range(3)] == [0, 128, 256]
