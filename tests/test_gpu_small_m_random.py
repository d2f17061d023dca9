"""Small M over seeded random shapes: every path a one-row-tile GEMM from codes
can take -- stacked rows in groups of 16 (whole groups in one 4-D box, a
partial group from a 3-D map, either code tensor first in memory), the two-tile
form above 64 rows, each with or without its k blocks split over a cluster of
CTAs -- against the oracle, fp32 outputs bit-exact, every row.  Shapes: M in
1..128, K a multiple of 16 (not always of 128), N a multiple of 16."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import workloads as W

from parity_util import Case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_quantized_linear_b200 as pq  # noqa: F401  (fails loudly without the library)
    O.build()
    yield


def _shapes(n=24, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        M = int(rng.integers(1, 129))
        K = int(rng.choice([int(rng.integers(8, 300)) * 16, int(rng.integers(2, 40)) * 128]))
        N = int(rng.integers(2, 200)) * 16
        out.append((i, M, K, N, bool(rng.integers(0, 2))))
    return out


@pytest.mark.parametrize("i,M,K,N,neg_below", _shapes())
def test_small_m_random_shapes(i, M, K, N, neg_below):
    import post_quantized_linear_b200 as pq
    c = Case(W.small_case(M, K, N, seed=5000 + i, out="f32"))
    ldq = (K + 15) // 16 * 16
    buf = torch.zeros((2 * M, ldq), dtype=torch.int8, device="cuda")
    lo, hi = buf[:M, :K], buf[M:, :K]
    qp, qn = (hi, lo) if neg_below else (lo, hi)
    pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn, out=(qp, qn))
    y = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    y_ref, _ = c.oracle_rows(np.arange(M))
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref)
