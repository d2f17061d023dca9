"""Small M with stacked polarities: one row tile of M <= 64 rows puts its q+
code rows in rows [0, P) and its q- rows in rows [P, 2P) of one A tile
(P = 16, 32 or 64), so one tcgen05 MMA per k step yields both DualScale
products (SegQuant DualScale, Spanish technical summary 2.B: two int8
products per unit, folded in the epilogue).  The q- accumulators reach the
folding warps by a shuffle (P = 16) or through shared memory (P = 32, 64).

Checked against the oracle (fp32 outputs bit-exact, bf16 within one ulp,
every row), and bit for bit against the two-tile form (the development
build's SEGQUANT_STACK=0) at every narrow tile width, including a ragged
last tile column.  At M <= 16 with few N tiles the K range of a tile is
split over a cluster of CTAs; that form is checked the same way."""
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


@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("M", [1, 15, 16, 17, 32, 33, 63, 64])
def test_stacked_rows_against_oracle_and_two_tile_form(M, out, monkeypatch, dev_lib):
    import post_quantized_linear_b200 as pq
    K, N = 1152, 400                      # nine k blocks, N = 400: ragged at every width
    c = Case(W.small_case(M, K, N, seed=300 + M, out=out))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    res = {}
    for stack in ("1", "0"):
        monkeypatch.setenv("SEGQUANT_STACK", stack)
        for bn in ("32", "64", "96", "128"):
            monkeypatch.setenv("SEGQUANT_BN_SMALL", bn)
            res[(stack, bn)] = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b,
                                                    out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(res[("1", "96")], np.arange(M))
    if out == "f32":
        y_ref, _ = c.oracle_rows(np.arange(M))
        np.testing.assert_array_equal(res[("1", "96")].cpu().numpy(), y_ref)
    iv = torch.int32 if out == "f32" else torch.int16
    ref = res[("0", "96")].view(iv)
    for key, y in res.items():
        assert torch.equal(y.view(iv), ref), key


@pytest.mark.parametrize("M", [16, 64])
def test_stacked_product_library_full_weight(M):
    """The product library's default path (stacked at M <= 64) on the
    (K, N) = (3072, 12288) weight the bench streams: every row against the
    oracle."""
    import post_quantized_linear_b200 as pq
    c = Case(W.small_case(M, 3072, 12288, seed=7, act="silu", bias=False, out="bf16"))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    y = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, None)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(y, np.arange(M))


@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("M", [1, 16, 17, 33, 64, 65, 100, 128])
@pytest.mark.parametrize("K,N", [(1152, 1152), (4608, 1152), (1152, 400), (3072, 2048),
                                 (3072, 12288)])
def test_k_split_over_a_cluster(K, N, M, out, monkeypatch, dev_lib):
    """One row tile (M <= 128): each N tile's k blocks are shared evenly by the
    CTAs of a cluster (2 to 8; 9 k blocks over 4 CTAs gives 2, 2, 2, 3), which
    add their int32 accumulators (every warp its lanes: of the stacked q+ and
    q- rows at M <= 64, of both accumulators of the two-tile form above) into
    the first CTA's shared memory before it folds.
    Integer sums, so the result is bit-identical to one CTA per tile (the
    development build's SEGQUANT_CSPLIT=0) at every tile width -- the widths
    fixed here and the library's own choice ("0": up to 256 columns) -- and
    fp32 outputs equal the oracle's."""
    import post_quantized_linear_b200 as pq
    c = Case(W.small_case(M, K, N, seed=900 + M + K // 128, out=out))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    res = {}
    for split in ("1", "0"):
        monkeypatch.setenv("SEGQUANT_CSPLIT", split)
        for bn in ("32", "64", "128", "0"):
            monkeypatch.setenv("SEGQUANT_BN_SMALL", bn)
            res[(split, bn)] = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b,
                                                    out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    c.compare_rows(res[("1", "32")], np.arange(M))
    if out == "f32":
        y_ref, _ = c.oracle_rows(np.arange(M))
        np.testing.assert_array_equal(res[("1", "32")].cpu().numpy(), y_ref)
    iv = torch.int32 if out == "f32" else torch.int16
    ref = res[("0", "32")].view(iv)
    for key, y in res.items():
        assert torch.equal(y.view(iv), ref), key


@pytest.mark.parametrize("layout", ["neg_below", "neg_far_above"])
@pytest.mark.parametrize("M,K", [(16, 1152), (40, 1152), (16, 1040), (48, 1152), (64, 3072)])
def test_code_boxes_follow_the_buffers(M, K, layout):
    """Stacked rows come in groups of 16 (each group's q+ rows, then its q-
    rows).  One box of a 4-D map brings the whole groups of both polarities
    for a k block and a 3-D map over all M rows the partial last group (M =
    40: two whole groups and 8 rows); both maps start at the lower of the two
    code tensors, so with q- below q+ each group's q- rows come first and the
    fold swaps the halves.  Codes written into one buffer with q- in its first
    half (below q+), or far above q+, K = 1040 (a partial last k block): every
    row against the oracle (fp32 out, bit-exact)."""
    import post_quantized_linear_b200 as pq
    N = 400
    c = Case(W.small_case(M, K, N, seed=77 + M + K, out="f32"))
    ldq = (K + 15) // 16 * 16
    gap = 1 if layout == "neg_below" else 4096
    buf = torch.zeros(((1 + gap) * M, ldq), dtype=torch.int8, device="cuda")
    if layout == "neg_below":
        qn, qp = buf[:M, :K], buf[M:, :K]
    else:
        qp, qn = buf[:M, :K], buf[gap * M:, :K]
    pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn, out=(qp, qn))
    y = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    y_ref, _ = c.oracle_rows(np.arange(M))
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref)


@pytest.mark.parametrize("M", [16, 100])
def test_k_split_starved_pipeline_times_out_and_context_recovers(M, dev_lib):
    """(K, N) = (4608, 1152) splits each N tile's k blocks over a cluster (M =
    16: stacked rows; M = 100: the two-tile form).  With the producer starved
    (development build) every CTA gives up on a bounded wait; the CTAs of rank
    > 0 still send their slices and rank 0 waits for them before the cluster
    leaves, so the call ends with a timeout status, and the next call on the
    same context gives the oracle's rows."""
    import post_quantized_linear_b200 as pq
    from post_quantized_linear_b200 import _lib
    c = Case(W.small_case(M, 4608, 1152, seed=40 + M, out="f32"))
    qp, qn = pq.quantize_activations(c.x, c.wl.kseg, c.sp, c.sn)
    torch.cuda.synchronize()
    assert pq.stream_status() == _lib.SQ_OK
    pq.set_wait_budget(2_000_000)
    pq.debug_starve_pipeline(True)
    try:
        pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
        assert pq.stream_status() == _lib.SQ_ERR_TIMEOUT
    finally:
        pq.debug_starve_pipeline(False)
        pq.set_wait_budget(0)
    y = pq.linear_from_codes(qp, qn, c.qw, c.sp, c.sn, c.b, out_dtype=c.out_dtype)
    torch.cuda.synchronize()
    assert pq.stream_status() == _lib.SQ_OK
    y_ref, _ = c.oracle_rows(np.arange(M))
    np.testing.assert_array_equal(y.cpu().numpy(), y_ref)
