"""Stream order across dependent calls.  The GEMMs from codes are programmatic
dependent launches: their setup may overlap the kernel ahead of them in the
stream, but they must read their codes and scales, and write Y, only after
that kernel has finished.  A chain of dependent calls issued back to back
(eagerly and from one CUDA graph) gives the same bits as the same calls with
a synchronisation between each; small-M layers (stacked rows, whose CTAs may
share SMs with the previous GEMM's, and layers whose k blocks are split over
clusters) and a large-M layer."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_quantized_linear_b200 as pq  # noqa: F401  (fails loudly without the library)
    yield


def _layers(M, dims, seed):
    import post_quantized_linear_b200 as pq
    g = torch.Generator().manual_seed(seed)
    x = torch.nn.functional.silu(torch.randn((M, dims[0]), generator=g)).to(torch.bfloat16).cuda()
    qws = []
    for k, n in zip(dims[:-1], dims[1:]):
        w = (torch.randn((n, k), generator=g) * 0.02).cuda()
        qws.append(pq.quantize_weights(w, [0, k], bits=8))
    torch.cuda.synchronize()
    return x, qws


def _chain(x, qws, sync: bool):
    """x -> [calibrate, codes, GEMM from codes (bf16 out)] per layer."""
    import post_quantized_linear_b200 as pq
    outs = []
    h = x
    for qw in qws:
        kseg = [0, h.shape[1]]
        sp, sn = pq.calibrate(h, kseg)
        if sync:
            torch.cuda.synchronize()
        qp, qn = pq.quantize_activations(h, kseg, sp, sn)
        if sync:
            torch.cuda.synchronize()
        h = pq.linear_from_codes(qp, qn, qw, sp, sn, None)
        if sync:
            torch.cuda.synchronize()
        outs.append(h)
    return outs


@pytest.mark.parametrize("M,dims", [(16, [1024, 1536, 512, 768]), (48, [1024, 1536, 512, 768]),
                                    (300, [1024, 1536, 512, 768]),
                                    # DiT-like widths: the 4608-deep layers split their
                                    # k blocks over clusters at M = 16 (stacked rows),
                                    # 40 (stacked, P = 64) and 100 (two-tile form)
                                    (16, [4608, 1152, 4608, 1152]), (40, [4608, 1152, 4608, 1152]),
                                    (100, [4608, 1152, 4608, 1152])])
def test_dependent_layers_back_to_back(M, dims):
    import post_quantized_linear_b200 as pq
    x, qws = _layers(M, dims, seed=M)
    ref = [y.clone() for y in _chain(x, qws, sync=True)]
    for _ in range(3):
        got = _chain(x, qws, sync=False)
        torch.cuda.synchronize()
        assert pq.stream_status() == 0
        for a, b in zip(got, ref):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # the same chain captured once and replayed
    static = {}

    def body():
        static["out"] = _chain(x, qws, sync=False)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        body()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        body()
    for _ in range(3):
        for y in static["out"]:
            y.fill_(0)
        graph.replay()
        torch.cuda.synchronize()
        for a, b in zip(static["out"], ref):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_two_gemms_write_the_same_output_in_turn():
    """The second GEMM's Y writes land after the first GEMM's (write after
    write through one buffer), and a third call reads the second's Y."""
    import post_quantized_linear_b200 as pq
    M = 16
    x, qws = _layers(M, [1024, 2048], seed=5)
    _, qws2 = _layers(M, [1024, 2048], seed=6)
    kseg = [0, 1024]
    sp, sn = pq.calibrate(x, kseg)
    qp, qn = pq.quantize_activations(x, kseg, sp, sn)
    y_ref2 = pq.linear_from_codes(qp, qn, qws2[0], sp, sn, None)
    torch.cuda.synchronize()
    y = torch.empty_like(y_ref2)
    for _ in range(5):
        pq.linear_from_codes(qp, qn, qws[0], sp, sn, None, out=y)
        pq.linear_from_codes(qp, qn, qws2[0], sp, sn, None, out=y)
        s = y.float().sum()
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    assert torch.equal(y.view(torch.int16), y_ref2.view(torch.int16))
    assert s.item() == y_ref2.float().sum().item()


def test_first_call_of_the_process_inside_graph_capture(tmp_path):
    """A process whose first forward (small M, so the cluster-split choice and
    its one-time device queries run) happens while a CUDA graph is being
    captured: the graph replays to the same bits as an eager call."""
    import subprocess
    import sys
    import os
    script = tmp_path / "first_in_graph.py"
    script.write_text(r'''
import sys, torch
import post_quantized_linear_b200 as pq
M, K, N = 16, 4608, 1152
g = torch.Generator().manual_seed(3)
x = torch.nn.functional.silu(torch.randn((M, K), generator=g)).to(torch.bfloat16).cuda()
w = (torch.randn((N, K), generator=g) * 0.02).cuda()
sp = torch.tensor([0.05], device="cuda"); sn = torch.tensor([0.01], device="cuda")
qw = pq.quantize_weights(w, [0, K], bits=8)
qp, qn = pq.quantize_activations(x, [0, K], sp, sn)
y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
torch.cuda.synchronize()
graph = torch.cuda.CUDAGraph()
with torch.cuda.graph(graph):
    pq.linear_from_codes(qp, qn, qw, sp, sn, out=y)   # the process's first forward
y.zero_()
graph.replay()
torch.cuda.synchronize()
ref = pq.linear_from_codes(qp, qn, qw, sp, sn)
torch.cuda.synchronize()
assert pq.stream_status() == 0
sys.exit(0 if torch.equal(y.view(torch.int16), ref.view(torch.int16)) else 3)
''')
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, PYTHONPATH=root + os.pathsep + os.environ.get("PYTHONPATH", ""))
    res = subprocess.run([sys.executable, str(script)], capture_output=True, text=True, timeout=600,
                         cwd=root, env=env)
    assert res.returncode == 0, res.stdout[-2000:] + res.stderr[-2000:]
