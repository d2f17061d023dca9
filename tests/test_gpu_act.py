"""The activation fused into the combined-code producer, on the GPU against the
oracle (SegQuant, Spanish technical summary 1 and 2.B; Korean technical summary
section 2: the negative tail DualScale keeps comes from the SiLU / GELU in
front of the layer).

Reading: x = act(z) rounded once to bf16.  The kernels evaluate act in fp32 and
fall back to fp64 near bf16 rounding midpoints; the oracle evaluates it in
double and flags the elements whose double lies within 2^-40 of a midpoint.
Codes and scales are compared bit-exact on every element except the flagged
ones (their count is asserted small and printed); the forward from the fused
codes is compared with the oracle's forward on x.

Inputs: random pre-activations at several spreads, plus fp32 pre-activations
chosen (with the oracle) so that act(z) lies within 2^-21 of a bf16 midpoint,
where the kernels' fp32 result cannot decide the rounding and the fp64 path
must run."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import post_quantized_linear_b200 as pq  # noqa: F401  (fails loudly without the library)
    O.build()
    yield


def _near_midpoint_z(act: str, n: int, seed: int) -> np.ndarray:
    """fp32 z whose act(z) (the oracle's double) is within a relative 2^-21 of
    a bf16 rounding midpoint."""
    rng = np.random.default_rng(seed)
    out = []
    while sum(len(o) for o in out) < n:
        z = (rng.standard_normal(1 << 20) * 3).astype(np.float32)
        zd = z.astype(np.float64)
        v = zd / (1 + np.exp(-zd)) if act == "silu" else None
        if v is None:
            from scipy.special import erfc
            v = 0.5 * zd * erfc(-zd / np.sqrt(2.0))
        a = np.abs(v)
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
        q = a / np.exp2(np.maximum(e, -126) - 7)
        near = (np.abs(q - np.floor(q) - 0.5) < q * 2.0 ** -21) & (a > 1e-30)
        out.append(z[near])
    return np.concatenate(out)[:n]


def _z_matrix(act: str, M: int, K: int, dtype: str, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((M, K)).astype(np.float32)
    z[:, : K // 4] *= 4.0                        # a wider spread in the first quarter
    z[M // 2:, K // 2:] *= 0.25
    if dtype == "f32":
        near = _near_midpoint_z(act, 256, seed + 1)
        pos = rng.choice(M * K, len(near), replace=False)
        z.reshape(-1)[pos] = near
        return z
    return ((z.view(np.uint32) >> 16) << 16).view(np.float32)   # bf16 values


def _to_device(z: np.ndarray, dtype: str):
    if dtype == "bf16":
        bits = (z.view(np.uint32) >> 16).astype(np.uint16)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda(), bits
    return torch.from_numpy(np.ascontiguousarray(z)).cuda(), np.ascontiguousarray(z)


@pytest.mark.parametrize("act", ["silu", "gelu"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fused_activation_scales_and_codes_bit_exact(act, dtype):
    import post_quantized_linear_b200 as pq
    kseg = [0, 256, 640]
    z = _z_matrix(act, 300, 640, dtype, seed=3 + (act == "gelu"))
    zd, zo = _to_device(z, dtype)
    sp, sn = pq.calibrate_act(zd, act, kseg)
    c = pq.quantize_activations_combined_act(zd, act, kseg, sp, sn)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    osp, osn = O.calibrate_act(zo, act, kseg)
    np.testing.assert_array_equal(sp.cpu().numpy(), osp)
    np.testing.assert_array_equal(sn.cpu().numpy(), osn)
    oc, flags = O.quantize_activations_combined_act(zo, act, kseg, osp, osn)
    got = c.cpu().numpy()
    print(f"{act} {dtype}: {int(flags.sum())} elements flagged as undecided in double")
    assert flags.sum() <= 2
    np.testing.assert_array_equal(got[~flags], oc[~flags])
    assert (oc < 0).sum() > 0                      # the negative tail is there


@pytest.mark.parametrize("act,out", [("silu", "f32"), ("gelu", "bf16")])
def test_forward_from_fused_codes_matches_oracle(act, out):
    """The combined codes of act(z) through the GEMM from combined codes equal
    the oracle's forward on x = bf16_RN(act(z)) (fp32 out bit-exact)."""
    import post_quantized_linear_b200 as pq
    from parity_util import assert_bf16_within_1ulp, bf16_bits
    kseg = [0, 256, 640]
    M, K, N = 300, 640, 400
    z = _z_matrix(act, M, K, "bf16", seed=11)
    zd, zo = _to_device(z, "bf16")
    g = torch.Generator().manual_seed(5)
    w = torch.randn((N, K), generator=g) * 0.02
    b = torch.randn(N, generator=g) * 0.01
    qw = pq.quantize_weights(w.cuda(), kseg, bits=8)
    sp, sn = pq.calibrate_act(zd, act, kseg)
    c = pq.quantize_activations_combined_act(zd, act, kseg, sp, sn)
    odt = torch.float32 if out == "f32" else torch.bfloat16
    y = pq.linear_from_combined(c, qw, sp, sn, b.cuda(), out_dtype=odt)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    x, flags = O.activation_bf16(zo, act)
    assert not flags.any()
    osp, osn = O.calibrate(x, kseg)
    wc, ws = O.quantize_weights_w8(w.numpy(), kseg)
    y_ref = O.linear_forward(x, kseg, osp, osn, 8, wc, ws, b.numpy(), out=out)
    if out == "f32":
        np.testing.assert_array_equal(y.cpu().numpy(), y_ref)
    else:
        assert_bf16_within_1ulp(bf16_bits(y), y_ref)


@pytest.mark.parametrize("name,act", [("dit_xl2_fc2_cfg", "gelu"), ("w4a8", "silu")])
def test_fused_activation_full_size_every_element(name, act):
    """The DiT fc2 input (GELU, 8192 x 4608) and the W4A8 input (SiLU, 16384 x
    3072) as bf16 pre-activations: scales and every code against the oracle."""
    import post_quantized_linear_b200 as pq
    wl = W.WORKLOADS[name]
    g = torch.Generator().manual_seed(wl.seed)
    zt = torch.randn((wl.M, wl.K), generator=g).to(torch.bfloat16)
    zd = zt.cuda()
    zo = zt.view(torch.int16).numpy().view(np.uint16)
    calib = zd if wl.calib_rows is None else zd[: wl.calib_rows]
    sp, sn = pq.calibrate_act(calib, act, wl.kseg)
    c = pq.quantize_activations_combined_act(zd, act, wl.kseg, sp, sn)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    ocal = zo if wl.calib_rows is None else zo[: wl.calib_rows]
    osp, osn = O.calibrate_act(ocal, act, wl.kseg)
    np.testing.assert_array_equal(sp.cpu().numpy(), osp)
    np.testing.assert_array_equal(sn.cpu().numpy(), osn)
    got = c.cpu().numpy()
    flagged = 0
    for r0 in range(0, wl.M, 4096):
        oc, flags = O.quantize_activations_combined_act(zo[r0:r0 + 4096], act, wl.kseg, osp, osn)
        flagged += int(flags.sum())
        part = got[r0:r0 + 4096]
        np.testing.assert_array_equal(part[~flags], oc[~flags])
    print(f"{name} {act}: {flagged} elements flagged as undecided in double")
    assert flagged <= 4


@pytest.mark.parametrize("act", ["silu", "gelu"])
def test_table_and_direct_paths_agree_on_every_bf16_input(act):
    """bf16 pre-activations go through the activation table, fp32 ones through
    the direct evaluation: on all 65536 bf16 patterns (non-finite ones replaced
    by zero) both give the oracle's codes."""
    import post_quantized_linear_b200 as pq
    bits = np.arange(65536, dtype=np.uint32)
    finite = ((bits >> 7) & 0xFF) != 0xFF
    bits = np.where(finite, bits, 0).astype(np.uint16).reshape(64, 1024)
    z32 = (bits.astype(np.uint32) << 16).view(np.float32)
    kseg = [0, 512, 1024]
    osp = np.float32([2.0 ** -3, 0.0371])
    osn = np.float32([2.0 ** -5, 0.0113])
    sp, sn = torch.from_numpy(osp).cuda(), torch.from_numpy(osn).cuda()
    zb = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    c_tab = pq.quantize_activations_combined_act(zb, act, kseg, sp, sn)
    c_dir = pq.quantize_activations_combined_act(torch.from_numpy(z32).cuda(), act, kseg, sp, sn)
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    oc, flags = O.quantize_activations_combined_act(bits, act, kseg, osp, osn)
    # Only |z| < 2^-125 can be undecided: act(z) = z/2 + O(z^2) there, z/2 falls
    # in bf16's subnormal range where it is a rounding midpoint for half of
    # them, and the O(z^2) term lies far below double precision; every flagged
    # element must be one of those.
    tiny = np.abs(z32) < 2.0 ** -125
    assert not flags[~tiny].any()
    np.testing.assert_array_equal(c_tab.cpu().numpy()[~flags], oc[~flags])
    np.testing.assert_array_equal(c_dir.cpu().numpy()[~flags], oc[~flags])


@pytest.mark.parametrize("act", ["silu", "gelu"])
def test_fused_activation_k_not_a_multiple_of_128(act):
    """K = 208 (a multiple of 16 only): the last block of 128 columns is
    partial; bf16 pre-activations through the code table, every code against
    the oracle, and nothing written past K."""
    import post_quantized_linear_b200 as pq
    M, K = 37, 208
    z = _z_matrix(act, M, K, "bf16", seed=21)
    zd, zo = _to_device(z, "bf16")
    kseg = [0, K]
    sp, sn = pq.calibrate_act(zd, act, kseg)
    out = torch.full((M, 224), 55, dtype=torch.int8, device="cuda")
    c = pq.quantize_activations_combined_act(zd, act, kseg, sp, sn, out=out[:, :K])
    torch.cuda.synchronize()
    assert pq.stream_status() == 0
    osp, osn = O.calibrate_act(zo, act, kseg)
    oc, flags = O.quantize_activations_combined_act(zo, act, kseg, osp, osn)
    assert not flags.any()
    np.testing.assert_array_equal(c.cpu().numpy(), oc)
    assert (out[:, K:].cpu().numpy() == 55).all()
