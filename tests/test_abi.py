"""Host-only checks of the C ABI: the library loads, exports every entry point
declared in include/segquant.h, and rejects bad arguments before touching the
GPU (every call below returns during host validation)."""
import ctypes
import os
import re

import pytest

from post_quantized_linear_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "segquant.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_entry_point():
    names = declared_functions()
    assert len(names) >= 9
    for lib in (_lib.load(), _lib.load_dev()):
        for n in names:
            assert hasattr(lib, n), n
            assert n in _lib.SIGNATURES, n


def test_test_hooks_live_only_in_the_development_library():
    """The product library refuses the wait hooks (fixed budget, no starvation
    switch); the development build accepts them."""
    prod, dev = _lib.load(), _lib.load_dev()
    assert prod.sq_set_wait_budget(1000) == _lib.SQ_ERR_UNSUPPORTED
    assert prod.sq_debug_starve_pipeline(1) == _lib.SQ_ERR_UNSUPPORTED
    assert dev.sq_set_wait_budget(0) == _lib.SQ_OK
    assert dev.sq_debug_starve_pipeline(0) == _lib.SQ_OK


def test_product_library_reads_no_environment():
    """No switch of the product build reads the environment: the variable names
    the development build's switches look up are absent from the product
    library's binary, present in the development library's."""
    def has_switch_names(path):
        data = open(path, "rb").read()
        return b"SEGQUANT_BN" in data or b"SEGQUANT_PAIR" in data or b"SEGQUANT_KPS" in data
    assert not has_switch_names(_lib.LIB_PATH)
    assert has_switch_names(_lib.DEV_LIB_PATH)


def test_binding_arity_matches_every_declaration():
    """Each prototype in include/segquant.h takes as many parameters as the
    ctypes signature the binding gives it (guards the two against drift)."""
    src = open(os.path.join(ROOT, "include", "segquant.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    protos = re.findall(r"\b(?:sq_status|const char\s*\*|void)\s+(sq_[a-z_0-9]+)\s*\(([^)]*)\)\s*;",
                        src)
    assert len(protos) == len(declared_functions())
    for name, params in protos:
        params = params.strip()
        n = 0 if params in ("", "void") else len([p for p in params.split(",") if p.strip()])
        assert len(_lib.SIGNATURES[name][1]) == n, name


def test_status_strings():
    assert _lib.status_string(0) == "SQ_OK"
    assert _lib.status_string(6) == "SQ_ERR_TIMEOUT"
    assert _lib.status_string(99) == "SQ_UNKNOWN_STATUS"


def _sizes(bits, N, K, J, group):
    cb, sb = ctypes.c_size_t(), ctypes.c_size_t()
    st = _lib.load().sq_qweight_sizes(bits, N, K, J, group, ctypes.byref(cb), ctypes.byref(sb))
    return st, cb.value, sb.value


def test_qweight_sizes():
    assert _sizes(8, 1152, 4608, 1, 0) == (0, 1152 * 4608, 4 * 1152)
    assert _sizes(8, 3456, 2304, 2, 0) == (0, 3456 * 2304, 2 * 4 * 3456)
    assert _sizes(4, 3072, 3072, 1, 128) == (0, 3072 * 1536, 2 * 3072 * 24)
    assert _sizes(4, 16, 200, 1, 128)[0] == _lib.SQ_ERR_UNSUPPORTED
    assert _sizes(4, 16, 256, 1, 64)[0] == _lib.SQ_ERR_UNSUPPORTED
    assert _sizes(6, 16, 256, 1, 0)[0] == _lib.SQ_ERR_UNSUPPORTED
    assert _sizes(8, 0, 256, 1, 0)[0] == _lib.SQ_ERR_INVALID_ARG
    assert _sizes(8, 16, 256, 17, 0)[0] == _lib.SQ_ERR_UNSUPPORTED


FAKE = 1 << 20          # a 16-byte aligned, never dereferenced address
FAKE_ODD = FAKE + 4     # 4-byte aligned only


def _qw(bits=8, N=256, K=512, kb=(0, 512), nb=None, codes=FAKE, scales=FAKE):
    ks, ka = _lib.segments(kb)
    ns, na = _lib.segments(nb or (0, N))
    qw = _lib.SqQWeight(bits, 0 if bits == 8 else 128, N, K, ks, ns, codes, scales)
    return qw, (ka, na)


def _fwd(x=FAKE, xt=_lib.SQ_BF16, M=256, K=512, ldx=512, qw=None, sp=FAKE, sn=FAKE, bias=None,
         y=FAKE, yt=_lib.SQ_BF16, ldy=256):
    if qw is None:
        qw, keep = _qw(K=K)
    return _lib.load().sq_linear_forward(x, xt, M, K, ldx, ctypes.byref(qw), sp, sn, bias, y, yt,
                                         ldy, None)


def test_forward_validation_rejects_before_launch():
    L = _lib
    assert _fwd(M=-1) == L.SQ_ERR_INVALID_ARG
    assert _fwd(xt=7) == L.SQ_ERR_INVALID_ARG
    assert _fwd(ldx=100) == L.SQ_ERR_INVALID_ARG
    assert _fwd(x=None) == L.SQ_ERR_INVALID_ARG
    assert _fwd(x=FAKE + 8) == L.SQ_ERR_ALIGNMENT
    assert _fwd(y=FAKE + 2) == L.SQ_ERR_ALIGNMENT
    assert _fwd(ldy=260) == L.SQ_ERR_ALIGNMENT       # 520 bytes: not a multiple of 16
    assert _fwd(bias=FAKE_ODD) == L.SQ_ERR_ALIGNMENT
    assert _fwd(sp=FAKE + 2) == L.SQ_ERR_ALIGNMENT
    qw, k = _qw(kb=(0, 200, 512))                     # interior bound not a multiple of 128
    assert _fwd(qw=qw) == L.SQ_ERR_UNSUPPORTED
    qw, k = _qw(kb=(0, 256, 256, 512))                # not increasing
    assert _fwd(qw=qw) == L.SQ_ERR_INVALID_ARG
    qw, k = _qw(kb=(0, 384))                          # does not end at K
    assert _fwd(qw=qw) == L.SQ_ERR_INVALID_ARG
    qw, k = _qw(N=200)                                # N % 16 != 0
    assert _fwd(qw=qw, ldy=200) == L.SQ_ERR_UNSUPPORTED
    qw, k = _qw(nb=(0, 100, 250))                     # output segments must end at N
    assert _fwd(qw=qw) == L.SQ_ERR_INVALID_ARG
    qw, k = _qw(K=512, codes=FAKE + 1)
    assert _fwd(qw=qw) == L.SQ_ERR_ALIGNMENT
    qw, k = _qw(K=256)                                # weight K differs from x K
    assert _fwd(qw=qw) == L.SQ_ERR_INVALID_ARG
    qw, k = _qw(K=262144, kb=(0, 262144))
    assert _fwd(qw=qw, K=262144, ldx=262144) == L.SQ_ERR_RANGE
    many = tuple(range(0, 128 * 18, 128))
    qw, k = _qw(K=128 * 17, kb=many)
    assert _fwd(qw=qw, K=128 * 17, ldx=128 * 17) == L.SQ_ERR_UNSUPPORTED
    assert _fwd(M=0) == L.SQ_OK                       # empty input: no launch, no error


def test_calibrate_and_quantize_validation():
    lib = _lib.load()
    seg, keep = _lib.segments((0, 512))
    bad, keep2 = _lib.segments((0, 100, 512))
    assert lib.sq_calibrate(FAKE, 1, 16, 512, 512, ctypes.byref(bad), FAKE, FAKE, None) == _lib.SQ_ERR_UNSUPPORTED
    assert lib.sq_calibrate(FAKE, 1, -1, 512, 512, ctypes.byref(seg), FAKE, FAKE, None) == _lib.SQ_ERR_INVALID_ARG
    assert lib.sq_calibrate(FAKE, 1, 16, 512, 512, ctypes.byref(seg), None, FAKE, None) == _lib.SQ_ERR_INVALID_ARG
    assert lib.sq_calibrate(FAKE + 8, 1, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, None) == _lib.SQ_ERR_ALIGNMENT
    assert lib.sq_quantize_activations(FAKE, 1, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE,
                                       FAKE, 520, None) == _lib.SQ_ERR_ALIGNMENT
    assert lib.sq_quantize_activations(FAKE, 1, 0, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE,
                                       FAKE, 512, None) == _lib.SQ_OK
    qw, k = _qw(bits=4, K=512)
    qw.N = 128
    assert lib.sq_quantize_weights(FAKE, 0, 256, 512, 512, ctypes.byref(qw), None) == _lib.SQ_ERR_INVALID_ARG
    qw, k = _qw(bits=4, K=500, kb=(0, 500))
    assert lib.sq_quantize_weights(FAKE, 0, 256, 500, 500, ctypes.byref(qw), None) == _lib.SQ_ERR_UNSUPPORTED


def test_combined_code_entry_points_validate_before_launch():
    lib = _lib.load()
    L = _lib
    seg, keep = _lib.segments((0, 512))
    qc = lib.sq_quantize_activations_combined
    assert qc(FAKE, 1, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE, 520, None) == L.SQ_ERR_ALIGNMENT
    assert qc(FAKE, 1, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, None, 512, None) == L.SQ_ERR_INVALID_ARG
    assert qc(FAKE, 1, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE, 256, None) == L.SQ_ERR_INVALID_ARG
    assert qc(FAKE, 1, 0, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE, 512, None) == L.SQ_OK
    bad, keep2 = _lib.segments((0, 100, 512))
    assert qc(FAKE, 1, 16, 512, 512, ctypes.byref(bad), FAKE, FAKE, FAKE, 512, None) == L.SQ_ERR_UNSUPPORTED

    def fwd(c=FAKE, ldc=512, M=256, K=512, qw=None, y=FAKE, yt=L.SQ_BF16, ldy=256):
        if qw is None:
            qw, k = _qw(K=K)
            return lib.sq_linear_forward_combined(c, ldc, M, K, ctypes.byref(qw), FAKE, FAKE, None,
                                                  y, yt, ldy, None)
        return lib.sq_linear_forward_combined(c, ldc, M, K, ctypes.byref(qw), FAKE, FAKE, None, y,
                                              yt, ldy, None)
    assert fwd(c=None) == L.SQ_ERR_INVALID_ARG
    assert fwd(c=FAKE + 8) == L.SQ_ERR_ALIGNMENT
    assert fwd(ldc=520) == L.SQ_ERR_ALIGNMENT
    assert fwd(ldc=256) == L.SQ_ERR_INVALID_ARG
    qw4, k4 = _qw(bits=4, K=512)
    assert fwd(qw=qw4) == L.SQ_ERR_UNSUPPORTED        # int8 weights only
    assert fwd(M=0) == L.SQ_OK


def test_single_scale_entry_points_validate_before_launch():
    lib = _lib.load()
    L = _lib
    seg, keep = _lib.segments((0, 512))
    qs = lib.sq_quantize_activations_single
    assert qs(FAKE, 1, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE, 520, None) == L.SQ_ERR_ALIGNMENT
    assert qs(FAKE, 1, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, None, 512, None) == L.SQ_ERR_INVALID_ARG
    assert qs(FAKE, 9, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE, 512, None) == L.SQ_ERR_INVALID_ARG
    assert qs(FAKE, 1, 0, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE, 512, None) == L.SQ_OK
    qw, k = _qw(K=512)
    fs = lib.sq_linear_forward_single
    assert fs(None, 512, 256, 512, ctypes.byref(qw), FAKE, FAKE, None, FAKE, L.SQ_BF16, 256, None) == L.SQ_ERR_INVALID_ARG
    assert fs(FAKE + 8, 512, 256, 512, ctypes.byref(qw), FAKE, FAKE, None, FAKE, L.SQ_BF16, 256, None) == L.SQ_ERR_ALIGNMENT
    assert fs(FAKE, 512, 256, 512, ctypes.byref(qw), None, FAKE, None, FAKE, L.SQ_BF16, 256, None) == L.SQ_ERR_INVALID_ARG
    qw4, k4 = _qw(bits=4, K=512)
    assert fs(FAKE, 512, 256, 512, ctypes.byref(qw4), FAKE, FAKE, None, FAKE, L.SQ_BF16, 256, None) == L.SQ_ERR_UNSUPPORTED
    assert fs(FAKE, 512, 0, 512, ctypes.byref(qw), FAKE, FAKE, None, FAKE, L.SQ_BF16, 256, None) == L.SQ_OK


def test_splitk_entry_points_validate_before_launch():
    lib = _lib.load()
    L = _lib
    n = ctypes.c_size_t()
    assert lib.sq_splitk_workspace_size(129, 1024, 1024, ctypes.byref(n)) == L.SQ_ERR_INVALID_ARG
    assert lib.sq_splitk_workspace_size(0, 1024, 1024, ctypes.byref(n)) == L.SQ_ERR_INVALID_ARG
    assert lib.sq_splitk_workspace_size(64, 1024, 1024, None) == L.SQ_ERR_INVALID_ARG
    qw, k = _qw(K=512)
    f = lib.sq_linear_forward_codes_splitk

    def call(M=64, q=FAKE, ws=FAKE, wsb=1 << 30, qw_=qw, y=FAKE):
        return f(q, q, 512, M, 512, ctypes.byref(qw_), FAKE, FAKE, None, y, L.SQ_BF16, 256, ws,
                 wsb, None)
    assert call(M=200) == L.SQ_ERR_UNSUPPORTED
    qws, ks = _qw(kb=(0, 256, 512))
    assert call(qw_=qws) == L.SQ_ERR_UNSUPPORTED
    qw4, k4 = _qw(bits=4, K=512)
    assert call(qw_=qw4) == L.SQ_ERR_UNSUPPORTED
    assert call(ws=None) == L.SQ_ERR_INVALID_ARG
    assert call(ws=FAKE + 16) == L.SQ_ERR_ALIGNMENT          # 256-byte alignment
    assert call(wsb=16) == L.SQ_ERR_INVALID_ARG
    assert call(q=FAKE + 8) == L.SQ_ERR_ALIGNMENT
    assert call(M=0) == L.SQ_OK


def test_hadamard_entry_points_validate_before_launch():
    lib = _lib.load()
    L = _lib
    seg, keep = _lib.segments((0, 512))
    ca = lib.sq_calibrate_hadamard
    assert ca(FAKE, 1, 16, 512, 512, ctypes.byref(seg), None, FAKE, None) == L.SQ_ERR_INVALID_ARG
    assert ca(FAKE, 1, -1, 512, 512, ctypes.byref(seg), FAKE, FAKE, None) == L.SQ_ERR_INVALID_ARG
    assert ca(FAKE + 8, 1, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, None) == L.SQ_ERR_ALIGNMENT
    odd, keep2 = _lib.segments((0, 520))
    assert ca(FAKE, 0, 16, 520, 520, ctypes.byref(odd), FAKE, FAKE, None) == L.SQ_ERR_UNSUPPORTED
    qa = lib.sq_quantize_activations_hadamard
    assert qa(FAKE, 1, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE, FAKE, 520, None) == L.SQ_ERR_ALIGNMENT
    assert qa(FAKE, 1, 16, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE, None, 512, None) == L.SQ_ERR_INVALID_ARG
    assert qa(FAKE, 1, 0, 512, 512, ctypes.byref(seg), FAKE, FAKE, FAKE, FAKE, 512, None) == L.SQ_OK
    qw4, k4 = _qw(bits=4, K=512)
    qw8, k8 = _qw(bits=8, K=512)
    ro = lib.sq_rotate_weights_hadamard
    assert ro(ctypes.byref(qw8), FAKE, 512, None) == L.SQ_ERR_UNSUPPORTED
    assert ro(ctypes.byref(qw4), None, 512, None) == L.SQ_ERR_INVALID_ARG
    assert ro(ctypes.byref(qw4), FAKE, 256, None) == L.SQ_ERR_INVALID_ARG
    assert ro(ctypes.byref(qw4), FAKE, 520, None) == L.SQ_ERR_ALIGNMENT
    assert ro(ctypes.byref(qw4), FAKE + 8, 512, None) == L.SQ_ERR_ALIGNMENT
    fh = lib.sq_linear_forward_codes_hadamard

    def fwd(qw=qw4, wr=FAKE, ldr=512, M=256, q=FAKE):
        return fh(q, q, 512, M, 512, ctypes.byref(qw), wr, ldr, FAKE, FAKE, None, FAKE, L.SQ_BF16,
                  256, None)
    assert fwd(qw=qw8) == L.SQ_ERR_UNSUPPORTED
    assert fwd(wr=None) == L.SQ_ERR_INVALID_ARG
    assert fwd(ldr=256) == L.SQ_ERR_INVALID_ARG
    assert fwd(ldr=520) == L.SQ_ERR_ALIGNMENT
    assert fwd(wr=FAKE + 8) == L.SQ_ERR_ALIGNMENT
    assert fwd(q=None) == L.SQ_ERR_INVALID_ARG
    assert fwd(M=0) == L.SQ_OK


def test_no_cpu_fallback_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_libs", {})
    monkeypatch.setattr(_lib, "_active", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        _lib.load()
