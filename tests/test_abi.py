"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host before touching a GPU (no compute call is
made here)."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svdq.h")


@pytest.fixture(scope="module")
def lib():
    from bit_w4a4_quantized_smooth_b200 import build, binding
    build.build()
    return binding.load()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert {"svdq_pack_residual", "svdq_quantize_act", "svdq_linear"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    from bit_w4a4_quantized_smooth_b200 import status_string
    assert status_string(0) == "SVDQ_OK"
    assert status_string(5) == "SVDQ_ERR_TIMEOUT"
    assert status_string(99) == "SVDQ_UNKNOWN_STATUS"


def test_packed_sizes(lib):
    from bit_w4a4_quantized_smooth_b200 import packed_sizes, SvdqError
    assert packed_sizes(4608, 3072) == (4608 * 1536, 4608 * 192)
    assert packed_sizes(1, 64) == (32, 128 * 4)
    assert packed_sizes(200, 320) == (200 * 160, 256 * 20)
    with pytest.raises(SvdqError):
        packed_sizes(10, 100)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


def test_linear_validation(lib):
    P = ctypes.c_void_p
    ok = dict(xc=FAKE, xs=FAKE, T=FAKE, rc=FAKE, rs=FAKE, L2=FAKE, bias=None, M=128, K=256, N=256,
              r=32, Y=FAKE)

    def call(**kw):
        a = dict(ok, **kw)
        return lib.svdq_linear(P(a["xc"]), P(a["xs"]), P(a["T"]), P(a["rc"]), P(a["rs"]), P(a["L2"]),
                               P(a["bias"]), a["M"], a["K"], a["N"], a["r"], P(a["Y"]), None)

    assert call(xc=None) == 1
    assert call(Y=None) == 1
    assert call(T=None) == 1           # r > 0 needs T
    assert call(M=0) == 1
    assert call(K=100) == 2
    assert call(N=24) == 2
    assert call(r=24) == 2
    assert call(r=144) == 2
    assert call(xc=FAKE + 8) == 3
    assert call(bias=FAKE + 2) == 3


def test_quantize_and_pack_validation(lib):
    P = ctypes.c_void_p
    q = lib.svdq_quantize_act
    assert q(P(FAKE), P(FAKE), P(FAKE), 16, 64, 16, P(FAKE), P(FAKE), None, None, 0, None) == 1  # T missing
    assert q(P(FAKE), P(FAKE), None, 16, 96, 0, P(FAKE), P(FAKE), None, None, 0, None) == 2
    assert q(P(FAKE + 4), P(FAKE), None, 16, 64, 0, P(FAKE), P(FAKE), None, None, 0, None) == 3
    assert q(P(FAKE), P(FAKE), None, 16, 64, 0, P(FAKE), P(FAKE), None, P(FAKE + 8), 64, None) == 3
    p = lib.svdq_pack_residual
    assert p(None, 64, 16, P(FAKE), P(FAKE), None) == 1
    assert p(P(FAKE), 64, 8, P(FAKE), P(FAKE), None) == 2
    assert p(P(FAKE), 64, 16, P(FAKE + 1), P(FAKE), None) == 3
    assert lib.svdq_selftest_wait_timeout(0, None) == 1
    assert lib.svdq_set_wait_timeout(0) == 1
    assert lib.svdq_set_wait_timeout(61_000_000_000) == 1


def test_size_limits_are_rejected_on_the_host(lib):
    """M, N <= 2^22 and K <= 2^20 keep every grid dimension and index of the
    kernels in range; beyond that the calls refuse with UNSUPPORTED_SHAPE."""
    P = ctypes.c_void_p
    big_k = (1 << 20) + 64
    assert lib.svdq_pack_residual(P(FAKE), big_k, 16, P(FAKE), P(FAKE), None) == 2
    assert lib.svdq_pack_residual(P(FAKE), 64, (1 << 22) + 16, P(FAKE), P(FAKE), None) == 2
    q = lib.svdq_quantize_act
    assert q(P(FAKE), P(FAKE), None, (1 << 22) + 1, 64, 0, P(FAKE), P(FAKE), None, None, 0, None) == 2
    assert q(P(FAKE), P(FAKE), None, 16, big_k, 0, P(FAKE), P(FAKE), None, None, 0, None) == 2
    lin = lib.svdq_linear
    args = lambda M, K, N: (P(FAKE), P(FAKE), None, P(FAKE), P(FAKE), None, None, M, K, N, 0, P(FAKE), None)
    assert lin(*args((1 << 22) + 1, 64, 16)) == 2
    assert lin(*args(16, big_k, 16)) == 2
    assert lin(*args(16, 64, (1 << 22) + 16)) == 2
    from bit_w4a4_quantized_smooth_b200 import packed_sizes, SvdqError
    with pytest.raises(SvdqError):
        packed_sizes(16, big_k)


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from bit_w4a4_quantized_smooth_b200 import binding
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        binding.load()


def test_attach_lora_validation(lib):
    P = ctypes.c_void_p
    f = lib.svdq_attach_lora
    ok = (P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), 64, 32, 16, 16, P(FAKE), P(FAKE), None)
    bad = lambda i, v: tuple(v if j == i else a for j, a in enumerate(ok))
    assert f(*bad(3, None)) == 1        # A missing
    assert f(*bad(0, None)) == 1        # L1 missing with r > 0
    assert f(*bad(8, 8)) == 2           # ra not a multiple of 16
    assert f(*bad(7, 128)) == 2         # r + ra > 128
    assert f(*bad(6, 24)) == 2          # N not a multiple of 16
    assert f(*bad(2, P(FAKE + 4))) == 3 # lambda misaligned


def test_channel_absmax_validation(lib):
    P = ctypes.c_void_p
    f = lib.svdq_channel_absmax
    assert f(None, 4, 64, P(FAKE), None) == 1            # null X
    assert f(P(FAKE), 0, 64, P(FAKE), None) == 1         # no rows
    assert f(P(FAKE), 4, 60, P(FAKE), None) == 2         # K not a multiple of 8
    assert f(P(FAKE + 4), 4, 64, P(FAKE), None) == 3     # misaligned X
    assert f(P(FAKE), 4, 64, P(FAKE + 8), None) == 3     # misaligned amax


def test_linear_scaled_alpha_validation(lib):
    P = ctypes.c_void_p
    f = lib.svdq_linear_scaled
    f.argtypes = [P, P, P, P, P, P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                  ctypes.c_float, P, P]
    args = [P(FAKE)] * 6 + [None, 128, 256, 256, 32]
    for bad in (0.0, -2.0, 3.0, 0.3, float("inf"), float("nan"), 2.0 ** -110, 2.0 ** 110):
        assert f(*args, bad, P(FAKE), None) == 1, bad   # SVDQ_ERR_INVALID_ARG before any launch
    # a power of two passes the alpha check and fails later on the shape (K % 64)
    args_bad_k = [P(FAKE)] * 6 + [None, 128, 250, 256, 32]
    assert f(*args_bad_k, 0.5, P(FAKE), None) == 2


def test_global_scale_helpers():
    import math
    from bit_w4a4_quantized_smooth_b200 import prep
    assert prep.global_scale(0.0) == 1.0
    for amax in (1e-6, 0.37, 1.0, 2688.0, 2688.5, 1e5):
        g = prep.global_scale(amax)
        assert math.frexp(g)[0] == 0.5                     # a power of two
        s = amax / (6.0 * g)                               # the largest group's scale
        assert 224.0 < s <= 448.0, (amax, g, s)


def test_launch_overlap_setting(lib):
    from bit_w4a4_quantized_smooth_b200 import set_launch_overlap
    assert lib.svdq_set_launch_overlap(2) == 1      # SVDQ_ERR_INVALID_ARG
    assert lib.svdq_set_launch_overlap(-1) == 1
    set_launch_overlap(False)
    set_launch_overlap(True)                         # the default, restored
