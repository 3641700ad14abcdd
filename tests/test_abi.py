"""The C-ABI library builds for sm_100a, loads, exports every function include/qt2.h declares,
and rejects bad arguments on the host before any CUDA work (CPU only: no compute call needs a
GPU here; without one, a valid call must fail with QT2_ERR_DEVICE, never fall back)."""
import ctypes
import subprocess

import numpy as np
import pytest
import torch

from nvfp4_quantized_b200 import build as qbuild
from nvfp4_quantized_b200 import qt2
from tests.layout import canonical_to_scales, scale_offsets, scales_to_canonical


@pytest.fixture(scope="module")
def L():
    qbuild.build()
    return qt2.lib()


def test_exports_every_header_function(L):
    names = qt2.header_functions()
    assert len(names) == 28
    out = subprocess.run(["nm", "-D", "--defined-only", qt2.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(L, n)
    # nothing but the C ABI leaks out of the library
    assert {e for e in exported if e.startswith("qt2")} == set(names)


def test_checked_build_exports_the_same_abi(L):
    """libqt2_checked.so (QT2_CHECKED: every kernel store checked) has exactly the product
    library's entry points and says which build it is; the product library says it is not."""
    path = qbuild.build(checked=True)
    names = qt2.header_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    assert {e for e in exported if e.startswith("qt2")} == set(names)
    C = ctypes.CDLL(path)
    assert C.qt2_build_checked() == 1
    assert L.qt2_build_checked() == 0
    assert qt2.qt2_status_string(qt2.QT2_ERR_BOUNDS).startswith("a kernel store")


def test_built_for_sm100a_only():
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", qt2.LIB_PATH], capture_output=True,
                         text=True).stdout
    assert "sm_100a" in out and "sm_90" not in out


def test_version_and_status_strings(L):
    assert qt2.qt2_version() >= 100
    for code in range(0, -10, -1):
        s = qt2.qt2_status_string(code)
        assert s and s != "unknown status"


def test_workspace_size_queries(L):
    M, K, N = 256, 512, 384
    fwd = qt2.qt2_linear_fwd_workspace_size(M, K, N)
    view = lambda R, C: (R * C // 2 + 255) // 256 * 256 + (R * C // 16 + 255) // 256 * 256 + 256
    assert fwd == 256 + view(M, K) + view(N, K)
    bwd = qt2.qt2_linear_bwd_workspace_size(M, K, N)
    assert bwd >= view(M, N) * 2 + view(K, N) + view(K, M) + 4 * (M * N + N * K + M * K) // 16
    assert qt2.qt2_quant_msedEN_workspace_size(M, K, qt2.QT2_LAYOUT_BOTH) == 256 + 2 * (M * K // 16 * 4)
    with pytest.raises(qt2.QT2Error) as e:
        qt2.qt2_linear_fwd_workspace_size(100, 128, 128)
    assert e.value.status == qt2.QT2_ERR_SHAPE


def _view(codes=0x10000, scales=0x20000, ts=0x30000):
    return qt2.NVFP4ViewC(codes, scales, ts)


def test_dimension_limit(L):
    """Dimensions reach the kernels as 32-bit ints: 2^31 - 128 is accepted by the size queries,
    2^31 is refused with QT2_ERR_SHAPE before any CUDA call."""
    big = (1 << 31) - 128
    assert qt2.qt2_quant_msedEN_workspace_size(big, 128, qt2.QT2_LAYOUT_ROW) > 0
    for bad in (1 << 31, 1 << 32):
        with pytest.raises(qt2.QT2Error) as e:
            qt2.qt2_quant_msedEN_workspace_size(bad, 128, qt2.QT2_LAYOUT_ROW)
        assert e.value.status == qt2.QT2_ERR_SHAPE
        with pytest.raises(qt2.QT2Error) as e:
            qt2.qt2_linear_fwd_workspace_size(128, bad, 128)
        assert e.value.status == qt2.QT2_ERR_SHAPE


def test_host_validation_codes(L):
    """Fake, never-dereferenced device addresses: validation happens before any CUDA call."""
    v = _view()
    f = L.qt2_quant_fwd46
    R = ctypes.byref
    assert f(None, 128, 128, 128, 1, R(v), None, 0x40000, 256, None) == qt2.QT2_ERR_INVALID_ARG
    assert f(0x1000, 100, 128, 128, 1, R(v), None, 0x40000, 256, None) == qt2.QT2_ERR_SHAPE
    assert f(0x1000, 0, 128, 128, 1, R(v), None, 0x40000, 256, None) == qt2.QT2_ERR_SHAPE      # empty
    assert f(0x1000, 128, 0, 128, 1, R(v), None, 0x40000, 256, None) == qt2.QT2_ERR_SHAPE
    assert f(0x1000, -128, 128, 128, 1, R(v), None, 0x40000, 256, None) == qt2.QT2_ERR_SHAPE
    assert f(0x1000, 128, 128, 64, 1, R(v), None, 0x40000, 256, None) == qt2.QT2_ERR_SHAPE
    assert f(0x1008, 128, 128, 128, 1, R(v), None, 0x40000, 256, None) == qt2.QT2_ERR_ALIGN
    assert f(0x1000, 128, 128, 132, 1, R(v), None, 0x40000, 256, None) == qt2.QT2_ERR_ALIGN
    assert f(0x1000, 128, 128, 128, 2, R(v), None, 0x40000, 256, None) == qt2.QT2_ERR_INVALID_ARG
    assert f(0x1000, 128, 128, 128, 1, R(v), None, None, 256, None) == qt2.QT2_ERR_WORKSPACE
    assert f(0x1000, 128, 128, 128, 1, R(_view(codes=0x10008)), None, 0x40000, 256, None) == qt2.QT2_ERR_ALIGN
    g = L.qt2_quant_msedEN
    assert g(0x1000, 128, 128, 128, 0, 1, 1, 2, R(v), R(v), 0x40000, 1 << 20, None) == qt2.QT2_ERR_INVALID_ARG
    assert g(0x1000, 128, 128, 128, 3, 1, 1, 2, R(v), None, 0x40000, 1 << 20, None) == qt2.QT2_ERR_INVALID_ARG
    assert g(0x1000, 128, 128, 128, 3, 1, 1, 2, R(v), R(v), 0x40000, 16, None) == qt2.QT2_ERR_WORKSPACE
    assert g(0x1000, 128, 128, 128, 3, 1, 1, 2, R(v), R(v), 0x40010, 1 << 20, None) == qt2.QT2_ERR_ALIGN
    h = L.qt2_gemm_nvfp4
    assert h(R(v), R(v), 128, 128, 128, 1.0, None, 0, 128, None) == qt2.QT2_ERR_INVALID_ARG
    assert h(R(v), R(v), 128, 128, 128, 1.0, 0x50000, 7, 128, None) == qt2.QT2_ERR_INVALID_ARG
    assert h(R(v), R(v), 128, 192, 128, 1.0, 0x50000, 0, 192, None) == qt2.QT2_ERR_SHAPE
    assert h(R(v), R(v), 128, 128, 128, 1.0, 0x50000, 0, 64, None) == qt2.QT2_ERR_SHAPE
    assert h(R(v), R(v), 128, 128, 0, 1.0, 0x50000, 0, 128, None) == qt2.QT2_ERR_SHAPE       # empty K
    assert h(R(v), R(v), 0, 128, 128, 1.0, 0x50000, 0, 128, None) == qt2.QT2_ERR_SHAPE
    assert L.qt2_linear_fwd(0x1000, 0x2000, 128, 128, 128, 0x3000, None, 0, None) == qt2.QT2_ERR_WORKSPACE
    assert L.qt2_linear_bwd(0x1000, 0x2000, 0x3000, 128, 128, 128, 0, 0x4000, 0x5000, 3, 0x6000, 1 << 30,
                            None) == qt2.QT2_ERR_INVALID_ARG
    fx = L.qt2_quant_fwd46_msedEN_col
    assert fx(0x1000, 128, 128, 128, 1, 4, R(v), None, 0x40000, 1 << 20, None) == qt2.QT2_ERR_INVALID_ARG
    assert fx(0x1000, 128, 192, 192, 1, 4, R(v), R(v), 0x40000, 1 << 20, None) == qt2.QT2_ERR_SHAPE
    assert fx(0x1000, 128, 128, 128, 1, 4, R(v), R(v), 0x40000, 16, None) == qt2.QT2_ERR_WORKSPACE
    assert fx(0x1000, 128, 128, 128, 1, 4, R(v), R(_view(scales=0x20004)), 0x40000, 1 << 20,
              None) == qt2.QT2_ERR_ALIGN
    lq = L.qt2_quant_fwd46_local
    assert lq(None, 128, 128, 128, R(v), None) == qt2.QT2_ERR_INVALID_ARG
    assert lq(0x1000, 192, 128, 128, R(v), None) == qt2.QT2_ERR_SHAPE
    assert lq(0x1000, 128, 128, 128, None, None) == qt2.QT2_ERR_INVALID_ARG
    lg = L.qt2_gemm_nvfp4_local
    assert lg(R(v), R(v), 128, 128, 128, 1.0, None, 0, 128, None) == qt2.QT2_ERR_INVALID_ARG
    assert lg(R(v), R(v), 128, 128, 128, 1.0, 0x50000, 0, 64, None) == qt2.QT2_ERR_SHAPE
    assert lg(R(v), R(v), 128, 128, 128, 1.0, 0x50008, 0, 128, None) == qt2.QT2_ERR_ALIGN
    sq = L.qt2_quant_fwd46_sq
    assert sq(0x1000, 128, 128, 128, None, R(v), 0x40000, 256, None) == qt2.QT2_ERR_INVALID_ARG
    assert sq(0x1000, 128, 200, 200, R(v), R(v), 0x40000, 256, None) == qt2.QT2_ERR_SHAPE
    assert sq(0x1000, 128, 128, 128, R(v), R(v), 0x40000, 8, None) == qt2.QT2_ERR_WORKSPACE
    assert sq(0x1002, 128, 128, 128, R(v), R(v), 0x40000, 256, None) == qt2.QT2_ERR_ALIGN
    bv = L.qt2_linear_bwd_views
    assert bv(0x1000, 128, 128, 128, 0, None, R(v), 0x4000, 0x5000, 1, 0x6000, 1 << 30, None) == \
        qt2.QT2_ERR_INVALID_ARG
    assert bv(0x1000, 128, 128, 128, 0, R(v), R(v), 0x4000, 0x5000, 9, 0x6000, 1 << 30, None) == \
        qt2.QT2_ERR_INVALID_ARG
    assert bv(0x1000, 128, 320, 128, 0, R(v), R(v), 0x4000, 0x5000, 1, 0x6000, 1 << 30, None) == qt2.QT2_ERR_SHAPE
    assert bv(0x1000, 128, 128, 128, 0, R(v), R(v), 0x4000, 0x5000, 1, 0x6000, 64, None) == qt2.QT2_ERR_WORKSPACE
    assert qt2.qt2_linear_bwd_views_workspace_size(256, 128, 384) < qt2.qt2_linear_bwd_workspace_size(256, 128, 384)
    assert qt2.qt2_quant_fwd46_msedEN_col_workspace_size(256, 512) == \
        qt2.qt2_quant_msedEN_workspace_size(256, 512, qt2.QT2_LAYOUT_COL)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU behaviour")
def test_valid_call_without_gpu_fails_loudly(L):
    v = _view()
    st = L.qt2_quant_fwd46(0x1000, 128, 128, 128, 1, ctypes.byref(v), None, 0x40000, 256, None)
    assert st == qt2.QT2_ERR_DEVICE
    assert L.qt2_selftest_wait_timeout(None) == qt2.QT2_ERR_DEVICE
    with pytest.raises(qt2.QT2Error):
        qt2._check("qt2_quant_fwd46", st)


def test_scale_layout_helpers_are_inverse():
    R, C = 256, 512
    off = scale_offsets(R, C)
    assert sorted(off.ravel().tolist()) == list(range(R * C // 16))
    canon = np.random.default_rng(0).integers(0, 127, (R, C // 16)).astype(np.uint8)
    assert np.array_equal(scales_to_canonical(canonical_to_scales(canon), R, C), canon)
    # one 512-byte atom holds 128 rows x 4 groups; rows r, r+32, r+64, r+96 share a 16-byte line
    assert off[0, 0] == 0 and off[32, 0] == 4 and off[1, 0] == 16 and off[0, 1] == 1 and off[0, 4] == 512


# --------------------------------------------------------------------------- host-side fault injection
def _skip_then_fail(fail_site):
    """Skip every CUDA call before `fail_site` (no GPU is touched) and fail at it."""
    return lambda site: qt2.FAULT_FAIL if site == fail_site else qt2.FAULT_SKIP


def test_injected_launch_failure_returns_cuda_error(L):
    """A launch that fails is reported as QT2_ERR_CUDA and nothing after it is enqueued; with
    every other CUDA call skipped, no GPU is needed or touched."""
    v = _view()
    R = ctypes.byref
    with qt2.fault_hook(_skip_then_fail("launch")) as h:
        st = L.qt2_quant_msedEN(0x1000, 256, 256, 256, qt2.QT2_LAYOUT_BOTH, 1, 1, 2, R(v), R(v), 0x40000, 1 << 20,
                                None)
    assert st == qt2.QT2_ERR_CUDA
    assert h.sites == ["device", "tensor_map", "memset", "launch"]   # the producer's launch failed first
    with qt2.fault_hook(_skip_then_fail("launch")) as h:
        st = L.qt2_quant_fwd46(0x1000, 128, 128, 128, 1, R(v), None, 0x40000, 256, None)
    assert st == qt2.QT2_ERR_CUDA and h.sites == ["device", "memset", "launch"]
    with qt2.fault_hook(_skip_then_fail("launch")) as h:
        st = L.qt2_linear_bwd(0x1000, 0x2000, 0x3000, 256, 256, 256, 0, 0x4000, 0x5000, 1, 0x100000, 1 << 30, None)
    assert st == qt2.QT2_ERR_CUDA and h.sites[-1] == "launch" and h.sites.count("launch") == 1
    with qt2.fault_hook(_skip_then_fail("launch")):
        assert L.qt2_selftest_wait_timeout(None) == qt2.QT2_ERR_CUDA


def test_injected_failures_at_every_site_of_a_layer_call(L):
    """Walk the layer's backward call through every CUDA call it makes: skipping all of them
    completes with QT2_OK having touched nothing; failing the k-th one returns the error of that
    site and stops there."""
    R = ctypes.byref
    args = (0x1000, 0x2000, 0x3000, 256, 256, 256, 0, 0x4000, 0x5000, 1, 0x100000, 1 << 30, None)
    with qt2.fault_hook(lambda site: qt2.FAULT_SKIP) as h:
        assert L.qt2_linear_bwd(*args) == qt2.QT2_OK
    sites = list(h.sites)
    # three MS-EDEN calls (descriptor, max reset, producer, scale pass) and two GEMMs (descriptors, launch)
    assert sites.count("launch") == 8 and sites[0] == "device"
    for k in range(len(sites)):
        calls = []

        def decide(site, k=k, calls=calls):
            calls.append(site)
            return qt2.FAULT_FAIL if len(calls) == k + 1 else qt2.FAULT_SKIP
        with qt2.fault_hook(decide):
            st = L.qt2_linear_bwd(*args)
        assert len(calls) == k + 1, (k, calls)
        assert st == (qt2.QT2_ERR_DEVICE if sites[k] == "device" else qt2.QT2_ERR_CUDA), (k, sites[k], st)
    # the hook is gone: the plain call fails on the device query again (no GPU here) or runs
    if not torch.cuda.is_available():
        assert L.qt2_linear_bwd(*args) == qt2.QT2_ERR_DEVICE


def test_injected_failure_of_the_noalloc_scratch_lookup(L):
    v = _view()
    R = ctypes.byref
    with qt2.fault_hook(_skip_then_fail("symbol")) as h:
        st = L.qt2_quant_msedEN_noalloc(0x1000, 256, 256, 256, qt2.QT2_LAYOUT_BOTH, 1, 1, 2, R(v), R(v), None)
    assert st == qt2.QT2_ERR_CUDA and h.sites == ["device", "symbol"]


# --------------------------------------------------------------------------- no-alloc capacity
def test_noalloc_capacity_boundary(L):
    """qt2_quant_msedEN_noalloc takes up to 32 MiB of pre-scales (rows*cols/4 bytes per view):
    8192 x 8192 with both views and 8192 x 16384 with one view are accepted, one 128-block
    more is refused with QT2_ERR_WORKSPACE before any CUDA call (fake addresses)."""
    v = _view()
    R = ctypes.byref
    f = L.qt2_quant_msedEN_noalloc
    # skip every CUDA call: an accepted call then enqueues nothing and returns QT2_OK
    with qt2.fault_hook(lambda site: qt2.FAULT_SKIP):
        assert f(0x1000, 8192, 8192, 8192, qt2.QT2_LAYOUT_BOTH, 1, 1, 2, R(v), R(v), None) == qt2.QT2_OK
        assert f(0x1000, 8192, 16384, 16384, qt2.QT2_LAYOUT_ROW, 1, 1, 2, R(v), None, None) == qt2.QT2_OK
        assert f(0x1000, 16384, 8192, 8192, qt2.QT2_LAYOUT_COL, 1, 1, 2, None, R(v), None) == qt2.QT2_OK
        assert f(0x1000, 8192, 8320, 8320, qt2.QT2_LAYOUT_BOTH, 1, 1, 2, R(v), R(v), None) == qt2.QT2_ERR_WORKSPACE
        assert f(0x1000, 8320, 8192, 8192, qt2.QT2_LAYOUT_BOTH, 1, 1, 2, R(v), R(v), None) == qt2.QT2_ERR_WORKSPACE
        assert f(0x1000, 8192, 16512, 16512, qt2.QT2_LAYOUT_ROW, 1, 1, 2, R(v), None, None) == qt2.QT2_ERR_WORKSPACE
    limit = 32 * 1024 * 1024
    assert qt2.qt2_quant_msedEN_workspace_size(8192, 8192, qt2.QT2_LAYOUT_BOTH) == 256 + limit
    assert qt2.qt2_quant_msedEN_workspace_size(8192, 16384, qt2.QT2_LAYOUT_ROW) == 256 + limit
