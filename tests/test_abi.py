"""The C ABI library loads on a machine without a GPU, exports every call that
include/mosaic.h declares, and validates arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from bit_quantized_gemm_zipperengine_b200 import build, mosaic
    build.build()
    return mosaic.lib()


def declared():
    """Every mq_* function that a header under include/ declares."""
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            with open(os.path.join(ROOT, "include", h)) as f:
                text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
            names |= set(re.findall(r"\b(mq_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(L):
    names = declared()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    assert set(mosaic.EXPORTED) == set(names)


def test_size_helpers(L):
    assert L.mq_sf_swz_bytes(16, 4096) == 128 * 256
    assert L.mq_sf_swz_bytes(300, 512) == 384 * 32
    assert L.mq_sf_swz_bytes(16, 100) == 0
    assert L.mq_budget_blocks(256, 512, 0.10) == 3
    assert L.mq_budget_blocks(4096, 4096, 0.10) == 409
    assert L.mq_budget_blocks(28672, 8192, 0.05) == 2867
    assert L.mq_budget_blocks(256, 512, 1.5) == -1
    assert L.mq_quantize_weight_workspace_bytes(4096, 4096) >= 4 * 148 * 8
    # decode GEMM at M=16, N=K=4096 (no GPU here: 148 SMs assumed): 32 weight tiles, each
    # split among the 4 CTAs of a cluster and added through its shared memory: nothing
    assert L.mq_gemm_workspace_bytes(16, 4096, 4096, 0) == 0
    # 150 weight tiles (more than half the SMs): the stream-K kernel, 2400 units over 148
    # CTAs, tiles split between CTAs: two fp32 partial slots of 128 x 16 per CTA, then one
    # counter per tile
    assert L.mq_gemm_workspace_bytes(16, 150 * 128, 4096, 0) == 2 * 148 * 16 * 128 * 4 + 150 * 4
    # a tile held whole by every CTA needs nothing: 148 tiles of one K stage each
    assert L.mq_gemm_workspace_bytes(16, 148 * 128, 256, 0) == 0
    # the large-M kernel needs no workspace
    assert L.mq_gemm_workspace_bytes(256, 1024, 4096, 0) == 0


class _Buffers:
    """Real buffers for the refusal checks: device memory when a GPU is present, host
    memory otherwise (no kernel can launch without a GPU). Never a made-up address, so a
    check that stopped refusing could not send a kernel to memory that is not there."""

    def __init__(self):
        import torch
        self.dev = "cuda" if torch.cuda.is_available() else "cpu"
        self.keep = []

    def __call__(self, nbytes, offset=0):
        import torch
        t = torch.zeros(nbytes + 256, dtype=torch.uint8, device=self.dev)
        self.keep.append(t)
        return ctypes.c_void_p(t.data_ptr() + offset)


def test_host_validation_rejects_bad_arguments(L):
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    buf = _Buffers()
    m = mosaic.NVFP4Mat(16, 4096, None, None, None, None)
    # null pointers and bad shapes are rejected before any CUDA call
    assert L.mq_quantize_act(None, 16, 4096, ctypes.byref(m), None) == 1
    assert L.mq_hessian_diag(None, 8, 64, None, None) == 1
    assert L.mq_gemm(ctypes.byref(m), ctypes.byref(m), None, None, 16, 4096, 4096, 0, None, 0, None) == 1

    def act(M, K):
        return mosaic.NVFP4Mat(M, K, buf(M * K // 2), None, buf(L.mq_sf_swz_bytes(M, K)), buf(4 * M))

    def wt(N, K):
        return mosaic.NVFP4Mat(N, K, buf(N * K // 2), None, buf(L.mq_sf_swz_bytes(N, K)), buf(4))

    xm, Y = act(16, 4096), buf(16 * (4096 + 64) * 2)
    wm = wt(4096 + 64, 4096)
    assert L.mq_gemm(ctypes.byref(xm), ctypes.byref(wm), None, Y, 16, 4096 + 64, 4096, 0, None, 0, None) == 2
    wm2 = wt(4096, 4096)
    assert L.mq_gemm(ctypes.byref(xm), ctypes.byref(wm2), None, Y, 16, 4096, 4096,
                     mosaic.MQ_GEMM_BASE_ONLY | mosaic.MQ_GEMM_RESIDUAL_ONLY, None, 0, None) == 1
    # a decode problem whose tiles are split between CTAs (the stream-K kernel at 150
    # tiles) needs its workspace
    wm1, Y1 = wt(19200, 4096), buf(16 * 19200 * 2)
    assert L.mq_gemm(ctypes.byref(xm), ctypes.byref(wm1), None, Y1, 16, 19200, 4096, 0, None, 0, None) == 3
    assert L.mq_status_string(3) == b"workspace missing or too small"
    # A2 takes 1..1024 calibration tokens and a 16-byte aligned Xcal
    xcal, H = buf(1025 * 4096 * 2), buf(4096 * 4)
    assert L.mq_hessian_diag(xcal, 1025, 4096, H, None) == 2
    assert L.mq_hessian_diag(ctypes.c_void_p(xcal.value + 2), 512, 4096, H, None) == 1
    assert L.mq_hessian_diag(xcal, 0, 4096, H, None) == 1
    # A6 holds a row in one CTA: K up to 65536
    big = act(16, 65536 + 64)
    assert L.mq_quantize_act(buf(16 * (65536 + 64) * 2), 16, 65536 + 64, ctypes.byref(big), None) == 2
    # top-K: budget outside [0, nblk]
    delta, rank, sel = buf(4096 * 8), buf(4097 * 4), buf(4097 * 4)
    assert L.mq_topk_blocks(delta, 4096, 4097, rank, sel, None) == 1
    assert L.mq_topk_blocks(delta, 4096, -1, rank, sel, None) == 1


def test_weight_bytes(L):
    # codes + tiled scales + the tensor scale padded to 16 bytes
    assert L.mq_weight_bytes(4096, 4096) == 4096 * 2048 + 4096 * 256 + 16
    assert L.mq_weight_bytes(300 // 64 * 64, 512) == 256 * 256 + 256 * 32 + 16
    assert L.mq_weight_bytes(192, 512) == 192 * 256 + 256 * 32 + 16  # scales padded to 128 rows
    assert L.mq_weight_bytes(100, 512) == 0 and L.mq_weight_bytes(128, 100) == 0 and L.mq_weight_bytes(0, 64) == 0


def test_binding_sizes_the_weight_from_weight_bytes(L):
    """The binding allocates the GEMM-ready weight as one buffer of mq_weight_bytes bytes
    and places codes, tiled scales and the tensor scale at the offsets the header states."""
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    for N, K in ((256, 512), (192, 1024), (4096, 4096)):
        base, _ = mosaic.alloc_weight(N, K, "cpu", with_sf=False)
        blob = base["blob"]
        parts = [base["codes"], base["sf_swz"], base["gscale"]]
        assert blob.numel() == L.mq_weight_bytes(N, K)
        assert sum(t.numel() * t.element_size() for t in parts) + 12 == L.mq_weight_bytes(N, K)
        b0 = blob.data_ptr()
        assert base["codes"].data_ptr() == b0
        assert base["sf_swz"].data_ptr() == b0 + N * K // 2
        assert base["gscale"].data_ptr() == b0 + N * K // 2 + L.mq_sf_swz_bytes(N, K)
        assert all((t.data_ptr() - b0) % 16 == 0 for t in parts)


def test_timeline_read_needs_the_timeline_build(L):
    # the event table exists only in the library built with MQ_TIMELINE
    buf = (ctypes.c_uint64 * (160 * 16))()
    assert L.mq_timeline_read(ctypes.byref(buf), ctypes.sizeof(buf)) == 1
    assert L.mq_timeline_read(None, 0) == 1


def test_wait_fault_hook_refuses_out_of_range(L):
    # the hook only arms the next decode GEMM launch; out-of-range arguments are refused
    assert L.mq_test_arm_wait_fault(-1, 1.0) == 1
    assert L.mq_test_arm_wait_fault(0, 0.0) == 1
    assert L.mq_test_arm_wait_fault(0, 5000.0) == 1
