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
    with open(os.path.join(ROOT, "include", "mosaic.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mq_[a-z0-9_]+)\s*\(", text)))


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
    # decode GEMM at M=16, N=K=4096: 32 weight tiles x 4 K splits reduced inside a cluster
    assert L.mq_gemm_workspace_bytes(16, 4096, 4096, 0) == 0
    # a narrow layer (8 weight tiles) splits K 16 ways: fp32 partials + tile counters
    assert L.mq_gemm_workspace_bytes(16, 1024, 4096, 0) == 16 * 16 * 1024 * 4 + 8 * 4


def test_host_validation_rejects_bad_arguments(L):
    from bit_quantized_gemm_zipperengine_b200 import mosaic
    m = mosaic.NVFP4Mat(16, 4096, None, None, None, None)
    # null pointers and bad shapes are rejected before any CUDA call
    assert L.mq_quantize_act(None, 16, 4096, ctypes.byref(m), None) == 1
    assert L.mq_hessian_diag(None, 8, 64, None, None) == 1
    assert L.mq_gemm(ctypes.byref(m), ctypes.byref(m), None, None, 16, 4096, 4096, 0, None, 0, None) == 1
    fake = ctypes.c_void_p(0x10000)
    xm = mosaic.NVFP4Mat(16, 4096, fake, None, fake, fake)
    wm = mosaic.NVFP4Mat(4096 + 64, 4096, fake, None, fake, fake)
    assert L.mq_gemm(ctypes.byref(xm), ctypes.byref(wm), None, fake, 16, 4096 + 64, 4096, 0, None, 0, None) == 2
    wm2 = mosaic.NVFP4Mat(4096, 4096, fake, None, fake, fake)
    assert L.mq_gemm(ctypes.byref(xm), ctypes.byref(wm2), None, fake, 16, 4096, 4096,
                     mosaic.MQ_GEMM_BASE_ONLY | mosaic.MQ_GEMM_RESIDUAL_ONLY, None, 0, None) == 1
    # a split-K problem on the workspace path needs its workspace
    xm1 = mosaic.NVFP4Mat(16, 4096, fake, None, fake, fake)
    wm1 = mosaic.NVFP4Mat(1024, 4096, fake, None, fake, fake)
    assert L.mq_gemm(ctypes.byref(xm1), ctypes.byref(wm1), None, fake, 16, 1024, 4096, 0, None, 0, None) == 3
    assert L.mq_status_string(3) == b"workspace missing or too small"
    # A2 takes 1..1024 calibration tokens and a 16-byte aligned Xcal
    assert L.mq_hessian_diag(fake, 1025, 4096, fake, None) == 2
    assert L.mq_hessian_diag(ctypes.c_void_p(0x10002), 512, 4096, fake, None) == 1
    assert L.mq_hessian_diag(fake, 0, 4096, fake, None) == 1
    # A6 holds a row in one CTA: K up to 65536
    big = mosaic.NVFP4Mat(16, 65536 + 64, fake, None, fake, fake)
    assert L.mq_quantize_act(fake, 16, 65536 + 64, ctypes.byref(big), None) == 2
    # top-K: budget outside [0, nblk]
    assert L.mq_topk_blocks(fake, 4096, 4097, fake, fake, None) == 1
    assert L.mq_topk_blocks(fake, 4096, -1, fake, fake, None) == 1
