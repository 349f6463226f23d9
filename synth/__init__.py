"""Seeded synthetic inputs shared by the CPU oracle's tests and the CUDA path.

Only random numbers live here (see ``synth.c``): bf16 weights and activations with
planted outliers, shaped like the layers the MosaicQuant pages evaluate (LLaMA3 and
Qwen3 linear layers, "Experimental results" section of the MosaicQuant summary). No
quantization, scoring or GEMM arithmetic is in this package.

Recipe (all draws from SplitMix64 streams, Box-Muller normals, rounded to bf16):

* W[N][K] = bf16(0.02 * z); ``floor(0.005*N*K)`` entries are multiplied by 20. They sit
  at distinct random positions inside a random subset of the 64x64 blocks
  (3 blocks for the tiny layer, ``floor(0.05 * #blocks)`` otherwise).
* X[M][K] = bf16(z); a set of input channels (4 for the tiny layer, else
  ``floor(frac * K)``) is multiplied by 30 in every token.
* Calibration tokens Xcal[T][K] follow X's recipe with their own stream and the same
  outlier channels.
* Streams: W = 1, X = 2, Xcal = 3, outlier placement = 4; each plus 100 * (workload
  index) + 10 * (matrix index within the workload).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, u64, i32, f64 = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int, ctypes.c_double
        vp = ctypes.c_void_p
        lib.synth_weight.argtypes = [u64, u64, i32, i32, f64, i64, i64, f64, vp]
        lib.synth_weight.restype = i32
        lib.synth_act.argtypes = [u64, u64, i32, i32, i64, f64, vp]
        lib.synth_act.restype = i32
        lib.synth_normal_bf16.argtypes = [u64, f64, i64, vp]
        lib.synth_normal_bf16.restype = None
        lib.synth_choose.argtypes = [u64, i64, i64, vp]
        lib.synth_choose.restype = i32
        lib.synth_draw.argtypes = [u64, u64]
        lib.synth_draw.restype = u64
        _lib = lib
    return _lib


def weight(N: int, K: int, seed_w: int, seed_o: int, sigma: float = 0.02, n_out: int = 0,
           n_out_blocks: int = 0, mult: float = 20.0) -> np.ndarray:
    """bf16 bits [N, K] (uint16)."""
    out = np.empty((N, K), dtype=np.uint16)
    rc = _load().synth_weight(seed_w, seed_o, N, K, sigma, n_out, n_out_blocks, mult, out.ctypes.data)
    if rc != 0:
        raise MemoryError("synth_weight failed")
    return out


def act(M: int, K: int, seed_x: int, seed_c: int, n_ch: int, mult: float = 30.0) -> np.ndarray:
    """bf16 bits [M, K] (uint16)."""
    out = np.empty((M, K), dtype=np.uint16)
    rc = _load().synth_act(seed_x, seed_c, M, K, n_ch, mult, out.ctypes.data)
    if rc != 0:
        raise MemoryError("synth_act failed")
    return out


def normal_bf16(shape, seed: int, sigma: float = 1.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    _load().synth_normal_bf16(seed, sigma, out.size, out.ctypes.data)
    return out


def choose(seed: int, n: int, k: int) -> np.ndarray:
    """k distinct indices of [0, n), ascending (used for sampled parity checks)."""
    out = np.empty(max(k, 0), dtype=np.int64)
    if k > 0 and _load().synth_choose(seed, n, k, out.ctypes.data) != 0:
        raise MemoryError("synth_choose failed")
    return out[: min(k, n)]


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Matrix:
    name: str
    N: int
    K: int


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    matrices: tuple
    Ms: tuple
    T: int
    n_out_blocks_frac: float       # share of 64x64 blocks holding the weight outliers
    n_out_blocks_fixed: int        # explicit count (tiny layer), overrides the share
    act_ch_frac: float
    act_ch_fixed: int
    budgets: tuple                 # block-budget fractions
    note: str = ""

    def matrix(self, name: str) -> Matrix:
        for m in self.matrices:
            if m.name == name:
                return m
        raise KeyError(name)


WORKLOADS = {
    "tiny": Workload(0, "tiny", (Matrix("w", 256, 512),), (16,), 128, 0.0, 3, 0.0, 4, (0.10,),
                     "M=16, K=512, N=256; outliers in 3 of 32 blocks; 4 hot channels"),
    "llama3_8b_qproj_decode": Workload(1, "llama3_8b_qproj_decode", (Matrix("q_proj", 4096, 4096),), (16,), 512,
                                       0.05, 0, 0.01, 0, (0.10,), "LLaMA3-8B q_proj, decode batch 16"),
    "llama3_8b_mlp_prefill": Workload(2, "llama3_8b_mlp_prefill",
                                      (Matrix("up", 14336, 4096), Matrix("gate", 14336, 4096),
                                       Matrix("down", 4096, 14336)), (2048,), 512, 0.05, 0, 0.01, 0, (0.10,),
                                      "LLaMA3-8B MLP, prefill 2048 tokens"),
    "qwen3_32b": Workload(3, "qwen3_32b",
                          (Matrix("q", 5120, 5120), Matrix("up", 25600, 5120), Matrix("down", 5120, 25600)),
                          (1, 16, 128, 1024, 8192), 512, 0.05, 0, 0.01, 0, (0.10,),
                          "Qwen3-32B-shaped layers, M swept"),
    "llama3_70b_mlp": Workload(4, "llama3_70b_mlp",
                               (Matrix("up", 28672, 8192), Matrix("gate", 28672, 8192),
                                Matrix("down", 8192, 28672)), (4096,), 512, 0.05, 0, 0.02, 0,
                               (0.0, 0.05, 0.10, 0.20), "LLaMA3-70B-shaped MLP, M=4096, budget swept"),
}


def budget_blocks(N: int, K: int, frac: float) -> int:
    """floor(frac * number of 64x64 blocks)."""
    return int(math.floor(frac * (N // 64) * (K // 64) + 1e-9))


def seeds(workload: Workload, matrix_index: int = 0) -> dict:
    base = 100 * workload.index + 10 * matrix_index
    return {"w": 1 + base, "x": 2 + base, "xcal": 3 + base, "o": 4 + base}


def layer(workload: str | Workload, matrix: str | None = None, M: int | None = None,
          with_x: bool = True, with_cal: bool = True) -> dict:
    """Generate one layer's inputs: W [N,K], X [M,K], Xcal [T,K] as bf16 bits."""
    wl = WORKLOADS[workload] if isinstance(workload, str) else workload
    mi = 0 if matrix is None else [m.name for m in wl.matrices].index(matrix)
    mat = wl.matrices[mi]
    N, K = mat.N, mat.K
    sd = seeds(wl, mi)
    nblk = (N // 64) * (K // 64)
    n_out = int(math.floor(0.005 * N * K))
    nob = wl.n_out_blocks_fixed or int(math.floor(wl.n_out_blocks_frac * nblk))
    n_ch = wl.act_ch_fixed or int(math.floor(wl.act_ch_frac * K))
    M = wl.Ms[0] if M is None else M
    out = {"workload": wl.name, "matrix": mat.name, "N": N, "K": K, "M": M, "T": wl.T,
           "W": weight(N, K, sd["w"], sd["o"], 0.02, n_out, nob, 20.0), "n_ch": n_ch}
    if with_x:
        out["X"] = act(M, K, sd["x"], sd["o"], n_ch, 30.0)
    if with_cal:
        out["Xcal"] = act(wl.T, K, sd["xcal"], sd["o"], n_ch, 30.0)
    return out
