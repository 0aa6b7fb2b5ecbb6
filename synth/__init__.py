"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This package draws numbers and shapes workloads; it computes nothing of the
method (no codebook, quantiser, packing, routing, selection or GEMV). Both
the oracle and the CUDA path take their inputs from here.

Generators (published definitions, implemented twice: ``synth.c`` on the
host and ``synth_dev.cu`` on the device, bit-identical):
  * SplitMix64 counter streams, keyed by ``(seed, stream id)``;
  * N(0, 1) by the Marsaglia polar method.

Workload shapes follow the pages' model (Qwen3.5-397B-A17B MoE layers: 512
experts, top-10, hidden 4096, expert intermediate 1024) and the smaller
configurations used as parity cases. Value distributions:
  * expert weights ~ N(0, 0.02^2), float32;
  * activations ~ N(0, 1), bf16 (float32 for the single-matrix case);
  * router logits ~ N(0, 1), float32, optionally plus a Zipf(1.1)
    popularity bias -1.1 * ln(rank_e) over a seeded permutation of ranks,
    or as an AR(1) process l_t = 0.8 l_{t-1} + 0.6 e_t per layer;
  * per-expert sensitivities s_e = exp(0.5 z_e) (LogNormal(0, 0.5)).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_HOST_SO = os.path.join(_HERE, "libpmoe_synth.so")
_DEV_SO = os.path.join(_HERE, "libpmoe_synth_dev.so")

# stream kinds
K_WEIGHT, K_X, K_LOGIT, K_SENS, K_PERM, K_AR, K_LEAF = 1, 2, 3, 4, 5, 6, 7


def build(force: bool = False, device: bool = True) -> None:
    """Compile the host generator (gcc) and, if asked, the device one (nvcc)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_HOST_SO) or os.path.getmtime(_HOST_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", _HOST_SO, src, "-lm"])
    if device:
        dsrc = os.path.join(_HERE, "synth_dev.cu")
        if force or not os.path.exists(_DEV_SO) or os.path.getmtime(_DEV_SO) < os.path.getmtime(dsrc):
            subprocess.check_call(["nvcc", "-O3", "-shared", "-Xcompiler", "-fPIC",
                                   "-gencode", "arch=compute_100a,code=sm_100a",
                                   "-fmad=false", "-o", _DEV_SO, dsrc])


_lib = None
_dlib = None


def _host():
    global _lib
    if _lib is None:
        if not os.path.exists(_HOST_SO):
            build(device=False)
        lib = ctypes.CDLL(_HOST_SO)
        u64, i64 = ctypes.c_uint64, ctypes.c_int64
        for name, ptr in (("syn_normal_f32", ctypes.c_void_p), ("syn_normal_f64", ctypes.c_void_p),
                          ("syn_normal_bf16", ctypes.c_void_p)):
            fn = getattr(lib, name)
            fn.argtypes = [u64, u64, u64, i64, ctypes.c_double, ptr]
            fn.restype = None
        lib.syn_u64.argtypes = [u64, u64, u64, i64, ctypes.c_void_p]
        lib.syn_u64.restype = None
        lib.syn_stream_key.argtypes = [u64, u64]
        lib.syn_stream_key.restype = u64
        _lib = lib
    return _lib


def _dev():
    global _dlib
    if _dlib is None:
        if not os.path.exists(_DEV_SO):
            build(device=True)
        lib = ctypes.CDLL(_DEV_SO)
        lib.syn_dev_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                           ctypes.c_int64, ctypes.c_double, ctypes.c_void_p,
                                           ctypes.c_void_p]
        lib.syn_dev_normal_f32.restype = ctypes.c_int
        _dlib = lib
    return _dlib


def stream_id(kind: int, a: int = 0, b: int = 0, c: int = 0) -> int:
    """Packs a stream identity into 64 bits: kind(8) | a(24) | b(24) | c(8)."""
    assert 0 <= kind < 256 and 0 <= a < (1 << 24) and 0 <= b < (1 << 24) and 0 <= c < 256
    return (kind << 56) | (a << 32) | (b << 8) | c


def normal_f32(seed: int, stream: int, n: int, scale: float = 1.0, start: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _host().syn_normal_f32(seed, stream, start, n, scale, out.ctypes.data)
    return out


def normal_f64(seed: int, stream: int, n: int, scale: float = 1.0, start: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _host().syn_normal_f64(seed, stream, start, n, scale, out.ctypes.data)
    return out


def normal_bf16(seed: int, stream: int, n: int, scale: float = 1.0, start: int = 0) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(0, scale^2) samples."""
    out = np.empty(n, dtype=np.uint16)
    _host().syn_normal_bf16(seed, stream, start, n, scale, out.ctypes.data)
    return out


def u64(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _host().syn_u64(seed, stream, start, n, out.ctypes.data)
    return out


def normal_f32_device(seed: int, stream: int, n: int, scale: float, dev_ptr: int,
                      cuda_stream: int = 0, start: int = 0) -> None:
    """Same numbers as :func:`normal_f32`, written to device memory."""
    rc = _dev().syn_dev_normal_f32(seed, stream, start, n, scale, dev_ptr, cuda_stream)
    if rc != 0:
        raise RuntimeError(f"syn_dev_normal_f32 failed with code {rc}")


def bf16_to_f32(u: np.ndarray) -> np.ndarray:
    return (u.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------- workloads

def expert_weights(seed: int, layer: int, expert: int, mat: int, n_rows: int, n_cols: int) -> np.ndarray:
    """Weights of one expert matrix (mat 0 = gate, 1 = up, 2 = down), N(0, 0.02^2)."""
    s = stream_id(K_WEIGHT, layer, expert, mat)
    return normal_f32(seed, s, n_rows * n_cols, 0.02).reshape(n_rows, n_cols)


def expert_weights_device(seed: int, layer: int, expert: int, mat: int, n: int, dev_ptr: int,
                          cuda_stream: int = 0) -> None:
    normal_f32_device(seed, stream_id(K_WEIGHT, layer, expert, mat), n, 0.02, dev_ptr, cuda_stream)


def activation_bf16(seed: int, token: int, layer: int, hidden: int) -> np.ndarray:
    return normal_bf16(seed, stream_id(K_X, layer, token), hidden)


def activation_f32(seed: int, token: int, layer: int, n: int) -> np.ndarray:
    return normal_f32(seed, stream_id(K_X, layer, token), n)


def router_logits(seed: int, token: int, layer: int, experts: int) -> np.ndarray:
    return normal_f32(seed, stream_id(K_LOGIT, layer, token), experts)


def sensitivities(seed: int, layer: int, experts: int, sigma: float = 0.5) -> np.ndarray:
    """s_e = exp(sigma * z_e): LogNormal(0, sigma), float32."""
    z = normal_f64(seed, stream_id(K_SENS, layer), experts)
    return np.exp(sigma * z).astype(np.float32)


def permutation(seed: int, stream: int, n: int) -> np.ndarray:
    """Fisher-Yates shuffle of 0..n-1 driven by the counter stream."""
    r = u64(seed, stream, n)
    p = np.arange(n, dtype=np.int64)
    for i in range(n - 1, 0, -1):
        j = int(r[i] % np.uint64(i + 1))
        p[i], p[j] = p[j], p[i]
    return p


def zipf_bias(seed: int, experts: int, s: float = 1.1) -> np.ndarray:
    """-s * ln(rank_e), ranks 1..E a seeded permutation (Zipf(s) log-pmf up to a constant)."""
    rank = permutation(seed, stream_id(K_PERM, 0), experts) + 1
    return (-s * np.log(rank.astype(np.float64))).astype(np.float32)


def ar1_logits(seed: int, layer: int, tokens: int, experts: int, rho: float = 0.8) -> np.ndarray:
    """AR(1) logits per layer: l_0 = e_0, l_t = rho l_{t-1} + sqrt(1-rho^2) e_t (marginal N(0,1))."""
    e = normal_f64(seed, stream_id(K_AR, layer), tokens * experts).reshape(tokens, experts)
    out = np.empty_like(e)
    out[0] = e[0]
    c = math.sqrt(1.0 - rho * rho)
    for t in range(1, tokens):
        out[t] = rho * out[t - 1] + c * e[t]
    return out.astype(np.float32)


def tree_leaves(seed: int, table: int = 0):
    """A skewed, heavy-tailed 256-entry leaf table, ascending, and leaf frequencies (float32).

    Stands in for a per-block K-means codebook of real weights: draws
    t = z0 / sqrt((z1^2 + z2^2 + z3^2) / 3) (Student-t, 3 degrees of freedom)
    plus a skew term 0.4 * |z0|, sorted; frequencies 1 + 999 * u with u
    uniform in [0, 1) from the counter stream, and two of them set to zero."""
    z = normal_f64(seed, stream_id(K_LEAF, table), 4 * 256).reshape(4, 256)
    t = z[0] / np.sqrt((z[1] ** 2 + z[2] ** 2 + z[3] ** 2) / 3.0) + 0.4 * np.abs(z[0])
    leaves = np.sort(t).astype(np.float32)
    u = u64(seed, stream_id(K_LEAF, table, 1), 256)
    freq = (1.0 + 999.0 * (u >> np.uint64(11)).astype(np.float64) / float(1 << 53)).astype(np.float32)
    freq[7] = 0.0
    freq[8] = 0.0
    return leaves, freq


@dataclass
class LayerShape:
    experts: int
    top_k: int
    hidden: int
    inter: int
    group: int
    avg_bits: float = 2.5
    tokens: int = 1
    layers: int = 1
    extra: dict = field(default_factory=dict)


# The parity configurations (sizes from the pages' workload, see the module docstring).
SINGLE_MATRIX = dict(N=128, K=256, G=64)                      # one expert matrix, b swept 1..8
LAYER_SMALL = LayerShape(experts=64, top_k=8, hidden=2048, inter=768, group=128)
LAYER_LARGE = LayerShape(experts=512, top_k=10, hidden=4096, inter=1024, group=128)
LAYER_BATCHED = LayerShape(experts=512, top_k=10, hidden=4096, inter=1024, group=128, tokens=32,
                           extra=dict(zipf_s=1.1))
LAYER_CACHED = LayerShape(experts=512, top_k=10, hidden=4096, inter=1024, group=128, tokens=256,
                          layers=16, extra=dict(rho=0.8, cache_frac=0.4))
