"""ORACLE — test infrastructure only.

Python access to the plain single-threaded C oracle in ``pmoe_oracle.c``
(double precision, no blocking, fusion or reordering beyond the method's own
definition). Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline leg may import this package. It shares no code with the CUDA
library in ``bitplane_mixed_precision_b200`` and never imports it.

Every function is pinned in ``tests/test_oracle_*.py`` to something other
than itself; see the header of each C function for the pins and the passage
of the PagedMoE pages it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libpmoe_oracle.so")
_SRC = os.path.join(_HERE, "pmoe_oracle.c")


def build(force: bool = False) -> None:
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", _SO, _SRC, "-lm"])


_lib = None


def _l():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        P = ctypes.c_void_p
        i32, i64, f32, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
        sig = {
            "or_norm_ppf": ([f64], f64),
            "or_tree_codebook": ([P], None),
            "or_tree_codebook_f32": ([P], None),
            "or_tree_from_leaves": ([P, P, P], None),
            "or_thresholds": ([P], None),
            "or_quantize": ([P, i32, i32, i32, P, P], None),
            "or_pack": ([P, i32, i32, i32, P], i32),
            "or_unpack": ([P, i32, i32, i32, P], i32),
            "or_gemv": ([P, P, P, i32, i32, i32, i32, P, P, i32], None),
            "or_route": ([P, i32, i32, i32, P, P], None),
            "or_budget": ([i32, f32], i32),
            "or_select": ([P, P, P, i32, i32, f32, P], i32),
            "or_moe_layer": ([i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, P, P, P, P, P,
                              i32], i32),
            "or_cache_sim_prefix": ([i32, i32, i64, i64, P, P, P, P, P, P, i64, P, P], i32),
            "or_cache_sim_independent": ([i32, i32, i64, i64, P, P, P, P, P, P], i32),
            "or_cache_sim_independent_down": ([i32, i32, i64, i64, P, P, P, P, P, P], i32),
            "or_select_cache_aware": ([P, P, P, P, i32, i32, i32, P], i32),
            "or_isotonic_nonincreasing": ([P, i32], None),
            "or_profile_repair": ([P, i32, P], None),
            "or_select_table": ([P, P, P, i32, i32, ctypes.c_float, P], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def norm_ppf(p: float) -> float:
    return _l().or_norm_ppf(p)


def tree_codebook() -> np.ndarray:
    """510 doubles: depth d (1..8) at offset 2^d - 2."""
    out = np.empty(510, dtype=np.float64)
    _l().or_tree_codebook(_p(out))
    return out


def tree_codebook_f32() -> np.ndarray:
    out = np.empty(510, dtype=np.float32)
    _l().or_tree_codebook_f32(_p(out))
    return out


def tree_from_leaves(leaves, freq) -> np.ndarray:
    """510 doubles: the tree over 256 sorted leaves, parents the frequency-weighted means."""
    leaves = np.ascontiguousarray(leaves, dtype=np.float64)
    freq = np.ascontiguousarray(freq, dtype=np.float64)
    assert leaves.shape == (256,) and freq.shape == (256,)
    out = np.empty(510, dtype=np.float64)
    _l().or_tree_from_leaves(_p(leaves), _p(freq), _p(out))
    return out


def level(cb: np.ndarray, d: int) -> np.ndarray:
    return cb[(1 << d) - 2:(1 << (d + 1)) - 2]


def thresholds() -> np.ndarray:
    out = np.empty(256, dtype=np.float64)
    _l().or_thresholds(_p(out))
    return out


def quantize(w: np.ndarray, G: int):
    """w float32 [N, K] -> (scales float32 [N, K/G], codes uint8 [N, K])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % G == 0
    scales = np.empty((N, K // G), dtype=np.float32)
    codes = np.empty((N, K), dtype=np.uint8)
    _l().or_quantize(_p(w), N, K, G, _p(scales), _p(codes))
    return scales, codes


def pack(codes: np.ndarray, depth: int = 8) -> np.ndarray:
    """codes uint8 [N, K] -> planes uint32 [depth, N*K/32]."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    out = np.empty((depth, N * K // 32), dtype=np.uint32)
    rc = _l().or_pack(_p(codes), N, K, depth, _p(out))
    if rc:
        raise ValueError("or_pack: bad shape or depth")
    return out


def unpack(planes: np.ndarray, N: int, K: int, b: int) -> np.ndarray:
    """b-bit prefix indices uint8 [N, K] read from planes 0..b-1."""
    planes = np.ascontiguousarray(planes, dtype=np.uint32)
    assert planes.shape[0] >= b and planes.shape[1] == N * K // 32
    out = np.empty((N, K), dtype=np.uint8)
    rc = _l().or_unpack(_p(planes), N, K, b, _p(out))
    if rc:
        raise ValueError("or_unpack: bad shape or depth")
    return out


def gemv(codes, scales, cb, G: int, b: int, x, bf16_weights: bool = False) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    cb = np.ascontiguousarray(cb, dtype=np.float32)
    x = np.ascontiguousarray(x, dtype=np.float64)
    N, K = codes.shape
    y = np.empty(N, dtype=np.float64)
    _l().or_gemv(_p(codes), _p(scales), _p(cb), N, K, G, b, _p(x), _p(y), int(bf16_weights))
    return y


def route(logits: np.ndarray, k: int):
    """logits float32 [T, E] -> (ids int32 [T, k], w float32 [T, k])."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float32)
    _l().or_route(_p(logits), T, E, k, _p(ids), _p(w))
    return ids, w


def budget(k: int, avg_bits: float) -> int:
    return _l().or_budget(k, avg_bits)


def select(w: np.ndarray, ids: np.ndarray, sens: np.ndarray, avg_bits: float) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.float32)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    sens = np.ascontiguousarray(sens, dtype=np.float32)
    T, k = w.shape
    out = np.empty((T, k), dtype=np.uint8)
    rc = _l().or_select(_p(w), _p(ids), _p(sens), T, k, avg_bits, _p(out))
    if rc:
        raise ValueError("or_select: bad arguments")
    return out


def select_cache_aware(w: np.ndarray, ids: np.ndarray, sens: np.ndarray, resident: np.ndarray,
                       fetch: int) -> np.ndarray:
    """Depths under a budget of fetched planes per token, resident planes free."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    sens = np.ascontiguousarray(sens, dtype=np.float32)
    resident = np.ascontiguousarray(resident, dtype=np.uint8)
    T, k = w.shape
    out = np.empty((T, k), dtype=np.uint8)
    rc = _l().or_select_cache_aware(_p(w), _p(ids), _p(sens), _p(resident), T, k, int(fetch), _p(out))
    if rc:
        raise ValueError("or_select_cache_aware: bad arguments")
    return out


def isotonic_nonincreasing(g) -> np.ndarray:
    g = np.array(g, dtype=np.float64)
    _l().or_isotonic_nonincreasing(_p(g), len(g))
    return g


def profile_repair(raw) -> np.ndarray:
    """raw: [n][8] errors at depths 1..8 -> repaired table [n][8]."""
    raw = np.ascontiguousarray(raw, dtype=np.float64)
    out = np.empty_like(raw)
    _l().or_profile_repair(_p(raw), raw.shape[0], _p(out))
    return out


def select_table(w: np.ndarray, ids: np.ndarray, table: np.ndarray, avg_bits: float) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.float32)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    table = np.ascontiguousarray(table, dtype=np.float32)
    T, k = w.shape
    out = np.empty((T, k), dtype=np.uint8)
    rc = _l().or_select_table(_p(w), _p(ids), _p(table), T, k, avg_bits, _p(out))
    if rc:
        raise ValueError("or_select_table: bad arguments")
    return out


def expert_profile(expert: "Expert", E: int, H: int, I: int, G: int, xs: np.ndarray) -> np.ndarray:
    """Relative output error of one expert at depths 1..8 against depth 8, averaged over the rows
    of xs (double); the dequantise-then-matvec layer with this expert alone at weight 1."""
    errs = np.zeros(8)
    need = {0: expert}
    ids = np.zeros((xs.shape[0], 1), np.int32)
    w = np.ones((xs.shape[0], 1), np.float32)
    ref = moe_layer(need, E, H, I, G, ids, w, np.full((xs.shape[0], 1), 8, np.uint8), xs)
    for b in range(1, 9):
        y = moe_layer(need, E, H, I, G, ids, w, np.full((xs.shape[0], 1), b, np.uint8), xs)
        errs[b - 1] = float(np.mean(np.sum((y - ref) ** 2, axis=1) / np.sum(ref ** 2, axis=1)))
    return errs


class Expert:
    """Quantised expert: codes, scales and codebook for gate, up, down."""

    def __init__(self, codes, scales, cbs):
        self.codes = [np.ascontiguousarray(c, dtype=np.uint8) for c in codes]
        self.scales = [np.ascontiguousarray(s, dtype=np.float32) for s in scales]
        self.cbs = [np.ascontiguousarray(c, dtype=np.float32) for c in cbs]


def moe_layer(experts: dict, E: int, H: int, I: int, G: int, ids, w, depth, x,
              bf16_weights: bool = False) -> np.ndarray:
    """experts: {expert id: Expert}; x float64 [T, H] -> y float64 [T, H]."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    depth = np.ascontiguousarray(depth, dtype=np.uint8)
    x = np.ascontiguousarray(x, dtype=np.float64)
    T, k = ids.shape
    arrs = []
    for m in range(3):
        for kind in ("codes", "scales", "cbs"):
            a = (ctypes.c_void_p * E)()
            for e, ex in experts.items():
                a[e] = getattr(ex, kind)[m].ctypes.data
            arrs.append((m, kind, a))
    get = {(m, kind): a for m, kind, a in arrs}
    y = np.empty((T, H), dtype=np.float64)
    rc = _l().or_moe_layer(T, k, H, I, G,
                           ctypes.cast(get[(0, "codes")], ctypes.c_void_p),
                           ctypes.cast(get[(1, "codes")], ctypes.c_void_p),
                           ctypes.cast(get[(2, "codes")], ctypes.c_void_p),
                           ctypes.cast(get[(0, "scales")], ctypes.c_void_p),
                           ctypes.cast(get[(1, "scales")], ctypes.c_void_p),
                           ctypes.cast(get[(2, "scales")], ctypes.c_void_p),
                           ctypes.cast(get[(0, "cbs")], ctypes.c_void_p),
                           ctypes.cast(get[(1, "cbs")], ctypes.c_void_p),
                           ctypes.cast(get[(2, "cbs")], ctypes.c_void_p),
                           _p(ids), _p(w), _p(depth), _p(x), _p(y), int(bf16_weights))
    if rc:
        raise ValueError(f"or_moe_layer failed ({rc}): missing expert or allocation")
    return y


def cache_sim_prefix(L: int, E: int, cap_planes: int, layer, expert, depth, batch,
                     evict_cap: int = 1 << 22):
    layer = np.ascontiguousarray(layer, dtype=np.int32)
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    depth = np.ascontiguousarray(depth, dtype=np.uint8)
    batch = np.ascontiguousarray(batch, dtype=np.int32)
    n = len(layer)
    before = np.empty(n, dtype=np.uint8)
    log = np.empty(evict_cap, dtype=np.int64)
    nev = ctypes.c_int64(0)
    fetched = ctypes.c_int64(0)
    rc = _l().or_cache_sim_prefix(L, E, cap_planes, n, _p(layer), _p(expert), _p(depth), _p(batch),
                                  _p(before), _p(log), evict_cap, ctypes.byref(nev),
                                  ctypes.byref(fetched))
    if rc:
        raise ValueError(f"or_cache_sim_prefix failed ({rc})")
    return before, log[:min(nev.value, evict_cap)].copy(), fetched.value


def cache_sim_independent(L: int, E: int, cap_planes: int, layer, expert, depth, batch):
    layer = np.ascontiguousarray(layer, dtype=np.int32)
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    depth = np.ascontiguousarray(depth, dtype=np.uint8)
    batch = np.ascontiguousarray(batch, dtype=np.int32)
    n = len(layer)
    hit = np.empty(n, dtype=np.uint8)
    fetched = ctypes.c_int64(0)
    rc = _l().or_cache_sim_independent(L, E, cap_planes, n, _p(layer), _p(expert), _p(depth),
                                       _p(batch), _p(hit), ctypes.byref(fetched))
    if rc:
        raise ValueError(f"or_cache_sim_independent failed ({rc})")
    return hit, fetched.value


def cache_sim_independent_down(L: int, E: int, cap_planes: int, layer, expert, depth, batch):
    """Independent objects with downward reuse: (hit uint8 [n], planes fetched)."""
    layer = np.ascontiguousarray(layer, dtype=np.int32)
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    depth = np.ascontiguousarray(depth, dtype=np.uint8)
    batch = np.ascontiguousarray(batch, dtype=np.int32)
    n = len(layer)
    hit = np.empty(n, dtype=np.uint8)
    fetched = ctypes.c_int64(0)
    rc = _l().or_cache_sim_independent_down(L, E, cap_planes, n, _p(layer), _p(expert), _p(depth),
                                            _p(batch), _p(hit), ctypes.byref(fetched))
    if rc:
        raise ValueError(f"or_cache_sim_independent_down failed ({rc})")
    return hit, fetched.value
