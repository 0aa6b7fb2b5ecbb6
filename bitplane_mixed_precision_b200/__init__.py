"""Python binding of libpmoe (bitplane-prefix MoE expert execution on B200).

Argument marshalling only: every function forwards to the C ABI declared in
``include/pmoe.h`` under the same name (without the ``pmoe_`` prefix) and
raises :class:`PmoeError` on a non-OK status. Pointers may be given as torch
tensors, numpy arrays or integers. There is no fallback: importing this
package fails if ``libpmoe.so`` has not been built (``build.build()``).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpmoe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libpmoe.so is missing at {LIB_PATH}; build it with "
                      "`python bitplane_mixed_precision_b200/build.py` or __graft_entry__.build()")

_lib = ctypes.CDLL(LIB_PATH)

P = ctypes.c_void_p
i32, i64, f32, sz = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


class Matrix(ctypes.Structure):
    """pmoe_matrix: one stored expert matrix (device pointers)."""
    _fields_ = [("planes", P), ("plane_stride_words", i64), ("scales", P), ("codebook", P),
                ("N", i32), ("K", i32), ("G", i32)]


class Layer(ctypes.Structure):
    """pmoe_layer: one MoE layer's experts in a plane-slot pool (device pointers)."""
    _fields_ = [("E", i32), ("H", i32), ("I", i32), ("G", i32), ("pool", P), ("slot_words", i64),
                ("slot_of", P), ("scales", P), ("codebooks", P)]


class CacheStats(ctypes.Structure):
    """pmoe_cache_stats: accumulated prefix-cache counters."""
    _fields_ = [("requests", i64), ("hits", i64), ("planes_fetched", i64), ("bytes_fetched", i64),
                ("planes_evicted", i64)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


_SIGS = {
    "pmoe_status_string": ([i32], ctypes.c_char_p),
    "pmoe_last_cuda_error": ([], i32),
    "pmoe_version": ([], i32),
    "pmoe_tree_codebook": ([P], i32),
    "pmoe_tree_codebook_from_leaves": ([P, P, P], i32),
    "pmoe_quantize": ([P, i32, i32, i32, P, P, P], i32),
    "pmoe_pack_bitplanes": ([P, i32, i32, i32, P, i64, i32, P], i32),
    "pmoe_extract_prefix": ([P, i64, i32, i32, i32, P, P], i32),
    "pmoe_route": ([P, i32, i32, i32, P, P, P], i32),
    "pmoe_select_prefix": ([P, P, P, i32, i32, f32, P, i32, P], i32),
    "pmoe_select_prefix_cache_aware": ([P, P, P, P, i32, i32, i32, P], i32),
    "pmoe_select_prefix_cache_aware_matched": ([P, P, P, P, i32, i32, f32, P, P], i32),
    "pmoe_relative_error": ([P, P, i32, i32, P, P], i32),
    "pmoe_profile_repair": ([P, i32, P], i32),
    "pmoe_select_prefix_table": ([P, P, P, i32, i32, f32, P, i32, P], i32),
    "pmoe_expert_gemv": ([ctypes.POINTER(Matrix), i32, P, i32, P, P], i32),
    "pmoe_layer_workspace_bytes": ([i32, i32, i32, i32, i32], sz),
    "pmoe_decode_host_workspace_bytes": ([i32, i32, i32, i32, i32], sz),
    "pmoe_moe_decode_step_host": ([ctypes.POINTER(Layer), P, P, P, i32, i32, f32, P, P, sz, P], i32),
    "pmoe_moe_layer_fwd": ([ctypes.POINTER(Layer), P, P, P, P, i32, i32, P, P, sz, P], i32),
    "pmoe_moe_decode_step": ([ctypes.POINTER(Layer), P, P, P, i32, i32, f32, P, P, P, P, P, sz, P],
                             i32),
    "pmoe_profile_events": ([P, P], i32),
    "pmoe_noalloc_scratch_bytes": ([], sz),
    "pmoe_noalloc_layer_error": ([ctypes.POINTER(i32), ctypes.POINTER(i32), P], i32),
    "pmoe_moe_layer_fwd_noalloc": ([ctypes.POINTER(Layer), P, P, P, P, i32, i32, P, P], i32),
    "pmoe_layer_error": ([P, ctypes.POINTER(i32), ctypes.POINTER(i32), P], i32),
    "pmoe_layer_counts": ([P, P, P], i32),
    "pmoe_set_tc_min_tokens": ([i32], i32),
    "pmoe_tc_selfcheck": ([P, P, P, i32, i32, P], i32),
    "pmoe_set_wait_limit_ns": ([ctypes.c_uint64], i32),
    "pmoe_materialise_workspace_bytes": ([i32, i32, i32, i32, i32], sz),
    "pmoe_materialise_layer_fwd": ([ctypes.POINTER(Layer), P, P, P, P, i32, i32, P, P, sz, P], i32),
    "pmoe_cache_create": ([i32, i32, i64, i64, P, P, i32, ctypes.POINTER(P)], i32),
    "pmoe_cache_extend": ([P, i32, P, P, i32, i64, P, P, P, P, P, ctypes.POINTER(CacheStats)], i32),
    "pmoe_cache_get_stats": ([P, ctypes.POINTER(CacheStats)], i32),
    "pmoe_cache_inject_copy_failure": ([P, i64], i32),
    "pmoe_cache_resident_depth": ([P, i32, P], i32),
    "pmoe_cache_eviction_log": ([P, P, i64, ctypes.POINTER(i64)], i32),
    "pmoe_cache_destroy": ([P], i32),
    "pmoe_cache_sim_independent": ([i32, i32, i64, i64, P, P, P, P, P, ctypes.POINTER(i64)], i32),
    "pmoe_cache_sim_independent_down": ([i32, i32, i64, i64, P, P, P, P, P, ctypes.POINTER(i64)], i32),
    "pmoe_route_host": ([P, i32, i32, i32, P, P], i32),
    "pmoe_residual_norm": ([P, P, i32, i32, P, P], i32),
}

for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


def exported_symbols():
    """Names the binding resolves in libpmoe.so (each must exist)."""
    return sorted(_SIGS)


class PmoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        msg = _lib.pmoe_status_string(code).decode()
        if code == 2:
            msg += f" (cudaError {_lib.pmoe_last_cuda_error()})"
        super().__init__(f"{fn}: {msg}")
        self.code = code


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    raise TypeError(f"cannot take a pointer of {type(x)}")


def _stream(s):
    if s is None:
        return None
    if hasattr(s, "cuda_stream"):
        return s.cuda_stream
    return int(s)


def _check(fn, rc):
    if rc != 0:
        raise PmoeError(fn, rc)


def version() -> int:
    return _lib.pmoe_version()


def tree_codebook(out) -> None:
    _check("pmoe_tree_codebook", _lib.pmoe_tree_codebook(_ptr(out)))


def tree_codebook_from_leaves(leaves, freq, out) -> None:
    """Host float32 arrays: 256 sorted leaves, 256 frequencies -> 510-entry tree."""
    _check("pmoe_tree_codebook_from_leaves", _lib.pmoe_tree_codebook_from_leaves(_ptr(leaves), _ptr(freq),
                                                                               _ptr(out)))


def quantize(w, N, K, G, scales, codes, stream=None) -> None:
    _check("pmoe_quantize", _lib.pmoe_quantize(_ptr(w), N, K, G, _ptr(scales), _ptr(codes), _stream(stream)))


def pack_bitplanes(codes, N, K, depth, planes, plane_stride_words, on_device=True, stream=None) -> None:
    _check("pmoe_pack_bitplanes", _lib.pmoe_pack_bitplanes(_ptr(codes), N, K, depth, _ptr(planes),
                                                           plane_stride_words, int(on_device),
                                                           _stream(stream)))


def extract_prefix(planes, plane_stride_words, N, K, b, idx, stream=None) -> None:
    _check("pmoe_extract_prefix", _lib.pmoe_extract_prefix(_ptr(planes), plane_stride_words, N, K, b,
                                                           _ptr(idx), _stream(stream)))


def route(logits, T, E, k, ids, w, stream=None) -> None:
    _check("pmoe_route", _lib.pmoe_route(_ptr(logits), T, E, k, _ptr(ids), _ptr(w), _stream(stream)))


def select_prefix(w, ids, sens, T, k, avg_bits, depth, on_device=True, stream=None) -> None:
    _check("pmoe_select_prefix", _lib.pmoe_select_prefix(_ptr(w), _ptr(ids), _ptr(sens), T, k, avg_bits,
                                                         _ptr(depth), int(on_device), _stream(stream)))


def select_prefix_cache_aware(w, ids, sens, resident, T, k, fetch_budget, depth) -> None:
    """Host arrays; depths under a budget of fetched planes per token (resident planes free)."""
    _check("pmoe_select_prefix_cache_aware", _lib.pmoe_select_prefix_cache_aware(
        _ptr(w), _ptr(ids), _ptr(sens), _ptr(resident), T, k, int(fetch_budget), _ptr(depth)))


def select_prefix_cache_aware_matched(w, ids, sens, resident, T, k, avg_bits, depth, surrogate=None) -> None:
    """Host arrays; the cache-aware depths with the cache-oblivious depths' fetch count as budget.
    surrogate: optional float64 numpy [2] accumulating sum (w s)^2 4^-b (oblivious, returned)."""
    _check("pmoe_select_prefix_cache_aware_matched", _lib.pmoe_select_prefix_cache_aware_matched(
        _ptr(w), _ptr(ids), _ptr(sens), _ptr(resident), T, k, avg_bits, _ptr(depth), _ptr(surrogate)))


def relative_error(y, ref, T, H, err, stream=None) -> None:
    _check("pmoe_relative_error", _lib.pmoe_relative_error(_ptr(y), _ptr(ref), T, H, _ptr(err), _stream(stream)))


def profile_repair(raw, n, table) -> None:
    _check("pmoe_profile_repair", _lib.pmoe_profile_repair(_ptr(raw), n, _ptr(table)))


def select_prefix_table(w, ids, table, T, k, avg_bits, depth, on_device=True, stream=None) -> None:
    _check("pmoe_select_prefix_table", _lib.pmoe_select_prefix_table(
        _ptr(w), _ptr(ids), _ptr(table), T, k, avg_bits, _ptr(depth), int(on_device), _stream(stream)))


def make_matrix(planes, plane_stride_words, scales, codebook, N, K, G) -> Matrix:
    return Matrix(_ptr(planes), plane_stride_words, _ptr(scales), _ptr(codebook), N, K, G)


def expert_gemv(m: Matrix, b, x, x_is_bf16, y, stream=None) -> None:
    _check("pmoe_expert_gemv", _lib.pmoe_expert_gemv(ctypes.byref(m), b, _ptr(x), int(x_is_bf16), _ptr(y),
                                                     _stream(stream)))


def make_layer(E, H, I, G, pool, slot_words, slot_of, scales, codebooks) -> Layer:
    return Layer(E, H, I, G, _ptr(pool), slot_words, _ptr(slot_of), _ptr(scales), _ptr(codebooks))


def layer_workspace_bytes(T, k, E, H, I) -> int:
    return _lib.pmoe_layer_workspace_bytes(T, k, E, H, I)


def moe_layer_fwd(L: Layer, x, ids, w, depth, T, k, y, ws, ws_bytes, stream=None) -> None:
    _check("pmoe_moe_layer_fwd", _lib.pmoe_moe_layer_fwd(ctypes.byref(L), _ptr(x), _ptr(ids), _ptr(w),
                                                         _ptr(depth), T, k, _ptr(y), _ptr(ws), ws_bytes,
                                                         _stream(stream)))


def noalloc_scratch_bytes() -> int:
    return _lib.pmoe_noalloc_scratch_bytes()


def noalloc_layer_error(stream=None):
    """(code, detail) of the error record in the allocation-free call's array (synchronises)."""
    code, detail = i32(0), i32(0)
    _check("pmoe_noalloc_layer_error", _lib.pmoe_noalloc_layer_error(ctypes.byref(code), ctypes.byref(detail),
                                                                     _stream(stream)))
    return code.value, detail.value


def moe_layer_fwd_noalloc(L: Layer, x, ids, w, depth, T, k, y, stream=None) -> None:
    """pmoe_moe_layer_fwd with the library's fixed scratch array instead of a workspace."""
    _check("pmoe_moe_layer_fwd_noalloc", _lib.pmoe_moe_layer_fwd_noalloc(
        ctypes.byref(L), _ptr(x), _ptr(ids), _ptr(w), _ptr(depth), T, k, _ptr(y), _stream(stream)))


def moe_decode_step(L: Layer, logits, sens, x, T, k, avg_bits, y, ids_out, w_out, depth_out, ws,
                    ws_bytes, stream=None) -> None:
    _check("pmoe_moe_decode_step", _lib.pmoe_moe_decode_step(
        ctypes.byref(L), _ptr(logits), _ptr(sens), _ptr(x), T, k, avg_bits, _ptr(y), _ptr(ids_out),
        _ptr(w_out), _ptr(depth_out), _ptr(ws), ws_bytes, _stream(stream)))


def decode_host_workspace_bytes(T, k, E, H, I) -> int:
    return _lib.pmoe_decode_host_workspace_bytes(T, k, E, H, I)


def moe_decode_step_host(L: Layer, logits, sens, x, T, k, avg_bits, y, ws, ws_bytes, stream=None) -> None:
    """The decode step with logits, x and y in (pinned) host memory: one call queues the input
    copies, the step and the output copy on the stream."""
    _check("pmoe_moe_decode_step_host", _lib.pmoe_moe_decode_step_host(
        ctypes.byref(L), _ptr(logits), _ptr(sens), _ptr(x), T, k, avg_bits, _ptr(y), _ptr(ws), ws_bytes,
        _stream(stream)))


def profile_events(start, stop) -> None:
    """start/stop: torch.cuda.Event (or raw cudaEvent_t ints); None, None disables."""
    def h(e):
        if e is None:
            return None
        return e.cuda_event if hasattr(e, "cuda_event") else int(e)
    _check("pmoe_profile_events", _lib.pmoe_profile_events(h(start), h(stop)))


def set_wait_limit_ns(ns) -> None:
    """Bound of the layer kernels' device waits (0 = the default, 200 ms)."""
    _check("pmoe_set_wait_limit_ns", _lib.pmoe_set_wait_limit_ns(int(ns)))


def layer_error(ws, stream=None):
    """(code, detail) of the device-side error record in a layer workspace (synchronises)."""
    code, detail = i32(0), i32(0)
    _check("pmoe_layer_error", _lib.pmoe_layer_error(_ptr(ws), ctypes.byref(code), ctypes.byref(detail),
                                                     _stream(stream)))
    return code.value, detail.value


def layer_counts(ws, stream=None):
    """(column blocks, expert units, tensor-core units, tensor-core operand rows) of the last layer
    call on workspace ws (synchronises)."""
    out = (i32 * 4)()
    _check("pmoe_layer_counts", _lib.pmoe_layer_counts(_ptr(ws), out, _stream(stream)))
    return tuple(out)


def set_tc_min_tokens(n) -> None:
    """Pairs at depth <= 4 an expert needs in one call before the tensor cores take them (>= 8; 0: never)."""
    _check("pmoe_set_tc_min_tokens", _lib.pmoe_set_tc_min_tokens(int(n)))


def tc_selfcheck(A, B, D, N, K, stream=None) -> None:
    """D[128 x N] = A[128 x K] * B[N x K]^T through the tensor-core operand path (f16 bit patterns as
    int16 tensors, D fp32)."""
    _check("pmoe_tc_selfcheck", _lib.pmoe_tc_selfcheck(_ptr(A), _ptr(B), _ptr(D), N, K, _stream(stream)))


def materialise_workspace_bytes(T, k, E, H, I) -> int:
    return _lib.pmoe_materialise_workspace_bytes(T, k, E, H, I)


def materialise_layer_fwd(L: Layer, x, ids, w, depth, T, k, y, ws, ws_bytes, stream=None) -> None:
    _check("pmoe_materialise_layer_fwd", _lib.pmoe_materialise_layer_fwd(
        ctypes.byref(L), _ptr(x), _ptr(ids), _ptr(w), _ptr(depth), T, k, _ptr(y), _ptr(ws), ws_bytes,
        _stream(stream)))


def route_host(logits, T, E, k, ids, w) -> None:
    """pmoe_route on host arrays (numpy), synchronous."""
    _check("pmoe_route_host", _lib.pmoe_route_host(_ptr(logits), T, E, k, _ptr(ids), _ptr(w)))


def residual_norm(r, y, T, H, x, stream=None) -> None:
    _check("pmoe_residual_norm", _lib.pmoe_residual_norm(_ptr(r), _ptr(y), T, H, _ptr(x), _stream(stream)))


def _event(e):
    if e is None:
        return None
    return e.cuda_event if hasattr(e, "cuda_event") else int(e)


class Cache:
    """pmoe_cache handle: the HBM prefix cache (host state in the library).

    pool / page_table: device tensors the caller keeps alive (both None for a
    host-only cache that only takes decisions)."""

    def __init__(self, layers, experts, slots, slot_words, pool=None, page_table=None, keep_log=False):
        h = P()
        _check("pmoe_cache_create", _lib.pmoe_cache_create(layers, experts, slots, slot_words, _ptr(pool),
                                                           _ptr(page_table), int(keep_log), ctypes.byref(h)))
        self._h = h
        self.layers, self.experts, self.slots, self.slot_words = layers, experts, slots, slot_words
        self._host_ptrs = None

    def set_host_planes(self, ptrs):
        """ptrs: one pinned host pointer (int or tensor) per layer."""
        arr = (P * self.layers)(*[_ptr(p) for p in ptrs])
        self._host_ptrs = arr

    def extend(self, layer, experts, need, batch, side=None, after=None, done=None, resident_before=None):
        """experts: int32 numpy [n]; need: uint8 numpy [n]. Returns CacheStats (accumulated)."""
        import numpy as np
        experts = np.ascontiguousarray(experts, dtype=np.int32)
        need = np.ascontiguousarray(need, dtype=np.uint8)
        st = CacheStats()
        _check("pmoe_cache_extend", _lib.pmoe_cache_extend(
            self._h, layer, _ptr(experts), _ptr(need), len(experts), int(batch), self._host_ptrs,
            _stream(side), _event(after), _event(done), _ptr(resident_before), ctypes.byref(st)))
        return st

    def inject_copy_failure(self, nth):
        """Testing hook: the nth next plane copy reports failure (0 disarms)."""
        _check("pmoe_cache_inject_copy_failure", _lib.pmoe_cache_inject_copy_failure(self._h, int(nth)))

    def stats(self):
        st = CacheStats()
        _check("pmoe_cache_get_stats", _lib.pmoe_cache_get_stats(self._h, ctypes.byref(st)))
        return st

    def resident_depth(self, layer):
        import numpy as np
        d = np.zeros(self.experts, dtype=np.uint8)
        _check("pmoe_cache_resident_depth", _lib.pmoe_cache_resident_depth(self._h, layer, _ptr(d)))
        return d

    def eviction_log(self):
        import numpy as np
        n = i64(0)
        _check("pmoe_cache_eviction_log", _lib.pmoe_cache_eviction_log(self._h, None, 0, ctypes.byref(n)))
        out = np.zeros(max(n.value, 1), dtype=np.int64)
        _check("pmoe_cache_eviction_log", _lib.pmoe_cache_eviction_log(self._h, _ptr(out), n.value,
                                                                       ctypes.byref(n)))
        return out[:n.value]

    def close(self):
        if self._h:
            _check("pmoe_cache_destroy", _lib.pmoe_cache_destroy(self._h))
            self._h = P()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def cache_sim_independent(layers, experts, cap_planes, layer, expert, need, batch):
    """Independent-precision baseline on a trace: (hit uint8 [n], planes_fetched)."""
    import numpy as np
    layer = np.ascontiguousarray(layer, dtype=np.int32)
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    need = np.ascontiguousarray(need, dtype=np.uint8)
    batch = np.ascontiguousarray(batch, dtype=np.int64)
    hit = np.zeros(len(layer), dtype=np.uint8)
    fetched = i64(0)
    _check("pmoe_cache_sim_independent", _lib.pmoe_cache_sim_independent(
        layers, experts, cap_planes, len(layer), _ptr(layer), _ptr(expert), _ptr(need), _ptr(batch),
        _ptr(hit), ctypes.byref(fetched)))
    return hit, fetched.value


def cache_sim_independent_down(layers, experts, cap_planes, layer, expert, need, batch):
    """Independent objects with downward reuse on a trace: (hit uint8 [n], planes_fetched)."""
    import numpy as np
    layer = np.ascontiguousarray(layer, dtype=np.int32)
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    need = np.ascontiguousarray(need, dtype=np.uint8)
    batch = np.ascontiguousarray(batch, dtype=np.int64)
    hit = np.zeros(len(layer), dtype=np.uint8)
    fetched = i64(0)
    _check("pmoe_cache_sim_independent_down", _lib.pmoe_cache_sim_independent_down(
        layers, experts, cap_planes, len(layer), _ptr(layer), _ptr(expert), _ptr(need), _ptr(batch),
        _ptr(hit), ctypes.byref(fetched)))
    return hit, fetched.value
