"""Stacked MoE layers decoded through the HBM prefix cache.

Every layer's experts live in pinned host memory (all 8 planes); the device
holds a pool of plane slots shared by all layers and managed by the library's
cache (``pmoe_cache_*``: one shared prefix per (layer, expert), only missing
planes copied, deepest planes evicted first; PagedMoE transcript cues 11, 13,
35). A decode step of one token, per layer l:

  host: route (top-k + softmax) and select depths from the layer's logits,
        then ``cache.extend`` -- copies of the missing planes on a side stream;
  device: wait for the layer's copies, run ``pmoe_moe_layer_fwd`` on the
        cached planes, then ``pmoe_residual_norm`` (r += y, x = bf16(r/rms)).

The host plans all layers of a token before the device reaches them, so the
top-ups of layer l+1.. overlap the expert kernels of layer l. One token is
one cache batch: its entries are pinned while its layers run, and the copies
of a token that evicts wait for the previous token's kernels.

This module allocates (torch) and calls the C ABI; it computes nothing itself.
"""
from __future__ import annotations

import numpy as np
import torch

from . import Cache, make_layer, moe_layer_fwd, layer_workspace_bytes, residual_norm, route_host, \
    select_prefix_cache_aware_matched, layer_error


class CachedStack:
    def __init__(self, L, E, H, I, G, k, avg_bits, slots, backing_layers, sens, device="cuda",
                 keep_log=False, cache_aware=False):
        """backing_layers: ResidentLayers (device) whose planes back the layers, as a list or as
        (count, make) with make(b) building backing b on demand: layer l uses backing
        l % count (host planes, scales, codebooks). Each backing's device pool is copied to
        pinned host memory and then released (the list's own references aside).
        sens: per-layer host float32 arrays [E] (indexed l % len(sens))."""
        self.L, self.E, self.H, self.I, self.G, self.k, self.avg_bits = L, E, H, I, G, k, avg_bits
        dev = torch.device(device)
        self.dev = dev
        if isinstance(backing_layers, tuple):
            nb, make = backing_layers
        else:
            nb, make = len(backing_layers), backing_layers.__getitem__
        self.slot_words = 3 * H * I // 32
        self.slots = slots
        self.pool = torch.empty(slots * self.slot_words, dtype=torch.int32, device=dev)
        self.page_table = torch.full((L * E * 8,), -1, dtype=torch.int32, device=dev)
        self.cache = Cache(L, E, slots, self.slot_words, self.pool, self.page_table, keep_log=keep_log)
        self.host = []
        self.scales, self.codebooks = [], []
        for b in range(nb):
            R = make(b)
            h = torch.empty(E * 8 * self.slot_words, dtype=torch.int32).pin_memory()
            h.copy_(R.pool)
            self.host.append(h)
            self.scales.append(R.scales)
            self.codebooks.append(R.codebooks)
            del R
        self.cache.set_host_planes([self.host[l % nb] for l in range(L)])
        self.layers = [make_layer(E, H, I, G, self.pool, self.slot_words,
                                  self.page_table[l * E * 8:(l + 1) * E * 8], self.scales[l % nb],
                                  self.codebooks[l % nb]) for l in range(L)]
        self.sens = [np.ascontiguousarray(s, dtype=np.float32) for s in sens]
        # cache-aware selection (transcript cue 61): per token-layer, the planes the cache-oblivious
        # depths would fetch are the budget, and resident planes come free
        self.cache_aware = cache_aware
        self.keep_log = keep_log
        self._sur = np.zeros(2, np.float64)  # sum of (w s)^2 4^-b: cache-oblivious depths, depths used
        self.side = torch.cuda.Stream(dev)
        self.done = [torch.cuda.Event() for _ in range(L)]
        for e in self.done:  # torch creates the CUDA event at its first record; the library records it
            e.record(torch.cuda.current_stream(dev))
        # routing results: two pinned sets (alternating tokens) and their device copies
        self.ids_h = [torch.zeros(L, k, dtype=torch.int32).pin_memory() for _ in range(2)]
        self.w_h = [torch.zeros(L, k, dtype=torch.float32).pin_memory() for _ in range(2)]
        self.dep_h = [torch.zeros(L, k, dtype=torch.uint8).pin_memory() for _ in range(2)]
        self.set_free = [torch.cuda.Event(), torch.cuda.Event()]
        self.set_used = [False, False]
        self.ids_d = torch.zeros(L, k, dtype=torch.int32, device=dev)
        self.w_d = torch.zeros(L, k, dtype=torch.float32, device=dev)
        self.dep_d = torch.zeros(L, k, dtype=torch.uint8, device=dev)
        self.ws_bytes = layer_workspace_bytes(1, k, E, H, I)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.token_done = torch.cuda.Event()
        self.token_done_valid = False
        self.ntok = 0
        # trace of accesses, for the independent-precision comparison
        self.trace = []

    def _select(self, l, ids, w, dep):
        """Depths of layer l's slots (host arrays of one token). Cache-aware: resident planes are
        free and the budget is what the cache-oblivious depths would fetch. Otherwise the same
        call with nothing counted as resident, which is the plain allocator."""
        sens = self.sens[l % len(self.sens)]
        if self.cache_aware:
            res = np.ascontiguousarray(self.cache.resident_depth(l)[ids], dtype=np.uint8)
        else:
            res = np.zeros(self.k, np.uint8)
        select_prefix_cache_aware_matched(w, ids, sens, res, 1, self.k, self.avg_bits, dep, self._sur)

    def plan(self, logits, t):
        """Host routing for all layers of token t (logits: float32 [L, E]); returns the set."""
        s = self.ntok % 2
        if self.set_used[s]:
            self.set_free[s].synchronize()  # that set's device copies of two tokens ago are done
        ids, w = self.ids_h[s].numpy(), self.w_h[s].numpy()
        for l in range(self.L):
            route_host(np.ascontiguousarray(logits[l], dtype=np.float32), 1, self.E, self.k, ids[l], w[l])
        return s

    def decode_token(self, logits, r, x, y, t, stream=None, y_out=None):
        """One token through all layers. r: device float [H] (residual, updated), x: device bf16
        [H] (input of layer 0, then of each next layer), y: device float [H] scratch.
        y_out: optional device float [L, H] receiving each layer's y."""
        st = stream if stream is not None else torch.cuda.current_stream(self.dev)
        s = self.plan(logits, t)
        ids, w, dep = self.ids_h[s].numpy(), self.w_h[s].numpy(), self.dep_h[s].numpy()
        after = self.token_done if self.token_done_valid else None
        for l in range(self.L):
            self._select(l, ids[l], w[l], dep[l])
            self.cache.extend(l, ids[l], dep[l], t, side=self.side, after=after, done=self.done[l])
            for e, b in zip(ids[l], dep[l]):
                self.trace.append((l, int(e), int(b), t))
        with torch.cuda.stream(st):
            self.ids_d.copy_(self.ids_h[s], non_blocking=True)
            self.w_d.copy_(self.w_h[s], non_blocking=True)
            self.dep_d.copy_(self.dep_h[s], non_blocking=True)
            self.set_free[s].record(st)
            self.set_used[s] = True
            for l in range(self.L):
                st.wait_event(self.done[l])
                moe_layer_fwd(self.layers[l], x, self.ids_d[l], self.w_d[l], self.dep_d[l], 1, self.k, y,
                              self.ws, self.ws_bytes, st)
                if y_out is not None:
                    y_out[l].copy_(y)
                residual_norm(r, y, 1, self.H, x, st)
            self.token_done.record(st)
        self.token_done_valid = True
        self.ntok += 1
        return s

    def reset_cache(self):
        """A cold cache over the same pool and host planes (device work must be finished)."""
        torch.cuda.synchronize(self.dev)
        self.cache.close()
        self.cache = Cache(self.L, self.E, self.slots, self.slot_words, self.pool, self.page_table,
                           keep_log=self.keep_log)
        nb = len(self.host)
        self.cache.set_host_planes([self.host[l % nb] for l in range(self.L)])
        self.trace = []
        self._sur[:] = 0.0
        self.token_done_valid = False

    @property
    def surrogate(self):
        """[sum of (w s)^2 4^-b with the cache-oblivious depths, with the depths used]."""
        return [float(self._sur[0]), float(self._sur[1])]

    def routing(self, s):
        """Host copies (ids, w, depth) of the token planned into set s."""
        return self.ids_h[s].numpy().copy(), self.w_h[s].numpy().copy(), self.dep_h[s].numpy().copy()

    def check_errors(self):
        return layer_error(self.ws)

    def trace_arrays(self):
        a = np.array(self.trace, dtype=np.int64).reshape(-1, 4)
        return a[:, 0], a[:, 1], a[:, 2], a[:, 3]

    def close(self):
        torch.cuda.synchronize(self.dev)
        self.cache.close()
