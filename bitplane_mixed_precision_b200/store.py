"""Resident expert store of one MoE layer in HBM (torch owns the memory).

Builds the plane-slot pool that ``pmoe_layer`` describes: for every expert,
its gate, up and down matrices are quantised (``pmoe_quantize``) and packed
(``pmoe_pack_bitplanes``) straight into 8 slots, one per bitplane, each slot
holding [gate plane | up plane | down plane]. Weights come from a caller
callback; this module only allocates and calls the C ABI.
"""
from __future__ import annotations

import numpy as np
import torch

from . import Layer, make_layer, pack_bitplanes, quantize, tree_codebook

GATE, UP, DOWN = 0, 1, 2


class ResidentLayer:
    def __init__(self, E: int, H: int, I: int, G: int, fill, device="cuda", stream=None,
                 codebook: np.ndarray | None = None, experts=None):
        """fill(expert, mat, w) writes float32 weights of shape (rows*cols,) into device tensor w
        (gate/up: I x H, down: H x I). ``experts`` restricts which experts are built (others
        keep zero planes but valid slots)."""
        self.E, self.H, self.I, self.G = E, H, I, G
        self.mat_words = H * I // 32
        self.slot_words = 3 * self.mat_words
        self.scale_len = 2 * I * (H // G) + H * (I // G)
        dev = torch.device(device)
        self.pool = torch.zeros(E * 8 * self.slot_words, dtype=torch.int32, device=dev)
        self.scales = torch.zeros(E * self.scale_len, dtype=torch.float32, device=dev)
        if codebook is None:
            codebook = np.empty(510, dtype=np.float32)
            tree_codebook(codebook)
        self.codebook = torch.from_numpy(np.ascontiguousarray(codebook, dtype=np.float32))
        self.codebooks = self.codebook.to(dev).repeat(E * 3).contiguous()
        self.slot_of = torch.arange(E * 8, dtype=torch.int32, device=dev)
        w = torch.empty(H * I, dtype=torch.float32, device=dev)
        codes = torch.empty(H * I, dtype=torch.uint8, device=dev)
        st = stream if stream is not None else torch.cuda.current_stream(dev)
        for e in (range(E) if experts is None else experts):
            for m in (GATE, UP, DOWN):
                N, K = (I, H) if m != DOWN else (H, I)
                fill(e, m, w)
                soff = e * self.scale_len + (0 if m == GATE else I * (H // G) if m == UP else 2 * I * (H // G))
                sc = self.scales[soff: soff + N * (K // G)]
                quantize(w, N, K, G, sc, codes, st)
                base = self.pool[(e * 8) * self.slot_words + m * self.mat_words:]
                pack_bitplanes(codes, N, K, 8, base, self.slot_words, True, st)
        self.layer: Layer = make_layer(E, H, I, G, self.pool, self.slot_words, self.slot_of,
                                       self.scales, self.codebooks)

    def plane_bytes_per_expert_plane(self) -> int:
        return self.slot_words * 4

    def expert_scales(self, e: int, m: int) -> torch.Tensor:
        I, H, G = self.I, self.H, self.G
        soff = e * self.scale_len + (0 if m == GATE else I * (H // G) if m == UP else 2 * I * (H // G))
        N, K = (I, H) if m != DOWN else (H, I)
        return self.scales[soff: soff + N * (K // G)].view(N, K // G)
