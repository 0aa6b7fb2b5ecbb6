"""Offline error profiles of a resident layer's experts (PagedMoE transcript
cues 29-31), for the profile-driven allocator (``select_prefix_table``).

For every expert and depth b = 1..8 the layer call runs the expert alone
(top-1, weight 1) on the same random Gaussian inputs, and ``relative_error``
compares its output with the 8-bit output; ``profile_repair`` then makes each
profile's gains non-increasing. Allocation and calls only.
"""
from __future__ import annotations

import numpy as np
import torch

from . import layer_workspace_bytes, moe_layer_fwd, profile_repair, relative_error


def expert_profiles(R, x_bf16, experts=None, stream=None, repair=True):
    """R: ResidentLayer; x_bf16: device int16 [n, H] (bf16 inputs, e.g. 10 Gaussian vectors).
    Returns (raw, table): float32 [E][8] errors at depths 1..8 and the repaired table."""
    dev = x_bf16.device
    n, H = x_bf16.shape
    E, I = R.E, R.I
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    ws_bytes = layer_workspace_bytes(n, 1, E, H, I)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    w = torch.ones(n, dtype=torch.float32, device=dev)
    ys = torch.empty(8, n, H, dtype=torch.float32, device=dev)
    err = torch.zeros(E, 8, dtype=torch.float32, device=dev)
    depth = [torch.full((n,), b, dtype=torch.uint8, device=dev) for b in range(1, 9)]
    for e in (range(E) if experts is None else experts):
        ids = torch.full((n,), e, dtype=torch.int32, device=dev)
        for b in range(1, 9):
            moe_layer_fwd(R.layer, x_bf16, ids, w, depth[b - 1], n, 1, ys[b - 1], ws, ws_bytes, st)
        for b in range(1, 9):
            relative_error(ys[b - 1], ys[7], n, H, err[e, b - 1:], st)
    raw = err.cpu().numpy()
    table = raw.copy()
    if repair:
        profile_repair(raw, E, table)
    return raw, table
