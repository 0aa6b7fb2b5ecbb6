"""Shared helpers of the GPU parity tests: seeded layers on both sides."""
import numpy as np
import torch

import oracle
import synth

REL_L2 = 1e-3       # relative L2 error bound on layer and GEMV outputs
MAX_ABS_RMS = 2e-3  # max abs error bound, as a fraction of the output RMS


def assert_close(y, ref, rel=REL_L2, max_abs_rms=MAX_ABS_RMS, msg=""):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert y.shape == ref.shape
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300))
    mx = float(np.max(np.abs(y - ref))) if y.size else 0.0
    assert err <= rel, f"{msg} relative L2 error {err:.3e} > {rel:.1e}"
    assert mx <= max_abs_rms * rms + 1e-30, f"{msg} max abs error {mx:.3e} > {max_abs_rms:.0e} * rms {rms:.3e}"
    return err, mx / max(rms, 1e-300)


def device_fill(seed, layer=0, stream=None):
    def fill(e, m, w):
        s = torch.cuda.current_stream() if stream is None else stream
        synth.expert_weights_device(seed, layer, e, m, w.numel(), w.data_ptr(), s.cuda_stream)
    return fill


class OracleExperts:
    """Oracle-side quantised experts, built lazily from the host generator."""

    def __init__(self, seed, H, I, G, layer=0):
        self.seed, self.H, self.I, self.G, self.layer = seed, H, I, G, layer
        self.cb = oracle.tree_codebook_f32()
        self.cache = {}

    def get(self, e):
        if e not in self.cache:
            codes, scales = [], []
            for m, (n, k) in enumerate(((self.I, self.H), (self.I, self.H), (self.H, self.I))):
                w = synth.expert_weights(self.seed, self.layer, e, m, n, k)
                s, c = oracle.quantize(w, self.G)
                codes.append(c)
                scales.append(s)
            self.cache[e] = oracle.Expert(codes, scales, [self.cb] * 3)
        return self.cache[e]

    def run(self, E, ids, w, depth, x64, bf16_weights=False):
        need = {int(e): self.get(int(e)) for e in np.unique(ids)}
        return oracle.moe_layer(need, E, self.H, self.I, self.G, ids, w, depth, x64, bf16_weights)


def tokens(seed, T, E, H, layer=0, token0=0, bias=None):
    logits = np.stack([synth.router_logits(seed, token0 + t, layer, E) for t in range(T)])
    if bias is not None:
        logits = (logits + bias[None, :]).astype(np.float32)
    xb = np.stack([synth.activation_bf16(seed, token0 + t, layer, H) for t in range(T)])
    return logits, xb
