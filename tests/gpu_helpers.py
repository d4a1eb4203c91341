"""Shared helpers of the GPU parity tests: seeded inputs on the device, the
oracle's view of the same weights, and the tolerance checks."""
from __future__ import annotations

import numpy as np
import torch

from mxfp4_moe_block_b200 import synth

# FFN tolerance (fp32 accumulation over exactly dequantised weights).
FFN_REL_L2 = 2e-3
FFN_MAX_ABS = 1e-2     # times max |reference|


def rel_l2(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def assert_ffn_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    r = rel_l2(got, ref)
    m = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    lim = FFN_MAX_ABS * float(np.max(np.abs(ref))) if ref.size else 0.0
    assert r <= FFN_REL_L2, f"{what}: rel-L2 {r:.3e} > {FFN_REL_L2}"
    assert m <= lim, f"{what}: max-abs {m:.3e} > {lim:.3e}"
    return r, m


def assert_route_weights(w_gpu, w64):
    """fp32 weights equal the oracle's, except where the oracle's double
    value sits within 2**-40 (relative) of the midpoint of two adjacent
    floats, where either neighbour is a correct rounding."""
    w_gpu = np.asarray(w_gpu, np.float32)
    w_or = w64.astype(np.float32)
    bad = w_gpu != w_or
    if not bad.any():
        return 0
    lo = np.minimum(w_gpu[bad], w_or[bad])
    hi = np.maximum(w_gpu[bad], w_or[bad])
    assert np.all(np.nextafter(lo, np.float32(np.inf)) == hi), "weights differ by more than 1 ulp"
    mid = (lo.astype(np.float64) + hi.astype(np.float64)) / 2
    assert np.all(np.abs(w64[bad] - mid) <= 2.0 ** -40 * mid), "mismatch away from a midpoint"
    return int(bad.sum())


def bf16_tensor(bits_u16: np.ndarray, device):
    return torch.from_numpy(bits_u16.astype(np.uint16).view(np.int16)).to(device).view(torch.bfloat16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class Layer:
    """One MoE layer's seeded inputs, on the device and for the oracle."""

    def __init__(self, sh: synth.Shape, layer: int, device, with_weights=True):
        self.sh, self.layer = sh, layer
        self.x_bits = synth.x_bf16_bits(sh, layer)
        self.x = bf16_tensor(self.x_bits, device)
        self.logits_np = synth.router_logits(sh, layer)
        self.logits = torch.from_numpy(self.logits_np).to(device)
        if with_weights:
            self.w = synth.weights_torch(sh, layer, device)

    def oracle_weights(self, e):
        sh, l = self.sh, self.layer
        return (synth.weight_codes_np(sh, "w13", e, l), synth.weight_scales_np(sh, "w13", e, l),
                synth.weight_codes_np(sh, "w2", e, l), synth.weight_scales_np(sh, "w2", e, l))

    def x_f64(self):
        return synth.bf16_bits_to_f32(self.x_bits).astype(np.float64)
