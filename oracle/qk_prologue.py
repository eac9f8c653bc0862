"""fp64 CPU oracle of the QK-norm + rotary prologue -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may use it.

The LTX-2.5 DiT feeds attention with "normed and rotated" queries and keys and keeps
RoPE tables per latent grid ("feat(ltx2): tile-parallel video VAE and the two-stage
pipeline", commit "Onboard Lightricks LTX-2.5" and the two-stage DiT plan).  The pages fix
neither the norm nor the rotary layout; this module states the plainest reading and
computes it by its definition, in float64, with no blocking or reordering:

    for each batch element b and token l, over the token's whole inner dimension
    (heads * head_dim):
        r        = sqrt(mean_{h,d} x[b,l,h,d]^2 + eps)                        (RMSNorm)
        y[h, d]  = x[b,l,h,d] / r * weight[h * head_dim + d]
    then within every head, for each pair i of adjacent channels (2i, 2i+1):
        out[2i]   = y[2i] cos[l,i] - y[2i+1] sin[l,i]                          (rotary)
        out[2i+1] = y[2i] sin[l,i] + y[2i+1] cos[l,i]

Inputs are torch tensors (bf16 activations and weights, fp32 tables) widened to float64;
the output is a float64 numpy array shaped like x.
"""
from __future__ import annotations

import numpy as np


def rms_norm_rope(x, weight, cos, sin, eps: float) -> np.ndarray:
    xf = x.double().numpy()                                          # [B, L, H, D]
    b, l, h, d = xf.shape
    w = weight.double().numpy().reshape(h, d)
    c = cos.double().numpy()                                          # [L, D/2]
    s = sin.double().numpy()
    ms = np.mean(xf.reshape(b, l, h * d) ** 2, axis=2)                 # [B, L]
    r = np.sqrt(ms + eps)[:, :, None, None]
    y = xf / r * w[None, None, :, :]
    out = np.empty_like(y)
    a, bb = y[..., 0::2], y[..., 1::2]
    cc, ss = c[None, :, None, :], s[None, :, None, :]
    out[..., 0::2] = a * cc - bb * ss
    out[..., 1::2] = a * ss + bb * cc
    return out
