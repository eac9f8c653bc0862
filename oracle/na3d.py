"""fp64 CPU oracle of 3-D neighbourhood attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may use it.

The LTX-2.5 diffusion decoder runs 3-D neighbourhood attention in its stages, through
NATTEN's fused ``na3d`` kernel or a FlexAttention block-mask fallback that agrees with it
to bf16 rounding ("LTX2.5", SGLang Diffusion cookbook, §4.6 Diffusion decoder).  The page
gives neither the grid nor the window, so this module takes the neighbourhood of
Neighborhood Attention as published (Hassani et al., "Neighborhood Attention
Transformer", CVPR 2023), in 3-D, without dilation and without causal masking:

    tokens sit on a T x Y x X grid in raster order, n = (t * Y + y) * X + x;
    along an axis of length N with odd window k <= N, the query at i sees the k
    positions starting at  s(i) = min(max(i - (k - 1) / 2, 0), N - k)
    (centred, shifted inward at the borders so that every query sees exactly k);
    the neighbourhood is the box of the three axes' windows;
    out[n] = sum_{m in nbhd(n)} softmax_m(scale * q[n] . k[m]) v[m]   per (batch, head).

Inputs are torch tensors (bf16) in [batch, T*Y*X, heads, head_dim] layout, widened to
float64; outputs are float64 numpy arrays.  The arithmetic is the definition above with
numpy gathers and sums, no blocking or reordering beyond processing query rows in chunks.
"""
from __future__ import annotations

import numpy as np
import torch


def window_start(i: np.ndarray, k: int, n: int) -> np.ndarray:
    """First position of the length-k window of positions i on an axis of length n."""
    return np.minimum(np.maximum(i - (k - 1) // 2, 0), n - k)


def check_shape(grid, kernel) -> None:
    for n, k in zip(grid, kernel):
        if n < 1 or k < 1 or k % 2 == 0 or k > n:
            raise ValueError(f"window {kernel} on grid {grid}: each k odd, 1 <= k <= n")


def neighbours(rows: np.ndarray, grid, kernel) -> np.ndarray:
    """[len(rows), kT*kY*kX] token indices of each query's neighbourhood (raster order)."""
    t_n, y_n, x_n = grid
    k_t, k_y, k_x = kernel
    rows = np.asarray(rows, dtype=np.int64)
    t, rem = np.divmod(rows, y_n * x_n)
    y, x = np.divmod(rem, x_n)
    st, sy, sx = window_start(t, k_t, t_n), window_start(y, k_y, y_n), window_start(x, k_x, x_n)
    a = np.arange(k_t)[None, :, None, None]
    b = np.arange(k_y)[None, None, :, None]
    c = np.arange(k_x)[None, None, None, :]
    idx = ((st[:, None, None, None] + a) * y_n + (sy[:, None, None, None] + b)) * x_n \
        + (sx[:, None, None, None] + c)
    return idx.reshape(len(rows), k_t * k_y * k_x)


def na3d(q, k, v, grid, kernel, scale: float, rows=None, chunk: int = 2048) -> np.ndarray:
    """Neighbourhood attention of every (batch, head); `rows` selects query tokens.

    Returns float64 [batch, len(rows), heads, head_dim] (all tokens when rows is None).
    """
    check_shape(grid, kernel)
    bsz, n_tok, heads, d = q.shape
    assert n_tok == grid[0] * grid[1] * grid[2], "sequence length = T * Y * X"
    rows = np.arange(n_tok) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.empty((bsz, len(rows), heads, d))
    for lo in range(0, len(rows), chunk):
        r = rows[lo:lo + chunk]
        idx = neighbours(r, grid, kernel)                      # [R, K]
        rt, it = torch.from_numpy(r), torch.from_numpy(idx)
        for b in range(bsz):
            # only the rows this chunk needs are widened to float64
            qs = q[b][rt].double().numpy()                     # [R, H, D]
            ks = k[b][it].double().numpy()                     # [R, K, H, D]
            vs = v[b][it].double().numpy()
            s = np.einsum("rhd,rkhd->rhk", qs, ks) * scale     # [R, H, K]
            s = s - s.max(axis=2, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=2, keepdims=True)
            out[b, lo:lo + len(r)] = np.einsum("rhk,rkhd->rhd", p, vs)
    return out
