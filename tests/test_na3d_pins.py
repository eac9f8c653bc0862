"""Pins of the 3-D neighbourhood-attention oracle against things other than itself (CPU).

- a window as large as the grid is full softmax attention (torch's fp64 SDPA);
- a 1 x 1 x 1 window returns each token's own value row;
- on small grids, the neighbourhood built by sliding a centred box inward step by step
  (a different procedure from the oracle's clamp) fed as a boolean mask to torch's fp64
  SDPA gives the oracle's result, on non-cubic grids and windows (axes not swapped);
- every neighbourhood has exactly kT*kY*kX distinct in-grid members including the query,
  and is the centred box away from the borders;
- moving the content one step along an axis moves the interior outputs with it.
"""
import itertools

import numpy as np
import pytest
import torch

from joint_audio_video_flash_b200 import synth
from oracle import na3d as na


def _sdpa(q, k, v, scale, mask=None):
    # torch fp64 reference: [B, N, H, D] -> [B, N, H, D]
    qt, kt, vt = (t.double().permute(0, 2, 1, 3) for t in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def _slide_in(i, k, n):
    # centred window, then moved one step at a time until it lies inside [0, n)
    s = i - k // 2
    while s < 0:
        s += 1
    while s + k > n:
        s -= 1
    return s


def _mask_by_sliding(grid, kernel):
    t_n, y_n, x_n = grid
    n = t_n * y_n * x_n
    m = torch.zeros(n, n, dtype=torch.bool)
    for t, y, x in itertools.product(range(t_n), range(y_n), range(x_n)):
        st = _slide_in(t, kernel[0], t_n)
        sy = _slide_in(y, kernel[1], y_n)
        sx = _slide_in(x, kernel[2], x_n)
        qi = (t * y_n + y) * x_n + x
        for a, b, c in itertools.product(range(kernel[0]), range(kernel[1]), range(kernel[2])):
            m[qi, ((st + a) * y_n + sy + b) * x_n + sx + c] = True
    return m


def test_window_as_large_as_grid_is_full_attention():
    grid = (3, 5, 7)
    q, k, v = synth.make_qkv(2, 105, 105, 3, 16, seed=40)
    got = na.na3d(q, k, v, grid, grid, 0.3)
    np.testing.assert_allclose(got, _sdpa(q, k, v, 0.3), rtol=0, atol=1e-12)


def test_unit_window_returns_own_value():
    grid = (2, 3, 4)
    q, k, v = synth.make_qkv(1, 24, 24, 2, 8, seed=41)
    got = na.na3d(q, k, v, grid, (1, 1, 1), 1.0)
    np.testing.assert_array_equal(got, v.double().numpy())


@pytest.mark.parametrize("grid,kernel", [((3, 4, 5), (1, 3, 5)), ((4, 6, 5), (3, 3, 1)),
                                         ((5, 3, 6), (3, 1, 5)), ((1, 1, 17), (1, 1, 5))])
def test_matches_sliding_box_mask(grid, kernel):
    n = grid[0] * grid[1] * grid[2]
    q, k, v = synth.make_qkv(2, n, n, 2, 8, seed=42 + n)
    got = na.na3d(q, k, v, grid, kernel, 0.25)
    want = _sdpa(q, k, v, 0.25, _mask_by_sliding(grid, kernel))
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_neighbourhood_properties():
    grid, kernel = (5, 7, 9), (3, 5, 7)
    n = grid[0] * grid[1] * grid[2]
    idx = na.neighbours(np.arange(n), grid, kernel)
    vol = kernel[0] * kernel[1] * kernel[2]
    for i in range(n):
        nb = idx[i]
        assert len(set(nb.tolist())) == vol and i in nb
        assert nb.min() >= 0 and nb.max() < n
    # away from the borders the box is centred: |delta| <= (k - 1) / 2 on every axis
    t, y, x = 2, 3, 4
    i = (t * grid[1] + y) * grid[2] + x
    want = {((t + a) * grid[1] + y + b) * grid[2] + x + c
            for a in range(-1, 2) for b in range(-2, 3) for c in range(-3, 4)}
    assert set(idx[i].tolist()) == want


def test_shift_moves_interior_outputs():
    grid, kernel = (3, 6, 12), (3, 3, 3)
    n = grid[0] * grid[1] * grid[2]
    q, k, v = synth.make_qkv(1, n, n, 1, 8, seed=43)
    shape = (1, *grid, 1, 8)

    def shifted(t):
        return torch.roll(t.reshape(shape), 1, dims=3).reshape(1, n, 1, 8)

    a = na.na3d(q, k, v, grid, kernel, 0.5).reshape(shape)
    b = na.na3d(shifted(q), shifted(k), shifted(v), grid, kernel, 0.5).reshape(shape)
    # x = 2 .. 9: the windows of x and x + 1 are interior for the unrolled content
    np.testing.assert_allclose(b[:, :, 1:5, 3:10], a[:, :, 1:5, 2:9], rtol=0, atol=1e-12)
    assert not np.allclose(b[:, :, 1:5, 3:10], a[:, :, 1:5, 3:10])


def test_rejects_even_or_oversized_windows():
    for kernel in [(2, 1, 1), (1, 1, 9)]:
        with pytest.raises(ValueError):
            na.check_shape((4, 4, 8), kernel)
