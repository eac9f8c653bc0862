"""3-D neighbourhood attention kernel vs its fp64 oracle, through the C ABI (needs a B200).

Same bar as the attention parity tests: max-abs error <= 2e-2 and relative L2 error
<= 5e-3 on the bf16 output.  The grids are chosen so that the host picks each of the
seven (query brick, key tile) shape pairs (bricks 2x8x8, 1x8x16, 4x4x8; key tiles of the
brick's own shape, 4x2x16, 1x16x8 or the 112-key 4x2x14), with ragged bricks on every axis,
one and two heads, batch 1 and 2, head_dim 64 and 128.
"""
import numpy as np
import pytest
import torch

from joint_audio_video_flash_b200 import build, ltxattn, synth
from oracle import na3d as na

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    ltxattn.create()


def _check(got, ref, what):
    g = got.cpu().to(torch.float64).numpy()
    assert np.all(np.isfinite(g)), what
    diff = g - ref
    max_abs = float(np.abs(diff).max())
    rel = float(np.linalg.norm(diff) / np.linalg.norm(ref))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"


CASES = [
    # batch, grid (T, Y, X), heads, head_dim, window   query brick (key tile) the host picks
    (1, (2, 8, 8), 1, 64, (1, 3, 3)),      # 2x8x8, a single brick
    (2, (3, 10, 13), 2, 64, (3, 5, 7)),    # 4x4x8, ragged on every axis
    (1, (5, 12, 20), 2, 128, (3, 7, 7)),   # 2x8x8 bricks over 4x2x14 key tiles (112 keys)
    (2, (1, 24, 40), 2, 64, (1, 7, 9)),    # 1x8x16 (1x16x8 key tiles), a 2-D grid
    (1, (16, 8, 8), 1, 128, (7, 3, 3)),    # 2x8x8, long time axis
    (1, (12, 6, 9), 2, 64, (5, 3, 5)),     # 2x8x8, bricks wider than the grid
    (2, (1, 8, 8), 2, 128, (1, 3, 3)),     # 2x8x8 on a one-frame grid: half of each brick is past it
    (1, (1, 5, 6), 1, 64, (1, 3, 5)),      # a grid smaller than one brick on every axis
    (2, (3, 10, 13), 2, 128, (3, 5, 7)),   # 4x4x8 at head_dim 128, batch 2
    (1, (9, 4, 5), 3, 128, (5, 3, 3)),     # 4x4x8, three heads, long time axis
    (1, (2, 3, 40), 2, 64, (1, 3, 9)),     # 2x8x8, long thin grid
    (1, (8, 12, 16), 2, 128, (3, 3, 9)),   # 2x8x8 bricks over 4x2x14 key tiles
    (1, (6, 12, 16), 2, 64, (3, 5, 5)),    # 2x8x8 / 4x2x14 at head_dim 64
    (1, (6, 12, 32), 2, 64, (3, 5, 9)),    # 2x8x8 / 4x2x16 (x boxes of 16)
    (2, (6, 13, 30), 2, 128, (3, 7, 7)),   # 2x8x8 / 4x2x14, ragged, batch 2
    (1, (5, 11, 29), 2, 64, (3, 5, 7)),    # 2x8x8 / 4x2x14 at head_dim 64, ragged
    (2, (3, 9, 17), 2, 64, (3, 3, 9)),     # 4x4x8 bricks over 4x2x16 key tiles, ragged
    (1, (4, 14, 22), 1, 128, (3, 7, 7)),   # 4x4x8 / 4x2x16 at head_dim 128
]


def _name(c):
    b, g, h, d, w = c
    return f"b{b}g{g[0]}x{g[1]}x{g[2]}h{h}d{d}w{w[0]}x{w[1]}x{w[2]}"


@pytest.mark.parametrize("case", CASES, ids=_name)
def test_matches_oracle(case):
    b, grid, h, d, win = case
    n = grid[0] * grid[1] * grid[2]
    q, k, v = synth.make_qkv(b, n, n, h, d, seed=300 + n + h)
    out = ltxattn.na3d_forward(*(t.cuda() for t in (q, k, v)), grid, win)
    ltxattn.check()
    _check(out, na.na3d(q, k, v, grid, win, d ** -0.5), _name(case))


def test_window_as_large_as_grid_is_full_attention():
    # 1x8x16 bricks; every query sees every key: the dense attention kernel's result
    grid, d = (3, 9, 11), 128
    n = grid[0] * grid[1] * grid[2]
    q, k, v = (t.cuda() for t in synth.make_qkv(1, n, n, 2, d, seed=310))
    out = ltxattn.na3d_forward(q, k, v, grid, grid)
    dense = ltxattn.forward(q, k, v)
    ltxattn.check()
    ref = na.na3d(q.cpu(), k.cpu(), v.cpu(), grid, grid, d ** -0.5)
    _check(out, ref, "full window")
    _check(dense, ref, "dense kernel, same inputs")


def test_unit_window_returns_values_exactly():
    grid = (2, 3, 4)
    q, k, v = (t.cuda() for t in synth.make_qkv(2, 24, 24, 3, 64, seed=311))
    out = ltxattn.na3d_forward(q, k, v, grid, (1, 1, 1))
    ltxattn.check()
    assert torch.equal(out, v)


def test_deterministic():
    grid, win = (5, 12, 20), (3, 7, 7)
    n = grid[0] * grid[1] * grid[2]
    q, k, v = (t.cuda() for t in synth.make_qkv(2, n, n, 2, 128, seed=312))
    a = ltxattn.na3d_forward(q, k, v, grid, win)
    b = ltxattn.na3d_forward(q, k, v, grid, win)
    ltxattn.check()
    assert torch.equal(a, b)


@pytest.mark.parametrize("win", [(3, 7, 7), (5, 9, 9)], ids=["w3x7x7", "w5x9x9"])
def test_decoder_grid_sampled_rows(win):
    # the bench grid, 16 x 34 x 60 tokens (2x8x8 bricks over 4x2x14 key tiles for 3x7x7, 4x4x8
    # bricks over 4x2x16 for 5x9x9),
    # 32 heads x 128; every head of a seeded sample of tokens, including the grid's corners
    grid, h, d = (16, 34, 60), 32, 128
    n = grid[0] * grid[1] * grid[2]
    q, k, v = synth.make_qkv(1, n, n, h, d, seed=313)
    out = ltxattn.na3d_forward(*(t.cuda() for t in (q, k, v)), grid, win)
    ltxattn.check()
    g = torch.Generator().manual_seed(5)
    rows = sorted(set(torch.randint(0, n, (96,), generator=g).tolist()) | {0, 59, n - 60, n - 1})
    ref = na.na3d(q, k, v, grid, win, d ** -0.5, rows=np.array(rows))
    _check(out[:, rows], ref, f"decoder grid {win}")


def test_host_checks():
    q = torch.zeros(1, 48, 1, 64, dtype=torch.bfloat16, device="cuda")
    for grid, win, status in [((2, 4, 6), (2, 1, 1), ltxattn.ERR_INVALID_ARG),   # even window
                              ((2, 4, 6), (1, 5, 1), ltxattn.ERR_INVALID_ARG)]:  # window > axis
        with pytest.raises(ltxattn.LtxAttnError) as e:
            ltxattn.na3d_forward(q, q, q, grid, win)
        assert e.value.status == status
    q96 = torch.zeros(1, 48, 1, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ltxattn.LtxAttnError) as e:
        ltxattn.na3d_forward(q96, q96, q96, (2, 4, 6), (1, 1, 1))
    assert e.value.status == ltxattn.ERR_UNSUPPORTED
    with pytest.raises(ltxattn.LtxAttnError) as e:
        ltxattn.na3d_forward(q, q, q, (2, 4, 6), (1, 1, 1), out=q)  # out overlaps q
    assert e.value.status == ltxattn.ERR_INVALID_ARG
