"""The allocation-free key-split entry point (ltxattn_forward_split_noalloc).

Callers that cannot let a library allocate device memory (a plugin host that owns
all of it, a serving loop with a fixed memory plan, a hard quota) use this call;
its partials live in the library's built-in scratch array.  Its output must match
the ordinary entry point's on the same inputs, on two calls in a row (the second
call reuses the scratch the first one left behind).  This file is collected last
on purpose and also runs on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from joint_audio_video_flash_b200 import build, ltxattn, synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    ltxattn.load()
    ltxattn.create()  # for the ordinary entry point used as the comparison
    yield


def close(a, b):
    a64, b64 = a.double().cpu().numpy(), b.double().cpu().numpy()
    assert np.all(np.isfinite(a64))
    diff = a64 - b64
    max_abs = float(np.abs(diff).max())
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(b64), 1e-30))
    assert max_abs <= MAX_ABS and rel <= REL_L2, (max_abs, rel)


@pytest.mark.parametrize("shape,splits", [
    ((2, 4, 64, 126, 2048, 2000), 4),     # v2a-like, ragged last key tile
    ((2, 32, 64, 128, 15360, 15360), 0),  # v2a at the 768x1280x121 block size, planned split
    ((1, 3, 128, 200, 1000, 900), 3),
])
def test_noalloc_matches_forward_on_two_calls(shape, splits):
    b, h, d, lq, lkv, valid = shape
    for call, seed in enumerate((21, 22)):  # two calls in a row, different inputs
        q, k, v = [t.cuda() for t in synth.make_qkv(b, lq, lkv, h, d, seed=seed + lq)]
        want = ltxattn.forward(q, k, v, kv_valid_len=valid, num_splits=splits)
        out = torch.full_like(q, float("nan"))
        st = ltxattn.forward_split_noalloc(q, k, v, out, kv_valid_len=valid, num_splits=splits)
        assert st == ltxattn.OK, ltxattn.status_string(st)
        torch.cuda.synchronize()
        close(out, want)


def test_noalloc_rejects_partials_beyond_the_scratch():
    # 8 parts x 4 x 64 heads x 2 query tiles x 129 floats = 8.7e7 bytes > 16 MiB
    q = torch.zeros(4, 256, 64, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(4, 2048, 64, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q)
    st = ltxattn.forward_split_noalloc(q, k, k, out, num_splits=8)
    assert st == ltxattn.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0  # nothing was enqueued
