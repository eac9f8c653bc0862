"""The allocation-free entry point (ltxattn_forward_split_noalloc).

Callers that cannot let a library allocate device memory (a plugin host that owns
all of it, a serving loop with a fixed memory plan, a hard quota) use this call;
key-split partials live in the library's built-in scratch array and a single key
part writes the output directly.  Its output must match the fp64 oracle and the
ordinary entry point on the same inputs, on two calls in a row (the second call
reuses the scratch the first one left behind).  This file is collected last on
purpose and also runs on its own in a fresh process.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from joint_audio_video_flash_b200 import build, ltxattn, synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    ltxattn.load()
    ltxattn.create()  # for the ordinary entry point used as the second comparison
    yield


def close(a, b):
    a64 = a.double().cpu().numpy().reshape(b.shape)
    b64 = b.double().cpu().numpy() if isinstance(b, torch.Tensor) else b
    assert np.all(np.isfinite(a64))
    diff = a64 - b64
    max_abs = float(np.abs(diff).max())
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(b64), 1e-30))
    assert max_abs <= MAX_ABS and rel <= REL_L2, (max_abs, rel)


def run_noalloc(q, k, v, valid, splits):
    out = torch.full_like(q, float("nan"))
    st = ltxattn.forward_split_noalloc(q, k, v, out, kv_valid_len=valid, num_splits=splits)
    assert st == ltxattn.OK, ltxattn.status_string(st)
    ltxattn.check()  # synchronises; reports a kernel wait that ran out in this call
    return out


@pytest.mark.parametrize("shape,splits", [
    ((2, 4, 64, 126, 2048, 2000), 4),     # v2a-like, ragged last key tile
    ((2, 32, 64, 128, 15360, 15360), 0),  # v2a at the 768x1280x121 block size, planned split
    ((1, 3, 128, 200, 1000, 900), 3),
    ((1, 16, 128, 256, 16384, 16384), 0),  # planned 9 parts, capped at the 7 that fit
    ((2, 32, 128, 256, 15360, 15360), 0),  # planned 2 parts; one fits: the direct kernel
    ((2, 8, 64, 2000, 128, 126), 0),       # a2v-like: one part, persistent short-key kernel
])
def test_noalloc_matches_oracle_and_forward_on_two_calls(oracle, shape, splits):
    b, h, d, lq, lkv, valid = shape
    for call, seed in enumerate((21, 22)):  # two calls in a row, different inputs
        qh, kh, vh = synth.make_qkv(b, lq, lkv, h, d, seed=seed + lq, kv_valid=valid)
        q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
        out = run_noalloc(q, k, v, valid, splits)
        want = ltxattn.forward(q, k, v, kv_valid_len=valid, num_splits=splits)
        torch.cuda.synchronize()
        close(out, want)
        # the oracle on every row of small cases, on sampled rows of the large ones
        rows = None
        if b * lq * h * lkv > 5e7:
            rows = synth.sample_rows(b, lq, h, 16, seed=seed, full_heads=((b - 1, h - 1),)).numpy()
        ref = oracle.attention(qh, kh, vh, d ** -0.5, kv_valid_len=valid, rows=rows)
        got = out.cpu().reshape(-1, d)[torch.as_tensor(rows)] if rows is not None else out.cpu()
        close(got, ref)


def test_noalloc_rejects_partials_beyond_the_scratch():
    # 8 parts x 4 x 64 heads x 2 query tiles x 129 floats = 8.7e7 bytes > 16 MiB
    g = torch.Generator().manual_seed(3)
    q = torch.randn(4, 256, 64, 128, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(4, 2048, 64, 128, generator=g).to(torch.bfloat16).cuda()
    out = torch.full_like(q, float("nan"))
    before = out.view(torch.int16).clone()
    st = ltxattn.forward_split_noalloc(q, k, k, out, num_splits=8)
    assert st == ltxattn.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), before)  # nothing was enqueued


def test_noalloc_rejects_tensors_the_c_abi_cannot_check():
    q = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    with pytest.raises(TypeError):
        ltxattn.forward_split_noalloc(q.float(), q, q, out)
    with pytest.raises(ValueError):
        ltxattn.forward_split_noalloc(q, q[:, :, :1], q[:, :, :1], out)  # fewer key heads
    with pytest.raises(ValueError):
        ltxattn.forward_split_noalloc(q, q, q, out.transpose(1, 2))  # not contiguous


_FRESH = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
from joint_audio_video_flash_b200 import ltxattn, synth
from oracle import oracle
torch.cuda.set_device(0)
q, k, v = synth.make_qkv(2, 126, 3000, 4, 64, seed=5, kv_valid=2990)
out = torch.full_like(q.cuda(), float("nan"))
for _ in range(2):
    st = ltxattn.forward_split_noalloc(q.cuda(), k.cuda(), v.cuda(), out, kv_valid_len=2990)
    assert st == ltxattn.OK, st
    ltxattn.check()  # no ltxattn_create in this process: reads the call's own status word
ref = oracle.attention(q, k, v, 0.125, kv_valid_len=2990)
got = out.cpu().double().numpy()
err = abs(got - ref).max()
rel = ((got - ref) ** 2).sum() ** 0.5 / (ref ** 2).sum() ** 0.5
assert err <= 2e-2 and rel <= 5e-3, (err, rel)
print("fresh-process ok", err, rel)
"""


def test_noalloc_in_a_process_that_never_creates_a_context():
    r = subprocess.run([sys.executable, "-c", _FRESH, ROOT], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "fresh-process ok" in r.stdout
