"""QK-norm + rotary prologue kernel vs its fp64 oracle, through the C ABI (needs a B200).

Same bar as the attention parity tests, per tensor: max-abs error <= 2e-2 and relative
L2 error <= 5e-3 on the bf16 output.
"""
import numpy as np
import pytest
import torch

from joint_audio_video_flash_b200 import build, ltxattn, synth
from oracle import qk_prologue as qp

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    ltxattn.load()


def _check(got, ref, what):
    g = got.cpu().to(torch.float64).numpy()
    assert np.all(np.isfinite(g))
    diff = g - ref
    max_abs = float(np.abs(diff).max())
    rel = float(np.linalg.norm(diff) / np.linalg.norm(ref))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"


SHAPES = [
    # batch, seq_len, heads, head_dim
    (1, 1, 4, 128),       # inner 512
    (2, 37, 16, 64),      # inner 1024, ragged length
    (3, 129, 32, 64),     # audio stream heads, inner 2048
    (2, 300, 32, 128),    # video stream heads, inner 4096
    (1, 50, 64, 64),      # inner 4096 with 64-channel heads
    (2, 21, 64, 128),     # inner 8192: one row per CTA
    (1, 9, 4, 256),       # inner 1024 with 256-channel heads
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "b{}l{}h{}d{}".format(*s))
def test_matches_oracle(shape):
    b, l, h, d = shape
    q, k, wq, wk, cos, sin = synth.make_qk_prologue_inputs(b, l, h, d, seed=b * 1000 + l + h)
    dev = [t.cuda() for t in (q, k, wq, wk, cos, sin)]
    qo, ko = ltxattn.qk_norm_rope(*dev, eps=1e-6)
    torch.cuda.synchronize()
    _check(qo, qp.rms_norm_rope(q, wq, cos, sin, 1e-6), f"q {shape}")
    _check(ko, qp.rms_norm_rope(k, wk, cos, sin, 1e-6), f"k {shape}")


def test_in_place_equals_out_of_place():
    q, k, wq, wk, cos, sin = synth.make_qk_prologue_inputs(2, 64, 32, 128, seed=7)
    dev = [t.cuda() for t in (q, k, wq, wk, cos, sin)]
    qo, ko = ltxattn.qk_norm_rope(*dev)
    qi, ki = dev[0].clone(), dev[1].clone()
    ltxattn.qk_norm_rope(qi, ki, *dev[2:], q_out=qi, k_out=ki)
    torch.cuda.synchronize()
    assert torch.equal(qi, qo) and torch.equal(ki, ko)


def test_video_size_sampled_tokens():
    # the bench's size: B2 x 15360 tokens x 32 heads x 128; tokens compared in full on a sample
    b, l, h, d = 2, 15360, 32, 128
    q, k, wq, wk, cos, sin = synth.make_qk_prologue_inputs(b, l, h, d, seed=11)
    dev = [t.cuda() for t in (q, k, wq, wk, cos, sin)]
    qo, ko = ltxattn.qk_norm_rope(*dev)
    torch.cuda.synchronize()
    g = torch.Generator().manual_seed(3)
    toks = torch.randint(0, l, (64,), generator=g).tolist() + [0, l - 1]
    for bi in range(b):
        sel = (slice(bi, bi + 1), toks)
        _check(qo[bi:bi + 1, toks], qp.rms_norm_rope(q[sel], wq, cos[toks], sin[toks], 1e-6),
               f"q b{bi}")
        _check(ko[bi:bi + 1, toks], qp.rms_norm_rope(k[sel], wk, cos[toks], sin[toks], 1e-6),
               f"k b{bi}")


def test_host_checks():
    q = torch.zeros(1, 4, 3, 64, dtype=torch.bfloat16, device="cuda")  # inner 192: unsupported
    w = torch.ones(192, dtype=torch.bfloat16, device="cuda")
    c = torch.ones(4, 32, device="cuda")
    with pytest.raises(ltxattn.LtxAttnError) as e:
        ltxattn.qk_norm_rope(q, q.clone(), w, w, c, c)
    assert e.value.status == ltxattn.ERR_UNSUPPORTED
    q = torch.zeros(1, 4, 8, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(512, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ltxattn.LtxAttnError) as e:
        ltxattn.qk_norm_rope(q, q, w, w, c, c, q_out=q, k_out=q)  # k_out overlaps q
    assert e.value.status == ltxattn.ERR_INVALID_ARG
