"""Pins of the QK-norm + rotary prologue oracle against what its definition fixes (CPU).

Each pin fails for a plausible mistake: a norm over the wrong axis or without the mean,
a missing weight, a rotation with a wrong sign or on the wrong pairs, or tables applied
at the wrong position.
"""
import math

import numpy as np
import torch

from joint_audio_video_flash_b200 import synth
from oracle import qk_prologue as qp


def _identity_tables(length, half):
    return torch.ones(length, half), torch.zeros(length, half)


def test_hand_case():
    # one token, one head of 4 channels: mean square 7.5; pair 0 turned by 90 degrees,
    # pair 1 not turned
    x = torch.tensor([1.0, 2.0, 3.0, 4.0]).view(1, 1, 1, 4).to(torch.bfloat16)
    w = torch.ones(4).to(torch.bfloat16)
    cos, sin = torch.tensor([[0.0, 1.0]]), torch.tensor([[1.0, 0.0]])
    got = qp.rms_norm_rope(x, w, cos, sin, 0.0).ravel()
    np.testing.assert_allclose(got, np.array([-2.0, 1.0, 3.0, 4.0]) / math.sqrt(7.5), rtol=1e-15)


def test_unit_weights_and_no_rotation_give_unit_rms_per_token():
    q, _, _, _, _, _ = synth.make_qk_prologue_inputs(2, 5, 3, 8, seed=1)
    w = torch.ones(3 * 8).to(torch.bfloat16)
    c, s = _identity_tables(5, 4)
    eps = 1e-6
    y = qp.rms_norm_rope(q, w, c, s, eps)
    ms_in = (q.double() ** 2).reshape(2, 5, -1).mean(dim=2).numpy()
    ms_out = (y ** 2).reshape(2, 5, -1).mean(axis=2)
    np.testing.assert_allclose(ms_out, ms_in / (ms_in + eps), rtol=1e-12)
    # the norm is per token over all heads: one head alone is not unit
    assert not np.allclose((y[:, :, 0] ** 2).mean(axis=2), 1.0, rtol=1e-3)


def test_weight_scales_channels_before_rotation():
    q, _, w, _, _, _ = synth.make_qk_prologue_inputs(1, 3, 2, 8, seed=2)
    c, s = _identity_tables(3, 4)
    ones = torch.ones_like(w)
    a = qp.rms_norm_rope(q, w, c, s, 1e-6)
    b = qp.rms_norm_rope(q, ones, c, s, 1e-6) * w.double().numpy().reshape(1, 1, 2, 8)
    np.testing.assert_allclose(a, b, rtol=1e-13)


def test_rotation_preserves_pair_norms_and_angle():
    q, _, w, _, cos, sin = synth.make_qk_prologue_inputs(2, 7, 2, 16, seed=3)
    c0, s0 = _identity_tables(7, 8)
    y = qp.rms_norm_rope(q, w, c0, s0, 1e-6)
    z = qp.rms_norm_rope(q, w, cos, sin, 1e-6)
    # (a c - b s)^2 + (a s + b c)^2 = (a^2 + b^2)(c^2 + s^2); the fp32 tables make
    # c^2 + s^2 differ from 1 by ~1e-7, so the factor is kept
    cs2 = (cos.double() ** 2 + sin.double() ** 2).numpy()[None, :, None, :]
    np.testing.assert_allclose(z[..., 0::2] ** 2 + z[..., 1::2] ** 2,
                               (y[..., 0::2] ** 2 + y[..., 1::2] ** 2) * cs2, rtol=1e-12,
                               atol=1e-15)
    # each pair turns counter-clockwise by its table angle
    ang = np.arctan2(z[..., 1::2], z[..., 0::2]) - np.arctan2(y[..., 1::2], y[..., 0::2])
    want = np.arctan2(sin.double().numpy(), cos.double().numpy())[None, :, None, :]
    np.testing.assert_allclose(np.angle(np.exp(1j * (ang - want))), 0.0, atol=1e-9)


def test_relative_position_property():
    # with angles p * w_i, <R_m a, R_n b> = <a, R_(n-m) b>: scores depend only on n - m
    length, heads, d = 9, 2, 8
    q, k, wq, wk, cos, sin = synth.make_qk_prologue_inputs(1, length, heads, d, seed=4)
    c0, s0 = _identity_tables(length, d // 2)
    qr = qp.rms_norm_rope(q, wq, cos, sin, 1e-6)[0]
    kr = qp.rms_norm_rope(k, wk, cos, sin, 1e-6)[0]
    qn = qp.rms_norm_rope(q, wq, c0, s0, 1e-6)[0]
    kn = qp.rms_norm_rope(k, wk, c0, s0, 1e-6)[0]
    inv_freq = 10000.0 ** (-np.arange(d // 2) * 2.0 / d)
    for m in range(length):
        for n in range(length):
            t = (n - m) * inv_freq
            a, b = kn[n][..., 0::2], kn[n][..., 1::2]
            rot = np.empty_like(kn[n])
            rot[..., 0::2] = a * np.cos(t) - b * np.sin(t)
            rot[..., 1::2] = a * np.sin(t) + b * np.cos(t)
            np.testing.assert_allclose(np.sum(qr[m] * kr[n], axis=-1),
                                       np.sum(qn[m] * rot, axis=-1), rtol=2e-6, atol=2e-7)


def test_scale_invariance():
    q, _, w, _, cos, sin = synth.make_qk_prologue_inputs(1, 4, 2, 8, seed=5)
    a = qp.rms_norm_rope(q, w, cos, sin, 0.0)
    b = qp.rms_norm_rope((q.float() * 4.0).to(torch.bfloat16), w, cos, sin, 0.0)  # exact
    np.testing.assert_allclose(a, b, rtol=1e-14)
