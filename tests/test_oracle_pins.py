"""Pins of the fp64 CPU oracle to facts other than itself (closed forms, invariants,
brute force, a library cross-check).  No GPU needed.

What is pinned and why (the pages print no worked attention example):
  * closed forms on hand-sized inputs (three keys with scores 0, 1, 2);
  * softmax rows sum to one and the output equals P @ V;
  * a single valid key returns its value row exactly;
  * equal scores return the mean of the valid value rows;
  * permuting keys together with values changes nothing;
  * keys under the mask (the zero-padded audio tail of "LTX-2: replicate audio
    stream across Ulysses ranks by default", Description) leave the result equal to
    the unpadded sequence, whatever the padded rows hold;
  * per-head-slice computation concatenated equals the full-head result (the
    head-split of v2a in the same Description);
  * attention over key ranges merged through their softmax statistics equals the full
    result ("feat(ltx2): tile-parallel video VAE and the two-stage pipeline", commit
    "Onboard Lightricks LTX-2.5");
  * scale -> 0 gives the mean of V; a dominant key gives its value row;
  * a pure-Python brute force and torch's fp64 softmax agree on non-square shapes.
"""
import math

import numpy as np
import pytest
import torch

from joint_audio_video_flash_b200 import synth


def bf(x):
    return torch.tensor(x, dtype=torch.float64).to(torch.bfloat16)


def f64(t):
    return t.to(torch.float64)


def textbook(q, k, v, scale, kv_valid=None):
    """torch fp64 softmax(scale q k^T) v per (b, h); a library cross-check only."""
    if kv_valid is not None:
        k, v = k[:, :kv_valid], v[:, :kv_valid]
    qd, kd, vd = f64(q), f64(k), f64(v)
    s = torch.einsum("bihd,bjhd->bhij", qd, kd) * scale
    p = torch.softmax(s, dim=-1)
    return torch.einsum("bhij,bjhd->bihd", p, vd).numpy()


def brute_force_row(q, k, v, scale, b, i, h, kv_valid):
    """Straight-line Python loops for one query row."""
    d = q.shape[3]
    s = []
    for j in range(kv_valid):
        acc = 0.0
        for x in range(d):
            acc += float(q[b, i, h, x]) * float(k[b, j, h, x])
        s.append(scale * acc)
    m = max(s)
    p = [math.exp(x - m) for x in s]
    l = sum(p)
    return [sum(p[j] * float(v[b, j, h, x]) for j in range(kv_valid)) / l for x in range(d)]


def test_closed_form_three_keys(oracle):
    # one batch, one head, d = 4; q = e0, k_j = j * e0 -> scores s_j = scale * j
    q = bf([[[[1.0, 0.0, 0.0, 0.0]]]])
    k = bf([[[[0.0, 0, 0, 0]], [[1.0, 0, 0, 0]], [[2.0, 0, 0, 0]]]])
    v = bf([[[[1.0, 2.0, -3.0, 0.5]], [[4.0, -1.0, 0.25, 8.0]], [[-2.0, 0.0, 6.0, -0.75]]]])
    for scale in (1.0, 0.5, 0.125):
        w = [math.exp(scale * j) for j in range(3)]
        z = sum(w)
        expect = [sum(w[j] * float(v[0, j, 0, x]) for j in range(3)) / z for x in range(4)]
        out, lse = oracle.attention(q, k, v, scale, return_lse=True)
        np.testing.assert_allclose(out[0, 0, 0], expect, rtol=1e-14, atol=1e-14)
        np.testing.assert_allclose(lse[0, 0, 0], math.log(z), rtol=1e-14)


def test_weights_sum_to_one_and_output_is_pv(oracle):
    q, k, v = synth.make_qkv(2, 5, 9, 3, 8, seed=11)
    for valid in (9, 4, 1):
        p = oracle.softmax_weights(q, k, 0.3, kv_valid_len=valid)
        np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
        assert np.all(p[..., valid:] == 0.0)
        assert np.all(p[..., :valid] > 0.0)
        out = oracle.attention(q, k, v, 0.3, kv_valid_len=valid)
        pv = np.einsum("bhij,bjhd->bihd", p, f64(v).numpy())
        np.testing.assert_allclose(out, pv, rtol=1e-12, atol=1e-13)


def test_single_key_returns_its_value(oracle):
    q, k, v = synth.make_qkv(2, 7, 16, 4, 64, seed=12)
    out = oracle.attention(q, k, v, 1 / 8, kv_valid_len=1)
    expect = f64(v[:, 0:1]).expand(-1, 7, -1, -1).numpy()
    assert np.array_equal(out, expect)


def test_equal_scores_return_mean(oracle):
    _, k, v = synth.make_qkv(2, 6, 10, 3, 16, seed=13)
    q = torch.zeros(2, 6, 3, 16, dtype=torch.bfloat16)
    for valid in (10, 7):
        out = oracle.attention(q, k, v, 0.25, kv_valid_len=valid)
        mean = f64(v[:, :valid]).mean(dim=1, keepdim=True).expand(-1, 6, -1, -1).numpy()
        np.testing.assert_allclose(out, mean, rtol=1e-13, atol=1e-14)
    # identical keys also give equal scores, whatever q is
    q2, _, _ = synth.make_qkv(2, 6, 10, 3, 16, seed=14)
    k_same = k[:, :1].expand(-1, 10, -1, -1).contiguous()
    out = oracle.attention(q2, k_same, v, 0.25)
    mean = f64(v).mean(dim=1, keepdim=True).expand(-1, 6, -1, -1).numpy()
    np.testing.assert_allclose(out, mean, rtol=1e-13, atol=1e-14)


def test_key_permutation_invariance(oracle):
    q, k, v = synth.make_qkv(2, 5, 33, 2, 64, seed=15)
    perm = torch.randperm(33, generator=torch.Generator().manual_seed(3))
    a = oracle.attention(q, k, v, 1 / 8)
    b = oracle.attention(q, k[:, perm].contiguous(), v[:, perm].contiguous(), 1 / 8)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-15)
    assert not np.allclose(a, oracle.attention(q, k[:, perm].contiguous(), v, 1 / 8))


def test_padded_keys_under_mask_change_nothing(oracle):
    # audio: 126 valid tokens zero-padded to 128, and the same with garbage in the pad
    q, k, v = synth.make_qkv(2, 128, 128, 4, 64, seed=16, q_valid=126, kv_valid=126)
    ref = oracle.attention(q, k[:, :126].contiguous(), v[:, :126].contiguous(), 1 / 8)
    masked = oracle.attention(q, k, v, 1 / 8, kv_valid_len=126)
    assert np.array_equal(ref, masked)
    g = torch.Generator().manual_seed(5)
    k2, v2 = k.clone(), v.clone()
    k2[:, 126:] = (torch.randn(2, 2, 4, 64, generator=g) * 1000).to(torch.bfloat16)
    v2[:, 126:] = (torch.randn(2, 2, 4, 64, generator=g) * 1e30).to(torch.bfloat16)
    assert np.array_equal(ref, oracle.attention(q, k2, v2, 1 / 8, kv_valid_len=126))
    # without the mask the padded keys do matter
    assert not np.allclose(ref, oracle.attention(q, k2, v2, 1 / 8, kv_valid_len=128))


def test_head_slice_concatenation_equals_full(oracle):
    q, k, v = synth.make_qkv(2, 9, 40, 6, 64, seed=17)
    full = oracle.attention(q, k, v, 1 / 8)
    lo = oracle.attention(q[:, :, :3].contiguous(), k[:, :, :3].contiguous(),
                          v[:, :, :3].contiguous(), 1 / 8)
    hi = oracle.attention(q[:, :, 3:].contiguous(), k[:, :, 3:].contiguous(),
                          v[:, :, 3:].contiguous(), 1 / 8)
    assert np.array_equal(full, np.concatenate([lo, hi], axis=2))
    # heads are not interchangeable: swapping the halves breaks equality
    assert not np.allclose(full, np.concatenate([hi, lo], axis=2))


@pytest.mark.parametrize("cuts", [(0, 20, 40), (0, 1, 39, 40), (0, 7, 13, 29, 40)])
def test_split_key_merge_equals_full(oracle, cuts):
    q, k, v = synth.make_qkv(2, 9, 40, 3, 32, seed=18)
    full, lse = oracle.attention(q, k, v, 0.2, return_lse=True)
    parts = [oracle.attention_part(q, k, v, 0.2, a, b) for a, b in zip(cuts[:-1], cuts[1:])]
    d = full.shape[-1]
    o = np.stack([p[0].reshape(-1, d) for p in parts])
    m = np.stack([p[1].reshape(-1) for p in parts])
    l = np.stack([p[2].reshape(-1) for p in parts])
    merged, mlse = oracle.merge_partials(o, m, l, return_lse=True)
    np.testing.assert_allclose(merged, full.reshape(-1, d), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(mlse, lse.reshape(-1), rtol=1e-13, atol=1e-13)
    # a plain average of the parts is not the merge
    assert not np.allclose(o.mean(0), full.reshape(-1, d), atol=1e-6)


def test_part_statistics_closed_form(oracle):
    q, k, v = synth.make_qkv(1, 3, 12, 2, 16, seed=19)
    o, m, l = oracle.attention_part(q, k, v, 0.5, 4, 10)
    s = torch.einsum("bihd,bjhd->bihj", f64(q), f64(k[:, 4:10])).numpy() * 0.5
    np.testing.assert_allclose(m, s.max(-1), rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(l, np.exp(s - s.max(-1, keepdims=True)).sum(-1), rtol=1e-13)


def test_scale_limits(oracle):
    q, k, v = synth.make_qkv(1, 4, 20, 2, 64, seed=20)
    tiny = oracle.attention(q, k, v, 1e-30)
    mean = f64(v).mean(dim=1, keepdim=True).expand(-1, 4, -1, -1).numpy()
    np.testing.assert_allclose(tiny, mean, rtol=1e-12, atol=1e-14)
    # one key aligned with q and a large scale: the output is that key's value row
    k2 = k.clone()
    k2[:, 13] = q[:, 0] * 4
    q2 = q[:, :1].contiguous()
    out = oracle.attention(q2, k2, v, 50.0)
    np.testing.assert_allclose(out[0, 0], f64(v[0, 13]).numpy(), rtol=0, atol=1e-12)
    assert np.all(np.isfinite(out))


def test_textbook_and_brute_force_on_non_square_shapes(oracle):
    q, k, v = synth.make_qkv(2, 5, 7, 3, 4, seed=21)
    for valid in (7, 5):
        out = oracle.attention(q, k, v, 0.7, kv_valid_len=valid)
        np.testing.assert_allclose(out, textbook(q, k, v, 0.7, valid), rtol=1e-12, atol=1e-14)
        for b in range(2):
            for i in range(5):
                for h in range(3):
                    np.testing.assert_allclose(
                        out[b, i, h], brute_force_row(q, k, v, 0.7, b, i, h, valid),
                        rtol=1e-12, atol=1e-14)


def test_tiny_workload_against_textbook_and_brute_force(oracle):
    from joint_audio_video_flash_b200 import workloads
    _, calls = workloads.configs()["tiny"]
    for c in calls:
        q, k, v = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed)
        out = oracle.attention(q, k, v, c.scale, kv_valid_len=c.kv_valid_len)
        np.testing.assert_allclose(out, textbook(q, k, v, c.scale, c.kv_valid_len),
                                   rtol=1e-11, atol=1e-13)
        for (b, i, h) in [(0, 0, 0), (0, c.q_len - 1, c.heads - 1)]:
            np.testing.assert_allclose(out[b, i, h],
                                       brute_force_row(q, k, v, c.scale, b, i, h, c.kv_valid_len),
                                       rtol=1e-11, atol=1e-13)


def test_row_sampling_matches_full(oracle):
    q, k, v = synth.make_qkv(2, 11, 30, 3, 32, seed=22)
    full, lse = oracle.attention(q, k, v, 0.3, kv_valid_len=25, return_lse=True)
    rows = synth.sample_rows(2, 11, 3, per_head=4, seed=1, full_heads=((1, 2),))
    part, plse = oracle.attention(q, k, v, 0.3, kv_valid_len=25, rows=rows.numpy(),
                                  return_lse=True)
    assert np.array_equal(part, full.reshape(-1, 32)[rows.numpy()])
    assert np.array_equal(plse, lse.reshape(-1)[rows.numpy()])


def test_large_scores_do_not_overflow(oracle):
    # scores of order 1e4 would overflow exp() without the max subtraction
    q = bf([[[[100.0, 0, 0, 0]]]])
    k = bf([[[[100.0, 0, 0, 0]], [[99.0, 0, 0, 0]], [[-50.0, 0, 0, 0]]]])
    v = bf([[[[1.0, 0, 0, 0]], [[0.0, 1.0, 0, 0]], [[0.0, 0, 1.0, 0]]]])
    out = oracle.attention(q, k, v, 1.0)
    np.testing.assert_allclose(out[0, 0, 0], [1.0, math.exp(-100.0), 0.0, 0.0], rtol=1e-12,
                               atol=1e-300)
    out = oracle.attention(q, k, v, 0.01)  # scores 100, 99, -50: weights 1, e^-1, ~0
    z = 1 + math.exp(-1) + math.exp(-150)
    np.testing.assert_allclose(out[0, 0, 0], [1 / z, math.exp(-1) / z, math.exp(-150) / z, 0.0],
                               rtol=1e-13)


def test_rejects_bad_arguments(oracle):
    q, k, v = synth.make_qkv(1, 3, 4, 1, 8, seed=23)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, 1.0, kv_valid_len=0)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, 1.0, kv_valid_len=5)
    with pytest.raises(ValueError):
        oracle.attention(q, k, v, 1.0, rows=np.array([12]))
