"""ltxattn_forward_plan (host only, no GPU): which attention kernel a call runs and into how
many key-range parts its keys are split.

Checks the block's calls against the dispatch the kernels document (video self on CTA
pairs, a2v on the persistent one-key-tile kernel, v2a split over two CTAs per SM, audio
self-attention on one CTA per query tile), the rules that pick each family, the split
invariants (no empty part, explicit part counts honoured up to the key tiles), and the size
rules without a device.
"""
import itertools

import pytest

from joint_audio_video_flash_b200 import build, ltxattn, workloads

SMS = 148


@pytest.fixture(scope="module", autouse=True)
def lib():
    build.build()
    ltxattn.load()


def plan(q_len, kv_len, valid, batch, heads, d, splits=0, sms=SMS):
    return ltxattn.forward_plan(q_len, kv_len, valid, batch, heads, d, splits, sms)


def test_block768_calls():
    _, calls = workloads.configs()["block768"]
    got = {c.name: plan(c.q_len, c.kv_len, c.kv_valid_len, c.batch, c.heads, c.head_dim)
           for c in calls}
    assert got["video_self"] == (ltxattn.KERNEL_PAIR, 1)
    assert got["a2v"] == (ltxattn.KERNEL_A2V, 1)
    assert got["audio_self"] == (ltxattn.KERNEL_ONE_TILE, 1)
    kernel, parts = got["v2a"]
    assert kernel == ltxattn.KERNEL_ONE_TILE_DUAL and parts == 4


def ceil_div(a, b):
    return -(-a // b)


SIZES = list(itertools.product((1, 100, 128, 300, 1025, 15360), (1, 126, 300, 2048, 15360),
                               (1, 2), (1, 8, 32), (64, 128)))


@pytest.mark.parametrize("q_len,kv_valid,batch,heads,d", SIZES)
def test_family_rules_and_parts(q_len, kv_valid, batch, heads, d):
    kernel, parts = plan(q_len, kv_valid, kv_valid, batch, heads, d)
    qt, kt = ceil_div(q_len, 128), ceil_div(kv_valid, 128)
    assert 1 <= parts <= kt
    short_kv = parts == 1 and kt <= 2 and batch * heads * qt > SMS
    if short_kv:
        want = ltxattn.KERNEL_A2V if (d == 64 and kt == 1) else ltxattn.KERNEL_SHORT_KV
        assert kernel == want
    elif d == 128 and parts == 1 and qt >= 8:
        assert kernel == ltxattn.KERNEL_PAIR
    elif d == 64 and kt > 2 and qt <= 1:
        assert kernel == ltxattn.KERNEL_ONE_TILE_DUAL
    else:
        assert kernel == (ltxattn.KERNEL_TWO_TILES if qt >= 2 else ltxattn.KERNEL_ONE_TILE)
    # splits only when the CTAs of one part (two query tiles per CTA on the two-tile
    # kernels) leave SMs idle, and only over at least 4 key tiles
    q_ctas = ceil_div(qt, 2) if qt >= 2 else qt
    if batch * heads * q_ctas >= SMS or kt < 4:
        assert parts == 1


@pytest.mark.parametrize("kv_valid,splits", [(1000, 3), (4000, 7), (15360, 9), (300, 5),
                                             (128, 4), (2990, 64)])
def test_explicit_parts_have_no_empty_part(kv_valid, splits):
    kernel, parts = plan(126, kv_valid, kv_valid, 2, 4, 64, splits)
    kt = ceil_div(kv_valid, 128)
    per = ceil_div(kt, min(splits, kt))
    assert parts == ceil_div(kt, per) and parts <= min(splits, kt)
    assert (parts - 1) * per < kt  # the last part holds at least one key tile


def test_more_sms_split_more():
    # a small query side over a long key side: more SMs, at least as many parts
    _, p148 = plan(126, 15360, 15360, 2, 32, 64, 0, 148)
    _, p1000 = plan(126, 15360, 15360, 2, 32, 64, 0, 1000)
    assert p1000 >= p148


def test_size_rules_without_a_device():
    bad_args = [(0, 128, 128, 1, 1, 64, 0, SMS), (128, 128, 129, 1, 1, 64, 0, SMS),
                (128, 128, 128, 1, 1, 64, -1, SMS), (128, 128, 128, 1, 1, 64, 0, 0),
                (128, 128, 0, 1, 1, 64, 0, SMS)]
    for a in bad_args:
        with pytest.raises(ltxattn.LtxAttnError) as e:
            ltxattn.forward_plan(*a)
        assert e.value.status == ltxattn.ERR_INVALID_ARG
    with pytest.raises(ltxattn.LtxAttnError) as e:
        ltxattn.forward_plan(128, 128, 128, 1, 1, 96, 0, SMS)
    assert e.value.status == ltxattn.ERR_UNSUPPORTED
