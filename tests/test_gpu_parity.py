"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Bar (for bf16 output): max-abs error <= 2e-2 and relative L2 error <= 5e-3 per
call; cosine similarity is reported alongside.  Small and ragged shapes are
compared element by element in full; the full-size workloads in the launch
configuration the benchmark times are compared on sampled query rows (whole
heads plus seeded random rows of every head), which the oracle computes one by
one.
"""
import numpy as np
import pytest
import torch

from joint_audio_video_flash_b200 import build, ltxattn, synth, workloads

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    ltxattn.load()
    ltxattn.create()
    yield
    ltxattn.check()


def gpu_run(q, k, v, kv_valid, scale, num_splits=0):
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    out, used = ltxattn.forward(dq, dk, dv, kv_valid_len=kv_valid, scale=scale,
                                num_splits=num_splits, return_splits=True)
    ltxattn.check()
    return out.cpu(), used


def errors(got_bf16, ref):
    g = got_bf16.to(torch.float64).numpy().reshape(ref.shape)
    assert np.all(np.isfinite(g))
    diff = g - ref
    max_abs = float(np.max(np.abs(diff)))
    rel_l2 = float(np.linalg.norm(diff) / np.linalg.norm(ref))
    cos = float(np.sum(g * ref) / (np.linalg.norm(g) * np.linalg.norm(ref)))
    return max_abs, rel_l2, cos


def assert_parity(got, ref, what=""):
    max_abs, rel_l2, cos = errors(got, ref)
    assert max_abs <= MAX_ABS and rel_l2 <= REL_L2, \
        f"{what}: max_abs={max_abs:.3e} rel_l2={rel_l2:.3e} cos={cos:.6f}"
    return max_abs, rel_l2, cos


def test_tiny_workload_full(oracle):
    _, calls = workloads.configs()["tiny"]
    for c in calls:
        q, k, v = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed)
        got, _ = gpu_run(q, k, v, c.kv_valid_len, c.scale)
        ref = oracle.attention(q, k, v, c.scale, kv_valid_len=c.kv_valid_len)
        assert_parity(got, ref, c.name)


RAGGED = [
    # batch, heads, head_dim, q_len, kv_len, kv_valid
    (1, 1, 64, 1, 1, 1),
    (1, 2, 64, 129, 130, 130),
    (2, 3, 128, 300, 700, 650),
    (2, 2, 64, 128, 128, 126),
    (1, 2, 128, 257, 1, 1),
    (2, 4, 64, 513, 255, 200),
    (1, 1, 128, 127, 1025, 1000),
    (1, 3, 128, 200, 256, 129),
    (2, 2, 64, 256, 256, 252),
    # one query tile over a long key side (two CTAs per SM): split and unsplit
    (2, 3, 64, 100, 1000, 999),
    (1, 2, 64, 64, 300, 290),
    (1, 1, 64, 128, 4096, 4000),
]


@pytest.mark.parametrize("shape", RAGGED, ids=lambda s: "b{}h{}d{}_q{}_kv{}v{}".format(*s))
def test_ragged_shapes_full(oracle, shape):
    b, h, d, lq, lkv, valid = shape
    q, k, v = synth.make_qkv(b, lq, lkv, h, d, seed=100 + lq + lkv + d)
    scale = 1.0 / np.sqrt(d)
    got, _ = gpu_run(q, k, v, valid, scale)
    assert_parity(got, oracle.attention(q, k, v, scale, kv_valid_len=valid), str(shape))


SHORT_KV_WALKS = [
    # more (batch, head, query tile) units than SMs: persistent CTAs cross head
    # boundaries, reloading K/V; one query tile per head makes every tile a new head
    (4, 64, 128, 128, 126, 64),
    (3, 50, 200, 256, 252, 64),
    # eight query tiles per head, two key tiles with the second holding one valid key
    (2, 16, 1000, 256, 129, 64),
    (1, 40, 2000, 300, 256, 64),
    # head_dim 128 (two 64-column boxes per row): one and two key tiles, and a padded
    # text-like key side (1024 rows, 256 valid)
    (1, 64, 300, 128, 100, 128),
    (2, 32, 512, 256, 252, 128),
    (2, 20, 1000, 1024, 256, 128),
]


@pytest.mark.parametrize("shape", SHORT_KV_WALKS,
                         ids=lambda s: "b{}h{}_q{}_kv{}v{}_d{}".format(*s))
def test_short_kv_persistent_walks(oracle, shape):
    b, h, lq, lkv, valid, d = shape
    q, k, v = synth.make_qkv(b, lq, lkv, h, d, seed=31 + lq + h, kv_valid=valid)
    scale = 1.0 / np.sqrt(d)
    got, used = gpu_run(q, k, v, valid, scale)
    assert used == 1
    assert_parity(got, oracle.attention(q, k, v, scale, kv_valid_len=valid), str(shape))


@pytest.mark.parametrize("gain,d", [(0.5, 64), (4.0, 64), (4.0, 128)])
def test_short_kv_second_tile_outgrows_first(oracle, gain, d):
    # two key tiles; the second tile's keys point along query 0, so rows' scores there
    # exceed the first tile's by a little (gain 0.5: large probabilities stored against
    # the first tile's max) or by far more than 2^64 (gain 4: the first tile's P is
    # rescaled to the larger max)
    b, h, lq, lkv, valid = 1, 40, 512, 256, 252
    q, k, v = synth.make_qkv(b, lq, lkv, h, d, seed=41, kv_valid=valid)
    k = k.float()
    k[:, 128:valid] = k[:, 128:valid] * 0.25 + q[:, :1].float() * gain
    k = k.to(torch.bfloat16)
    got, used = gpu_run(q, k, v, valid, 1.0)
    assert used == 1
    assert_parity(got, oracle.attention(q, k, v, 1.0, kv_valid_len=valid), f"gain={gain} d={d}")


@pytest.mark.parametrize("splits", [1, 2, 3, 5, 16, 40])
def test_forced_key_splits(oracle, splits):
    # v2a-like: few query rows, many keys; 2000 valid keys = 16 tiles (ragged last one)
    q, k, v = synth.make_qkv(2, 126, 2048, 4, 64, seed=7, kv_valid=2000)
    ref = oracle.attention(q, k, v, 0.125, kv_valid_len=2000)
    got, used = gpu_run(q, k, v, 2000, 0.125, num_splits=splits)
    assert used == min(splits, 16) or (splits == 5 and used == 4) or (splits == 40 and used == 16)
    assert_parity(got, ref, f"splits={splits}")


def test_split_parts_across_alternating_shapes(oracle):
    # one query tile over a long key side, split into key-range parts; calls of alternating
    # shapes reuse the per-stream workspace of partials
    shapes = [(2, 4, 126, 2048, 2000, 3), (3, 5, 100, 3000, 2999, 4), (2, 4, 126, 2048, 2000, 5),
              (1, 2, 64, 640, 600, 5)]
    for b, h, lq, lkv, valid, splits in shapes + shapes[:1]:
        q, k, v = synth.make_qkv(b, lq, lkv, h, 64, seed=lq + lkv + h, kv_valid=valid)
        got, used = gpu_run(q, k, v, valid, 0.125, num_splits=splits)
        assert used > 1
        assert_parity(got, oracle.attention(q, k, v, 0.125, kv_valid_len=valid),
                      f"b{b} h{h} q{lq} kv{lkv} splits {used}")


@pytest.mark.parametrize("d,splits", [(64, 3), (128, 2), (128, 7)])
def test_forced_key_splits_two_query_tiles(oracle, d, splits):
    # query side of several tiles (odd count: the last CTA's second tile is empty)
    q, k, v = synth.make_qkv(2, 300, 2048, 3, d, seed=17, kv_valid=2000)
    scale = 1.0 / np.sqrt(d)
    ref = oracle.attention(q, k, v, scale, kv_valid_len=2000)
    got, used = gpu_run(q, k, v, 2000, scale, num_splits=splits)
    assert used > 1
    assert_parity(got, ref, f"d={d} splits={splits}")


@pytest.mark.parametrize("lq,d,splits", [(130, 128, 0), (100, 64, 1), (100, 64, 2),
                                         (1100, 128, 1)])  # the last: the CTA-pair kernel
def test_growing_scores_force_rescales(oracle, lq, d, splits):
    # keys ordered so that the running max grows tile after tile (exercises the O rescale)
    q, k, v = synth.make_qkv(1, lq, 1024, 2, d, seed=8)
    ramp = torch.linspace(0.2, 3.0, 1024).view(1, 1024, 1, 1)
    k = (k.float() * ramp + q[:, :1].float() * ramp * 2).to(torch.bfloat16)
    scale = 0.25
    ref = oracle.attention(q, k, v, scale)
    got, _ = gpu_run(q, k, v, 1024, scale, num_splits=splits)
    assert_parity(got, ref, f"ramp lq={lq} d={d} splits={splits}")


def test_large_scores(oracle):
    g = torch.Generator().manual_seed(9)
    q = (torch.randn(1, 200, 2, 64, generator=g) * 3).to(torch.bfloat16)
    k = (torch.randn(1, 640, 2, 64, generator=g) * 3).to(torch.bfloat16)
    v = torch.randn(1, 640, 2, 64, generator=g).to(torch.bfloat16)
    ref = oracle.attention(q, k, v, 1.0)
    got, _ = gpu_run(q, k, v, 640, 1.0)
    assert_parity(got, ref, "large scores")


def test_single_key_and_equal_scores():
    q, k, v = synth.make_qkv(2, 300, 256, 2, 64, seed=10)
    got, _ = gpu_run(q, k, v, 1, 0.125)
    want = v[:, :1].expand(-1, 300, -1, -1)
    assert torch.equal(got, want)  # one key: P = 1 exactly, O = V row exactly
    zq = torch.zeros_like(q)
    got, _ = gpu_run(zq, k, v, 256, 0.125)
    mean = v.to(torch.float64).mean(dim=1, keepdim=True).expand(-1, 300, -1, -1)
    assert (got.to(torch.float64) - mean).abs().max() <= 4e-3


def test_padding_and_head_slices_are_exact():
    q, k, v = synth.make_qkv(2, 128, 128, 4, 64, seed=11, q_valid=126, kv_valid=126)
    base, _ = gpu_run(q, k, v, 126, 0.125)
    k2, v2 = k.clone(), v.clone()
    k2[:, 126:] = 1000.0
    v2[:, 126:] = 12345.0
    padded, _ = gpu_run(q, k2, v2, 126, 0.125)
    assert torch.equal(base, padded)
    lo, _ = gpu_run(q[:, :, :2].contiguous(), k[:, :, :2].contiguous(), v[:, :, :2].contiguous(),
                    126, 0.125)
    hi, _ = gpu_run(q[:, :, 2:].contiguous(), k[:, :, 2:].contiguous(), v[:, :, 2:].contiguous(),
                    126, 0.125)
    assert torch.equal(base, torch.cat([lo, hi], dim=2))


@pytest.mark.parametrize("lq", [384, 100])
def test_deterministic(lq):
    q, k, v = synth.make_qkv(1, lq, 3000, 2, 64, seed=12)
    a, _ = gpu_run(q, k, v, 3000, 0.125, num_splits=4)
    b, _ = gpu_run(q, k, v, 3000, 0.125, num_splits=4)
    assert torch.equal(a, b)


def _sampled(oracle, c, per_head, full_heads, tail_block=0):
    q, k, v = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed,
                             q_valid=c.q_valid, kv_valid=c.kv_valid_len)
    got, used = gpu_run(q, k, v, c.kv_valid_len, c.scale)
    rows = synth.sample_rows(c.batch, c.q_len, c.heads, per_head, seed=c.seed,
                             full_heads=full_heads)
    if tail_block:
        b, h = c.batch - 1, c.heads - 1
        i = torch.arange(c.q_len - tail_block, c.q_len)
        rows = torch.unique(torch.cat([rows, (b * c.q_len + i) * c.heads + h]))
    ref = oracle.attention(q, k, v, c.scale, kv_valid_len=c.kv_valid_len, rows=rows.numpy())
    flat = got.reshape(-1, c.head_dim)[rows]
    return assert_parity(flat, ref, f"{c.name} {c.batch}x{c.q_len}x{c.kv_len}"), used


def test_video_self_15360_sampled(oracle):
    _, calls = workloads.configs()["video15360_b1"]
    _sampled(oracle, calls[0], per_head=8, full_heads=((0, 0),), tail_block=128)


def test_audio_stream_full(oracle):
    _, calls = workloads.configs()["audio_stream"]
    for c in calls:
        q, k, v = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed,
                                 q_valid=c.q_valid, kv_valid=c.kv_valid_len)
        got, _ = gpu_run(q, k, v, c.kv_valid_len, c.scale)
        ref = oracle.attention(q, k, v, c.scale, kv_valid_len=c.kv_valid_len)
        assert_parity(got, ref, c.name)


def test_block768_sampled(oracle):
    _, calls = workloads.configs()["block768"]
    for c in calls:
        _sampled(oracle, c, per_head=4, full_heads=((1, 5),), tail_block=64)


def test_text_cross_attention(oracle):
    # video and audio queries over a padded text context (keys >= 256 masked)
    _, calls = workloads.configs()["text_xattn"]
    for c in calls:
        if c.q_len <= 256:
            q, k, v = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed,
                                     q_valid=c.q_valid, kv_valid=c.kv_valid_len)
            got, _ = gpu_run(q, k, v, c.kv_valid_len, c.scale)
            assert_parity(got, oracle.attention(q, k, v, c.scale, kv_valid_len=c.kv_valid_len),
                          c.name)
        else:
            _sampled(oracle, c, per_head=4, full_heads=((1, 31),), tail_block=128)


def test_longclip_sampled(oracle):
    _, calls = workloads.configs()["longclip"]
    for c in calls:
        _sampled(oracle, c, per_head=4, full_heads=((0, 0),) if c.q_len <= 256 else (),
                 tail_block=144 if c.q_len > 256 else 0)


def test_concurrent_streams_use_separate_workspaces(oracle):
    # key-range splits on two streams at once: each stream has its own partials workspace
    cases = [synth.make_qkv(2, 126, 4096, 4, 64, seed=51, kv_valid=4000),
             synth.make_qkv(1, 300, 3000, 3, 128, seed=52, kv_valid=2990)]
    valids, scales = [4000, 2990], [0.125, 1.0 / np.sqrt(128)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    dev = [[t.cuda() for t in c] for c in cases]
    outs = [torch.empty_like(d[0]) for d in dev]
    torch.cuda.synchronize()
    for rep in range(3):
        for i in range(2):
            with torch.cuda.stream(streams[i]):
                ltxattn.forward(*dev[i], outs[i], kv_valid_len=valids[i], scale=scales[i],
                                num_splits=4 + rep, stream=streams[i])
    torch.cuda.synchronize()
    ltxattn.check()
    for i in range(2):
        q, k, v = cases[i]
        assert_parity(outs[i].cpu(), oracle.attention(q, k, v, scales[i], kv_valid_len=valids[i]),
                      f"stream {i}")


def test_context_survives_destroy_and_create(oracle):
    q, k, v = synth.make_qkv(1, 200, 1000, 2, 64, seed=53)
    ref = oracle.attention(q, k, v, 0.125)
    for _ in range(2):
        ltxattn.destroy()
        with pytest.raises(ltxattn.LtxAttnError) as e:
            ltxattn.forward(q.cuda(), k.cuda(), v.cuda(), scale=0.125)
        assert e.value.status == ltxattn.ERR_NOT_INITIALIZED
        ltxattn.create()
        got, _ = gpu_run(q, k, v, 1000, 0.125, num_splits=3)
        assert_parity(got, ref, "after re-create")


def test_errors_on_device():
    q = torch.zeros(1, 64, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ltxattn.LtxAttnError) as e:
        ltxattn.forward(q, q.clone(), q.clone(), scale=-1.0)
    assert e.value.status == ltxattn.ERR_INVALID_ARG
    big = torch.zeros(1, 64 * 2 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    mis = big[0, 1:1 + 64 * 2 * 64].view(1, 64, 2, 64)  # 2-byte offset
    with pytest.raises(ltxattn.LtxAttnError) as e:
        ltxattn.forward(mis, q.clone(), q.clone())
    assert e.value.status == ltxattn.ERR_MISALIGNED


def test_bounded_wait_reports_timeout_and_context_survives(oracle):
    assert ltxattn.selftest_wait_timeout(1_000_000) == ltxattn.ERR_DEVICE_TIMEOUT
    ltxattn.check()  # status word was cleared
    q, k, v = synth.make_qkv(1, 130, 300, 2, 64, seed=13)
    got, _ = gpu_run(q, k, v, 300, 0.125)
    assert_parity(got, oracle.attention(q, k, v, 0.125), "after self-test")


def test_two_host_threads_share_one_stream(oracle):
    # two host threads enqueue key-split calls of different workspace sizes on one stream,
    # so that one thread grows the stream's workspace while the other launches on it
    import threading
    cases = [synth.make_qkv(2, 126, 1024 * (i + 2), 4, 64, seed=60 + i, kv_valid=1000 * (i + 2))
             for i in range(4)]
    valids = [1000 * (i + 2) for i in range(4)]
    dev = [[t.cuda() for t in c] for c in cases]
    outs = [torch.empty_like(d[0]) for d in dev]
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    errors = []

    def worker(idxs):
        try:
            torch.cuda.set_device(0)
            for rep in range(4):
                for i in idxs:
                    ltxattn.forward(*dev[i], outs[i], kv_valid_len=valids[i], scale=0.125,
                                    num_splits=2 + (rep + i) % 4, stream=stream)
        except Exception as e:  # reported below, on the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(ix,)) for ix in ([0, 3], [1, 2])]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    ltxattn.check(stream)
    for i, (q, k, v) in enumerate(cases):
        assert_parity(outs[i].cpu(), oracle.attention(q, k, v, 0.125, kv_valid_len=valids[i]),
                      f"thread case {i}")


PAIR_SHAPES = [
    # head_dim 128, at least 8 query tiles, unsplit: the CTA-pair kernel (cta_group::2).
    # batch, heads, q_len, kv_len, kv_valid
    (1, 1, 1024, 1024, 1024),    # two full pairs, one head
    (2, 3, 1100, 1100, 1100),    # 9 query tiles: the last pair holds one real tile of four
    (1, 2, 2048, 1000, 999),     # ragged last key tile (and a key side of 8 tiles)
    (1, 2, 1280, 128, 77),       # one key tile, 77 valid keys (too few query tiles for the
                                 # persistent short-key kernel)
    (2, 2, 1536, 4096, 4000),    # many key tiles, masked tail
    (1, 48, 2100, 300, 290),     # 240 items over at most 74 persistent pairs, three key
                                 # tiles, ragged query and key tails
]


@pytest.mark.parametrize("shape", PAIR_SHAPES, ids=lambda s: "b{}h{}_q{}_kv{}v{}".format(*s))
def test_cta_pair_kernel(oracle, shape):
    b, h, lq, lkv, valid = shape
    q, k, v = synth.make_qkv(b, lq, lkv, h, 128, seed=70 + lq + lkv, kv_valid=valid)
    scale = 128 ** -0.5
    got, used = gpu_run(q, k, v, valid, scale, num_splits=1)  # no key parts: the pair kernel
    assert used == 1
    rows = synth.sample_rows(b, lq, h, 48, seed=lq, full_heads=((b - 1, h - 1),))
    i = torch.arange(lq - 100, lq)
    rows = torch.unique(torch.cat([rows, (0 * lq + i) * h + 0]))
    ref = oracle.attention(q, k, v, scale, kv_valid_len=valid, rows=rows.numpy())
    assert_parity(got.reshape(-1, 128)[rows], ref, str(shape))
