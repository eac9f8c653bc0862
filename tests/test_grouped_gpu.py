"""ltxattn_forward_grouped vs the fp64 oracle (needs a B200).

Calls at head_dim 64 with every valid key in one 128-key tile (a2v, audio self-attention)
share one persistent launch, up to four per launch; every other call runs as
ltxattn_forward runs it.  Each output is compared with the oracle under the same bar as
the single-call tests (max-abs <= 2e-2, relative L2 <= 5e-3).
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


def _parity(got, ref, what):
    g = got.to(torch.float64).numpy().reshape(ref.shape)
    assert np.all(np.isfinite(g)), what
    diff = g - ref
    max_abs = float(np.max(np.abs(diff)))
    rel_l2 = float(np.linalg.norm(diff) / np.linalg.norm(ref))
    assert max_abs <= MAX_ABS and rel_l2 <= REL_L2, \
        f"{what}: max_abs={max_abs:.3e} rel_l2={rel_l2:.3e}"


def _calls(shapes, seed0):
    host, dev = [], []
    for i, (b, h, d, lq, lkv, valid) in enumerate(shapes):
        q, k, v = synth.make_qkv(b, lq, lkv, h, d, seed=seed0 + i, kv_valid=valid)
        host.append((q, k, v, valid, 1.0 / np.sqrt(d)))
        dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
        dev.append(dict(q=dq, k=dk, v=dv, out=torch.full_like(dq, float("nan")),
                        kv_valid_len=valid, scale=1.0 / np.sqrt(d)))
    return host, dev


GROUPS = {
    # a2v-like (ragged query side) + audio self: the block's two one-tile calls, one launch
    "a2v_audio": [(2, 8, 64, 1000, 128, 126), (2, 8, 64, 128, 128, 126)],
    # six eligible calls (two launches of the group kernel) mixed with calls that are not:
    # a v2a-like key split, head_dim 128, two key tiles at head_dim 64
    "mixed": [(2, 8, 64, 1000, 128, 126), (1, 1, 64, 1, 1, 1), (2, 4, 64, 126, 2048, 2000),
              (2, 8, 64, 128, 128, 126), (1, 4, 128, 300, 128, 100), (1, 3, 64, 257, 100, 77),
              (2, 2, 64, 513, 255, 200), (3, 5, 64, 129, 64, 64), (1, 40, 64, 300, 128, 128)],
}


@pytest.mark.parametrize("name", sorted(GROUPS))
def test_grouped_calls_match_the_oracle(oracle, name):
    host, dev = _calls(GROUPS[name], seed0=300)
    ltxattn.forward_grouped(dev)
    ltxattn.check()
    for (q, k, v, valid, scale), c, shape in zip(host, dev, GROUPS[name]):
        ref = oracle.attention(q, k, v, scale, kv_valid_len=valid)
        _parity(c["out"].cpu(), ref, f"{name} {shape}")


def test_grouped_calls_sharing_keys_and_values(oracle):
    # a2v and audio self-attention both read the audio stream's keys and values
    b, h, d = 2, 8, 64
    qv, k, v = synth.make_qkv(b, 700, 128, h, d, seed=77, kv_valid=126)
    qa, _, _ = synth.make_qkv(b, 128, 128, h, d, seed=78, kv_valid=126)
    dk, dv = k.cuda(), v.cuda()
    calls = [dict(q=x.cuda(), k=dk, v=dv, out=torch.empty(x.shape, dtype=x.dtype, device="cuda"),
                  kv_valid_len=126, scale=0.125) for x in (qv, qa)]
    ltxattn.forward_grouped(calls)
    ltxattn.check()
    for x, c in zip((qv, qa), calls):
        _parity(c["out"].cpu(), oracle.attention(x, k, v, 0.125, kv_valid_len=126), "shared kv")


def test_grouped_block768_sampled(oracle):
    # the block's four calls in the launch configuration the benchmark times: video self and
    # v2a on their own kernels, a2v and audio self in one grouped launch
    _, calls = workloads.configs()["block768"]
    host, dev = [], []
    for c in calls:
        q, k, v = synth.make_qkv(c.batch, c.q_len, c.kv_len, c.heads, c.head_dim, c.seed,
                                 q_valid=c.q_valid, kv_valid=c.kv_valid_len)
        host.append((q, k, v))
        dq = q.cuda()
        dev.append(dict(q=dq, k=k.cuda(), v=v.cuda(), out=torch.empty_like(dq),
                        kv_valid_len=c.kv_valid_len, scale=c.scale))
    ltxattn.forward_grouped(dev)
    ltxattn.check()
    for c, (q, k, v), d in zip(calls, host, dev):
        rows = synth.sample_rows(c.batch, c.q_len, c.heads, 4, seed=c.seed, full_heads=((1, 5),))
        ref = oracle.attention(q, k, v, c.scale, kv_valid_len=c.kv_valid_len, rows=rows.numpy())
        _parity(d["out"].cpu().reshape(-1, c.head_dim)[rows], ref, c.name)


def test_grouped_equals_single_calls_on_the_same_kernel():
    # an a2v-shaped call (more query tiles than SMs) runs on the group kernel alone too, so
    # grouping it with others changes nothing in its output, bit for bit
    host, dev = _calls([(2, 8, 64, 20000, 128, 126), (2, 8, 64, 128, 128, 126)], seed0=500)
    ltxattn.forward_grouped(dev)
    alone = ltxattn.forward(dev[0]["q"], dev[0]["k"], dev[0]["v"], kv_valid_len=126,
                            scale=0.125)
    ltxattn.check()
    assert torch.equal(alone, dev[0]["out"])
