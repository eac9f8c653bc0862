"""Partial attention, the merge of partials, and the context-parallel patterns on one GPU.

ltxattn_forward_partial over uneven key ranges (the last with a padded, masked tail) merged
by ltxattn_combine must give the fp64 oracle's attention over the whole key range, on the
one-tile (two CTAs per SM at head_dim 64), single-tile and two-tile kernel paths.  The
context-parallel module then runs through a real NCCL process group of world size 1.
Same bar as the attention tests: max-abs <= 2e-2, relative L2 <= 5e-3.
"""
import numpy as np
import pytest
import torch

from joint_audio_video_flash_b200 import build, cp, ltxattn, synth
from oracle import oracle

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


@pytest.mark.parametrize("b,lq,lkv,valid,h,d,cuts", [
    (2, 126, 1000, 990, 2, 64, (300, 700)),     # one query tile, head_dim 64: two CTAs per SM
    (1, 100, 640, 640, 2, 128, (128, 256)),     # one query tile, head_dim 128
    (2, 300, 777, 760, 2, 64, (250, 500)),      # three query tiles: two per CTA
    (1, 260, 512, 512, 3, 128, (1, 256)),       # a one-key range
], ids=["q126d64", "q100d128", "q300d64", "q260d128"])
def test_partials_merge_to_full_attention(b, lq, lkv, valid, h, d, cuts):
    q, k, v = synth.make_qkv(b, lq, lkv, h, d, seed=lq + lkv, kv_valid=valid)
    dq, dk, dv = (t.cuda() for t in (q, k, v))
    bounds = [0, *cuts, lkv]
    parts = []
    for a, e in zip(bounds[:-1], bounds[1:]):
        kp, vp = dk[:, a:e].contiguous(), dv[:, a:e].contiguous()
        part_valid = max(0, min(e, valid) - a)
        if part_valid > 0:
            parts.append(ltxattn.forward_partial(dq, kp, vp, kv_valid_len=part_valid))
    o_parts = torch.stack([o for o, _ in parts]).contiguous()
    lses = torch.stack([l for _, l in parts]).contiguous()
    out = ltxattn.combine(o_parts, lses, lq)
    ltxattn.check()
    _check(out, oracle.attention(q, k, v, d ** -0.5, kv_valid_len=valid), "merged partials")
    # each part's log-sum-exp against the oracle's (natural log -> base 2)
    _, lse_nat = oracle.attention(q, k[:, :cuts[0]], v[:, :cuts[0]], d ** -0.5, return_lse=True)
    got = lses[0, :, :, :lq].permute(0, 2, 1).cpu().double().numpy()
    np.testing.assert_allclose(got, lse_nat * np.log2(np.e), rtol=0, atol=2e-3)


def test_single_part_equals_forward():
    q, k, v = (t.cuda() for t in synth.make_qkv(2, 300, 600, 2, 128, seed=31))
    o, l = ltxattn.forward_partial(q, k, v)
    out = ltxattn.combine(o[None].contiguous(), l[None].contiguous(), 300)
    ref = ltxattn.forward(q, k, v)
    ltxattn.check()
    assert (out.float() - ref.float()).abs().max().item() <= 2 ** -7


def test_context_parallel_world_of_one():
    # the NCCL all-gathers and the merges of the context-parallel module on a real process
    # group (one rank: every gather is a copy)
    import datetime
    import socket

    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        q, k, v = synth.make_qkv(2, 500, 500, 2, 128, seed=41)
        out = cp.self_attention(q.cuda(), k.cuda(), v.cuda(), 500, dist.group.WORLD)
        _check(out, oracle.attention(q, k, v, 128 ** -0.5), "cp self, one rank")
        qa, kvk, kvv = synth.make_qkv(2, 126, 900, 2, 64, seed=42)
        out2 = cp.cross_attention(qa.cuda(), kvk.cuda(), kvv.cuda(), 900, dist.group.WORLD)
        ltxattn.check()
        _check(out2, oracle.attention(qa, kvk, kvv, 64 ** -0.5), "cp cross, one rank")
    finally:
        dist.destroy_process_group()


def test_host_checks():
    q = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ltxattn.LtxAttnError) as e:
        ltxattn.forward_partial(q, q, q, kv_valid_len=0)
    assert e.value.status == ltxattn.ERR_INVALID_ARG
    o = torch.zeros(1, 1, 2, 128, 96, dtype=torch.float32, device="cuda")
    lse = torch.zeros(1, 1, 2, 128, dtype=torch.float32, device="cuda")
    with pytest.raises(ltxattn.LtxAttnError) as e:
        ltxattn.combine(o, lse, 128)
    assert e.value.status == ltxattn.ERR_UNSUPPORTED
