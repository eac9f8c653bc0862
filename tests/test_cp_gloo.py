"""Context-parallel orchestration on CPU: two gloo ranks (world size 2).

The exchange logic of joint_audio_video_flash_b200.cp (which shards are gathered, in
which order the partial results are merged, which ranks contribute) runs here with the
fp64 oracle standing in for the GPU kernels; each rank's result is compared with the
oracle's attention over the whole sequence.  The kernels themselves are tested on a GPU
(test_cp_gpu.py).
"""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleBackend:
    """partial / combine computed by the fp64 oracle, in the library's result layout."""

    def partial(self, q, k, v, kv_valid_len, scale, o_part=None, lse=None):
        from oracle import oracle
        out, lse_nat = oracle.attention(q, k, v, scale, kv_valid_len=kv_valid_len,
                                        return_lse=True)
        b, lq, h, d = out.shape
        rp = -(-lq // 128) * 128
        o = torch.zeros(b, h, rp, d, dtype=torch.float32)
        o[:, :, :lq] = torch.from_numpy(out).permute(0, 2, 1, 3).float()
        lt = torch.zeros(b, h, rp, dtype=torch.float32)
        lt[:, :, :lq] = torch.from_numpy(lse_nat * math.log2(math.e)).permute(0, 2, 1).float()
        if o_part is None:
            return o, lt
        o_part.copy_(o)
        lse.copy_(lt)
        return o_part, lse

    def combine(self, o_parts, lses, q_len):
        o = o_parts.double()
        ls = lses.double()
        w = torch.exp2(ls - ls.max(0).values)
        out = (w[..., None] * o).sum(0) / w.sum(0)[..., None]
        return out[:, :, :q_len].permute(0, 2, 1, 3).to(torch.bfloat16).contiguous()


def _run(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from joint_audio_video_flash_b200 import cp, synth
    from oracle import oracle
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    be = OracleBackend()
    res = {}
    # video self-attention, sequence of 300 tokens over 2 ranks (150 each), 2 heads x 64
    n, h, d = 300, 2, 64
    qg, kg, vg = synth.make_qkv(1, n, n, h, d, seed=900)
    ls = cp.shard_len(n, world)
    sl = slice(rank * ls, min(n, (rank + 1) * ls))
    pad = lambda t: torch.nn.functional.pad(t[:, sl], (0, 0, 0, 0, 0, ls - (sl.stop - sl.start)))  # noqa: E731
    out = cp.self_attention(pad(qg), pad(kg), pad(vg), n, dist.group.WORLD, backend=be)
    ref = oracle.attention(qg, kg, vg, d ** -0.5)[:, sl]
    res["self"] = float(np.abs(out[:, : sl.stop - sl.start].double().numpy() - ref).max())
    # an uneven sequence: 257 tokens (129 + 128)
    n2 = 257
    qg2, kg2, vg2 = synth.make_qkv(1, n2, n2, h, d, seed=901)
    ls2 = cp.shard_len(n2, world)
    sl2 = slice(rank * ls2, min(n2, (rank + 1) * ls2))
    pad2 = lambda t: torch.nn.functional.pad(t[:, sl2], (0, 0, 0, 0, 0, ls2 - (sl2.stop - sl2.start)))  # noqa: E731
    out2 = cp.self_attention(pad2(qg2), pad2(kg2), pad2(vg2), n2, dist.group.WORLD, backend=be)
    ref2 = oracle.attention(qg2, kg2, vg2, d ** -0.5)[:, sl2]
    res["self_uneven"] = float(np.abs(out2[:, : sl2.stop - sl2.start].double().numpy() - ref2).max())
    # v2a: 126 audio queries (replicated) over 300 video keys sharded over the ranks
    qa, kv_k, kv_v = synth.make_qkv(2, 126, n, h, d, seed=902)
    kl = torch.nn.functional.pad(kv_k[:, sl], (0, 0, 0, 0, 0, ls - (sl.stop - sl.start)))
    vl = torch.nn.functional.pad(kv_v[:, sl], (0, 0, 0, 0, 0, ls - (sl.stop - sl.start)))
    out3 = cp.cross_attention(qa, kl, vl, n, dist.group.WORLD, backend=be)
    ref3 = oracle.attention(qa, kv_k, kv_v, d ** -0.5)
    res["cross"] = float(np.abs(out3.double().numpy() - ref3).max())
    q.put((rank, res))
    dist.destroy_process_group()


def test_two_ranks_match_whole_sequence_attention():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_run, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, res in results.items():
        for name, err in res.items():
            # bf16 rounding of the merged output (values below 4 in magnitude)
            assert err <= 2e-2, (rank, name, err)


def _run_tiny(rank, world, port, q):
    # 5 tokens over 4 ranks: shards of 2, 2, 1 and 0 real tokens
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from joint_audio_video_flash_b200 import cp, synth
    from oracle import oracle
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    be = OracleBackend()
    n, h, d = 5, 1, 64
    qg, kg, vg = synth.make_qkv(1, n, n, h, d, seed=903)
    ls = cp.shard_len(n, world)
    lo, hi = min(n, rank * ls), min(n, (rank + 1) * ls)
    pad = lambda t: torch.nn.functional.pad(t[:, lo:hi], (0, 0, 0, 0, 0, ls - (hi - lo)))  # noqa: E731
    out = cp.self_attention(pad(qg), pad(kg), pad(vg), n, dist.group.WORLD, backend=be)
    ref = oracle.attention(qg, kg, vg, d ** -0.5)[:, lo:hi]
    err_self = float(np.abs(out[:, : hi - lo].double().numpy() - ref).max()) if hi > lo else 0.0
    qa, _, _ = synth.make_qkv(1, 3, 3, h, d, seed=904)
    out2 = cp.cross_attention(qa, pad(kg), pad(vg), n, dist.group.WORLD, backend=be)
    err_cross = float(np.abs(out2.double().numpy() - oracle.attention(qa, kg, vg, d ** -0.5)).max())
    q.put((rank, {"self": err_self, "cross": err_cross}))
    dist.destroy_process_group()


def test_four_ranks_with_an_empty_shard():
    world, port = 4, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_run_tiny, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=240) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert len(results) == world
    for rank, res in results.items():
        for name, err in res.items():
            assert err <= 2e-2, (rank, name, err)


def test_shard_bounds():
    from joint_audio_video_flash_b200 import cp
    assert cp.shard_len(300, 2) == 150 and cp.shard_len(257, 2) == 129
    assert [cp.shard_valid(257, 2, r) for r in range(2)] == [129, 128]
    assert [cp.shard_valid(5, 4, r) for r in range(4)] == [2, 2, 1, 0]
