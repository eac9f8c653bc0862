"""Attention workloads of one LTX-2 joint audio-video DiT block, with their sizes.

Shapes come from the pages: 15360 video tokens and 126 audio tokens at
768x1280, 121 frames ("LTX-2: replicate audio stream across Ulysses ranks by
default", Description); 27,280 video tokens at 1280x704x241 ("feat(ltx2):
tile-parallel video VAE and the two-stage pipeline", Performance table); the
audio stream padded before attention (same Description).  Heads, head_dim and
batch 2 (a CFG pair) are the workload definitions this library is measured on;
the pages do not print them.

Each call is ``O = softmax(scale * Q K^T + mask) V`` with the mask excluding
keys >= kv_valid_len.  ``q_valid`` is the number of real (unpadded) query rows,
used only to count algorithmic work.
"""
from __future__ import annotations

import math
from dataclasses import dataclass


@dataclass(frozen=True)
class Call:
    name: str            # video_self | audio_self | v2a | a2v | v2t | a2t
    batch: int
    q_len: int
    kv_len: int
    kv_valid_len: int
    heads: int
    head_dim: int
    q_valid: int
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs: 4 * Lq_valid * Lkv_valid * H * d * B (2 for QK^T, 2 for PV)."""
        return 4.0 * self.q_valid * self.kv_valid_len * self.heads * self.head_dim * self.batch

    @property
    def bytes(self) -> float:
        """Algorithmic HBM bytes: bf16 Q, K, V read once and O written once."""
        per_b = 2.0 * self.heads * self.head_dim * (2 * self.q_len + 2 * self.kv_len)
        return per_b * self.batch


def _seed(cfg: int, i: int) -> int:
    return 1234 + 16 * cfg + i


def _audio_stream(cfg: int, batch: int, video: int, audio_pad: int, audio_valid: int,
                  first: int):
    h, d = 32, 64
    return [
        Call("audio_self", batch, audio_pad, audio_pad, audio_valid, h, d, audio_valid,
             _seed(cfg, first)),
        Call("v2a", batch, audio_pad, video, video, h, d, audio_valid, _seed(cfg, first + 1)),
        Call("a2v", batch, video, audio_pad, audio_valid, h, d, video, _seed(cfg, first + 2)),
    ]


def configs() -> dict:
    """The workloads, keyed by a short name; values are (description, [Call, ...])."""
    tiny = [
        Call("video_self", 1, 256, 256, 256, 2, 64, 256, _seed(1, 0)),
        Call("audio_self", 1, 8, 8, 8, 2, 64, 8, _seed(1, 1)),
        Call("v2a", 1, 8, 256, 256, 2, 64, 8, _seed(1, 2)),
        Call("a2v", 1, 256, 8, 8, 2, 64, 256, _seed(1, 3)),
    ]
    return {
        "tiny": ("tiny correctness: B1, 2 heads x 64; video self 256, audio self 8, v2a 8x256, "
                 "a2v 256x8", tiny),
        "video15360_b1": ("video self-attention 768x1280x121 (15360 tokens), B1, 32x128",
                          [Call("video_self", 1, 15360, 15360, 15360, 32, 128, 15360,
                                _seed(2, 0))]),
        "audio_stream": ("audio self 126->128 masked + v2a 126x15360 + a2v 15360x126, B2, 32x64",
                         _audio_stream(3, 2, 15360, 128, 126, 0)),
        "block768": ("full block attention set at 768x1280x121, B2: video self 15360 (32x128) + "
                     "audio self 126->128 masked + v2a + a2v (32x64), back to back on one stream",
                     [Call("video_self", 2, 15360, 15360, 15360, 32, 128, 15360, _seed(4, 0))]
                     + _audio_stream(4, 2, 15360, 128, 126, 1)),
        "ncu_small": ("profiling case sized for Nsight Compute replays: video self B1 8192 "
                      "(32x128, 201 MB of inputs) + a2v and v2a at the 768x1280x121 block size",
                      [Call("video_self", 1, 8192, 8192, 8192, 32, 128, 8192, _seed(6, 0))]
                      + _audio_stream(6, 2, 15360, 128, 126, 1)[1:]),
        "text_xattn": ("text cross-attention at 768x1280x121, B2: video queries 15360 (32x128) "
                       "and audio queries 126->128 (32x64) over a text context padded to 1024 "
                       "tokens with 256 valid (the context length is a reading: the pages "
                       "give none)",
                       [Call("v2t", 2, 15360, 1024, 256, 32, 128, 15360, _seed(7, 0)),
                        Call("a2t", 2, 128, 1024, 256, 32, 64, 126, _seed(7, 1))]),
        "longclip": ("long clip 1280x704x241 (27280 video tokens), audio 252->256 masked, B2: "
                     "video self (32x128) + audio self + v2a + a2v (32x64)",
                     [Call("video_self", 2, 27280, 27280, 27280, 32, 128, 27280, _seed(5, 0))]
                     + _audio_stream(5, 2, 27280, 256, 252, 1)),
    }
