"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module holds no attention arithmetic: it only draws bf16 tensors.  The
LTX-2 DiT activations the pages describe (768x1280x121 -> 15360 video tokens,
1280x704x241 -> 27280 video tokens, 126 or 252 audio tokens zero-padded to 128
or 256) are stood in for by i.i.d. N(0, 1) values, drawn in fp32 from a seeded
CPU ``torch.Generator`` and rounded to bf16.  Rows at or beyond ``valid`` (the
zero-padded audio tail) are set to exactly zero.
"""
from __future__ import annotations

import torch


def bf16_normal(shape, generator: torch.Generator) -> torch.Tensor:
    """N(0, 1) draws in fp32, rounded to bf16 (round-to-nearest-even)."""
    return torch.randn(tuple(shape), generator=generator, dtype=torch.float32).to(torch.bfloat16)


def make_qkv(batch: int, q_len: int, kv_len: int, heads: int, head_dim: int, seed: int,
             q_valid: int | None = None, kv_valid: int | None = None):
    """(q, k, v) bf16 CPU tensors in BSHD layout, drawn q, k, v in that order from ``seed``.

    Query rows >= ``q_valid`` and key/value rows >= ``kv_valid`` are zero (padding).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = bf16_normal((batch, q_len, heads, head_dim), g)
    k = bf16_normal((batch, kv_len, heads, head_dim), g)
    v = bf16_normal((batch, kv_len, heads, head_dim), g)
    if q_valid is not None and q_valid < q_len:
        q[:, q_valid:] = 0
    if kv_valid is not None and kv_valid < kv_len:
        k[:, kv_valid:] = 0
        v[:, kv_valid:] = 0
    return q, k, v


def sample_rows(batch: int, q_len: int, heads: int, per_head: int, seed: int,
                full_heads=((0, 0),)) -> torch.Tensor:
    """Flat query-row indices (b*q_len + i)*heads + h for parity sampling.

    Every row of each (b, h) in ``full_heads`` plus ``per_head`` seeded random rows
    of every (b, h); sorted and unique.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    idx = []
    for b, h in full_heads:
        i = torch.arange(q_len, dtype=torch.int64)
        idx.append((b * q_len + i) * heads + h)
    for b in range(batch):
        for h in range(heads):
            n = min(per_head, q_len)
            i = torch.randperm(q_len, generator=g)[:n].to(torch.int64)
            idx.append((b * q_len + i) * heads + h)
    return torch.unique(torch.cat(idx))


def rope_tables(length: int, head_dim: int, base: float = 10000.0):
    """Rotary tables for positions 0..length-1: cos, sin of p * base^(-2i/head_dim), fp32.

    Shape [length, head_dim // 2]; pair i of every head at position p turns by that angle.
    These are inputs to the rotary step (the caller owns the positional scheme), computed in
    fp64 and rounded to fp32.
    """
    half = head_dim // 2
    inv_freq = base ** (-torch.arange(half, dtype=torch.float64) * 2.0 / head_dim)
    ang = torch.arange(length, dtype=torch.float64)[:, None] * inv_freq[None, :]
    return torch.cos(ang).to(torch.float32), torch.sin(ang).to(torch.float32)


def make_qk_prologue_inputs(batch: int, seq_len: int, heads: int, head_dim: int, seed: int):
    """(q, k, q_weight, k_weight, cos, sin) for the QK-norm + rotary prologue.

    q, k: bf16 N(0, 1) [batch, seq_len, heads, head_dim]; weights: bf16 1 + 0.1 N(0, 1) over
    heads * head_dim; cos, sin: :func:`rope_tables` for positions 0..seq_len-1.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = bf16_normal((batch, seq_len, heads, head_dim), g)
    k = bf16_normal((batch, seq_len, heads, head_dim), g)
    wq = (1.0 + 0.1 * torch.randn(heads * head_dim, generator=g)).to(torch.bfloat16)
    wk = (1.0 + 0.1 * torch.randn(heads * head_dim, generator=g)).to(torch.bfloat16)
    cos, sin = rope_tables(seq_len, head_dim)
    return q, k, wq, wk, cos, sin
