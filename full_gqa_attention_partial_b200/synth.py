"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Every tensor is bfloat16 drawn i.i.d. from N(0, 1) by
torch's seeded generator, the distribution the workloads specify for Q, K, V
and the gate scores.  Token positions are the sequence indices 0..T-1 (or
start..start+T-1 after a cache prefix).

Layout of a prefill batch follows the fused q_k_v_proj output quoted in the
X2.5 teardown page ("百万 Token 塞进 4B 是怎么做到的？星火 X2.5 的长上下文架构
拆解与显存博弈", §"省显存的第二板斧：GQA、融合投影与输出门控"): one row of
4096 + 1024 + 1024 values per token, sliced into q, k and v.
"""
from __future__ import annotations

import torch

N_Q_HEADS = 16
N_KV_HEADS = 4
HEAD_DIM = 256
Q_DIM = N_Q_HEADS * HEAD_DIM            # 4096
KV_DIM = N_KV_HEADS * HEAD_DIM          # 1024
QKV_DIM = Q_DIM + 2 * KV_DIM            # 6144


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, gen: torch.Generator, device="cpu") -> torch.Tensor:
    """N(0,1) samples drawn in fp32 and rounded to bf16."""
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def prefill_inputs(B: int, T: int, seed: int, device="cpu", start=0):
    """Fused qkv rows [B, T, 6144] with q/k/v views, gate [B, T, 16], pos [B, T]."""
    g = generator(seed, device)
    qkv = randn_bf16((B, T, QKV_DIM), g, device)
    gate = randn_bf16((B, T, N_Q_HEADS), g, device)
    pos = (torch.arange(T, dtype=torch.int32, device=device) + int(start)).repeat(B, 1).contiguous()
    return {
        "qkv": qkv,
        "q": qkv[..., :Q_DIM].unflatten(-1, (N_Q_HEADS, HEAD_DIM)),
        "k": qkv[..., Q_DIM:Q_DIM + KV_DIM].unflatten(-1, (N_KV_HEADS, HEAD_DIM)),
        "v": qkv[..., Q_DIM + KV_DIM:].unflatten(-1, (N_KV_HEADS, HEAD_DIM)),
        "gate": gate,
        "pos": pos,
    }


def decode_query(B: int, seed: int, device="cpu"):
    """One query token per sequence: q [B, 16, 256], gate [B, 16], k/v [B, 1, 4, 256]."""
    g = generator(seed, device)
    return {
        "q": randn_bf16((B, N_Q_HEADS, HEAD_DIM), g, device),
        "gate": randn_bf16((B, N_Q_HEADS), g, device),
        "k": randn_bf16((B, 1, N_KV_HEADS, HEAD_DIM), g, device),
        "v": randn_bf16((B, 1, N_KV_HEADS, HEAD_DIM), g, device),
    }


def fill_cache_randn_(k_cache: torch.Tensor, v_cache: torch.Tensor, n_tokens: int, seed: int):
    """Fills slots [0, n_tokens) of caches laid out [B, KVH, cap, D] with N(0,1) bf16.

    The values stand for keys that are already rotated (a cache written by
    earlier appends); the decode workloads prefill caches this way instead
    of running a long prefill first.
    """
    g = generator(seed, k_cache.device)
    B, KVH, cap, D = k_cache.shape
    n = int(n_tokens)
    # draw one (b, head) row block at a time to bound fp32 scratch memory
    for b in range(B):
        for h in range(KVH):
            k_cache[b, h, :n].copy_(randn_bf16((n, D), g, k_cache.device))
            v_cache[b, h, :n].copy_(randn_bf16((n, D), g, k_cache.device))


def fill_cache_fp8_(k_codes: torch.Tensor, v_codes: torch.Tensor, k_scale: torch.Tensor, v_scale: torch.Tensor,
                    n_tokens: int, seed: int):
    """Fills slots [0, n_tokens) of FP8 caches (codes uint8 [B, KVH, cap, D],
    scales fp32 [B, KVH, cap]) with random e4m3 bit patterns -- random sign,
    exponent field 5..9, random 3-bit mantissa (values 0.25 .. 7.5) -- and
    random scales in [0.1, 0.3]: stored values of magnitude ~0.03 .. 2, no
    NaN codes.  They stand for rows written by earlier appends."""
    g = generator(seed, k_codes.device)
    B, KVH, cap, D = k_codes.shape
    n = int(n_tokens)
    dev = k_codes.device
    for b in range(B):
        for h in range(KVH):
            for codes, scale in ((k_codes, k_scale), (v_codes, v_scale)):
                sign = torch.randint(0, 2, (n, D), generator=g, device=dev, dtype=torch.int32) << 7
                expo = torch.randint(5, 10, (n, D), generator=g, device=dev, dtype=torch.int32) << 3
                mant = torch.randint(0, 8, (n, D), generator=g, device=dev, dtype=torch.int32)
                codes[b, h, :n].copy_((sign | expo | mant).to(torch.uint8))
                scale[b, h, :n].copy_(0.1 + 0.2 * torch.rand(n, generator=g, device=dev))


def ring_offset(seed: int) -> int:
    """Random starting slot of a sliding layer's ring write head, in [0, 512)."""
    g = generator(seed, "cpu")
    return int(torch.randint(0, 512, (1,), generator=g).item())
