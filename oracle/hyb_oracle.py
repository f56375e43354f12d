"""fp64 CPU oracle for the hybrid GQA attention core (Spark-X2.5 / X2.6-4B).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
/ ``--impl reference`` legs of ``bench.py`` use it.  It shares no code with
the CUDA library and does not import it.

It is the plain definition of what the CUDA kernels compute, written out
step by step in float64 with numpy:

* explicit cos/sin rotate-half RoPE per layer type,
* an explicit 4x repeat of the KV heads (query head h reads KV head h // 4),
* an explicit dense boolean mask per layer type,
* max-subtracted softmax, P @ V,
* the head-wise sigmoid output gate.

Sources (web pages; titles abbreviated as below):

[TEARDOWN] "百万 Token 塞进 4B 是怎么做到的？星火 X2.5 的长上下文架构拆解与显存博弈"
           (hotelren.com) -- the config.json / modeling_spark.py teardown.
[LAPTOP]   "不用高显存卡也能跑！4B参数挑战百万上下文，笔记本就能玩" (m.163.com).
[X26BASE]  the Spark-X2.6-4B-Base config walkthrough (lqnn.cn).
[CONFIG]   "读懂Spark-X2.6-4B的config.json：混合注意力与1M上下文的架构入门路线图"
           (sheratonhq.com).

Readings taken where the pages are silent:
* window edge: a sliding query at index t sees keys j with 0 <= t - j <= 511
  (512 keys including itself);
* softmax scale 1/sqrt(256) = 1/16, no soft-cap, no sinks;
* rotate-half pairs (k, k + R/2) inside the rotary sub-vector, with
  inv_freq_k = theta ** (-2k / R) and R the rotary dimension (64 on full
  layers, 256 on sliding layers);
* the gate multiplies the normalised attention output, one scalar per
  (token, head), sigmoid taken in floating point;
* token position = its sequence index unless positions are given.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# Model constants.  [TEARDOWN] §"省显存的第二板斧：GQA、融合投影与输出门控":
# 16 query heads, 4 KV heads, 4 query heads per KV head, head_dim 256.
# [TEARDOWN] §"混合注意力" and [X26BASE] §"滑动窗口 512": window of 512.
# ---------------------------------------------------------------------------
N_Q_HEADS = 16
N_KV_HEADS = 4
GROUP = N_Q_HEADS // N_KV_HEADS
HEAD_DIM = 256
WINDOW = 512
N_LAYERS = 36

SLIDING = 0
FULL = 1

# [TEARDOWN] §"滑动窗口的补救：分层 RoPE 与局部/全局分工" (rope_parameters) and
# [X26BASE] §"全局注意力 + 5M 基频 RoPE": full layers use theta 5e6 with
# partial_rotary_factor 0.25 (the first 64 of 256 dims); sliding layers use
# theta 1e4 with factor 1.0 (all 256 dims).
ROPE_THETA = {SLIDING: 1.0e4, FULL: 5.0e6}
PARTIAL_ROTARY_FACTOR = {SLIDING: 1.0, FULL: 0.25}


def rotary_dim(lt: int) -> int:
    return int(HEAD_DIM * PARTIAL_ROTARY_FACTOR[lt])


def window_of(lt: int):
    """Sliding layers see 512 keys; full layers see the whole prefix (None)."""
    return WINDOW if lt == SLIDING else None


def layer_type(i: int) -> int:
    """Layer schedule: full attention at indices 3, 7, ..., 35, sliding elsewhere.

    [TEARDOWN] §"混合注意力" lists the full indices (3, 7, 11 ... 35);
    [LAPTOP] §"27层滑动窗口加9层全局层" gives the 3-sliding + 1-full pattern
    repeated 9 times.  An index past the schedule falls back to full
    attention, as the decoder-layer code quoted in [TEARDOWN] does.
    """
    if i >= N_LAYERS:
        return FULL
    return FULL if i % 4 == 3 else SLIDING


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------
def rope_angles(pos: np.ndarray, theta: float, rdim: int) -> np.ndarray:
    """phi[..., k] = pos * theta ** (-2k / rdim) for k < rdim / 2, in float64."""
    k = np.arange(rdim // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * k / rdim)
    return np.asarray(pos, dtype=np.float64)[..., None] * inv_freq


def rope(x: np.ndarray, pos: np.ndarray, theta: float, rdim: int) -> np.ndarray:
    """Rotate-half RoPE on the first ``rdim`` dims of the last axis.

    x: [..., T, n_heads, HEAD_DIM] float64; pos: [..., T] integer positions.
    For k < rdim/2 with phi = pos * inv_freq_k:
        x'[k]          = x[k] cos(phi) - x[k + rdim/2] sin(phi)
        x'[k + rdim/2] = x[k + rdim/2] cos(phi) + x[k] sin(phi)
    dims >= rdim pass through unchanged ([X26BASE] §"全局注意力 + 5M 基频 RoPE":
    on full layers only the first 64 dims rotate).
    """
    x = np.asarray(x, dtype=np.float64)
    half = rdim // 2
    phi = rope_angles(pos, theta, rdim)[..., None, :]   # [..., T, 1, half]
    c, s = np.cos(phi), np.sin(phi)
    x1 = x[..., :half]
    x2 = x[..., half:rdim]
    out = x.copy()
    out[..., :half] = x1 * c - x2 * s
    out[..., half:rdim] = x2 * c + x1 * s
    return out


def rope_layer(x, pos, lt):
    return rope(x, pos, ROPE_THETA[lt], rotary_dim(lt))


# ---------------------------------------------------------------------------
# Masked GQA attention with the head-wise gate
# ---------------------------------------------------------------------------
def repeat_kv(x: np.ndarray, n_rep: int = GROUP) -> np.ndarray:
    """[Tk, KVH, D] -> [Tk, KVH * n_rep, D], query head h reading KV head h // n_rep.

    [LAPTOP] §"分组查询注意力": every 4 query heads share one KV head; the
    grouping is contiguous.
    """
    return np.repeat(x, n_rep, axis=1)


def dense_mask(q_idx: np.ndarray, k_idx: np.ndarray, window) -> np.ndarray:
    """M[t, j] = key j visible to query t: causal, and inside the window if any.

    [TEARDOWN] §"混合注意力" (create_causal_mask for full layers,
    create_sliding_window_causal_mask for sliding ones).
    """
    qi = np.asarray(q_idx)[:, None]
    kj = np.asarray(k_idx)[None, :]
    m = kj <= qi
    if window is not None:
        m &= (qi - kj) < window
    return m


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-np.asarray(x, dtype=np.float64)))


def gqa_attention(q, k, v, q_idx, k_idx, window, gate=None, scale=None):
    """One sequence.  q [Tq, H, D] (already roped), k/v [Tk, KVH, D] (k roped).

    q_idx [Tq], k_idx [Tk]: sequence indices used by the mask.
    gate [Tq, H] raw gate scores or None.
    Returns [Tq, H, D] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    n_rep = q.shape[1] // k.shape[1]
    kr = repeat_kv(np.asarray(k, dtype=np.float64), n_rep)
    vr = repeat_kv(np.asarray(v, dtype=np.float64), n_rep)
    if scale is None:
        scale = 1.0 / np.sqrt(q.shape[-1])
    mask = dense_mask(q_idx, k_idx, window)                 # [Tq, Tk]
    # scores s[h, t, j] = q[t, h] . k[j, h] as one matrix product per head
    s = np.matmul(q.transpose(1, 0, 2), kr.transpose(1, 2, 0)) * scale
    s = np.where(mask[None], s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)                    # fully masked row -> all zero
    p = np.exp(s - m)
    l = p.sum(axis=-1, keepdims=True)
    p = p / np.where(l > 0, l, 1.0)
    # o[t, h] = sum_j p[h, t, j] v[j, h]
    o = np.matmul(p, vr.transpose(1, 0, 2)).transpose(1, 0, 2)
    if gate is not None:
        # [TEARDOWN] §"省显存的第二板斧": attn_output * sigmoid(gate_score.float()),
        # one score per head.
        o = o * sigmoid(gate)[..., None]
    return o


# ---------------------------------------------------------------------------
# Whole calls, mirroring the library's three operations
# ---------------------------------------------------------------------------
def prefill(q, k, v, gate, pos, lt, rows=None, start=None,
            hist_k=None, hist_v=None, hist_idx=None):
    """Prefill attention for a batch.

    q [B, T, 16, 256], k/v [B, T, 4, 256]: raw (not roped) values.
    gate [B, T, 16] or None; pos [B, T] RoPE positions; lt layer type.
    rows: indices of the query tokens to compute (default: all).
    start [B]: sequence index of token 0 of each sequence (default 0); token t
    has sequence index start + t, which the mask uses.
    Optional history (earlier tokens of the same sequences, e.g. a KV cache's
    content): hist_k / hist_v [B][L_b, 4, 256] with K already roped, and
    hist_idx [B][L_b] their sequence indices (all < start).
    Returns [B, len(rows), 16, 256] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, T = q.shape[:2]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    out = np.zeros((B, len(rows), q.shape[2], q.shape[3]))
    for b in range(B):
        s0 = 0 if start is None else int(start[b])
        qr = rope_layer(q[b, rows], pos[b, rows], lt)
        keys_k = rope_layer(k[b], pos[b], lt)
        keys_v = v[b]
        k_idx = s0 + np.arange(T)
        if hist_k is not None and len(hist_idx[b]) > 0:
            keys_k = np.concatenate([np.asarray(hist_k[b], np.float64), keys_k], axis=0)
            keys_v = np.concatenate([np.asarray(hist_v[b], np.float64), keys_v], axis=0)
            k_idx = np.concatenate([np.asarray(hist_idx[b]), k_idx])
        g = None if gate is None else np.asarray(gate[b, rows], np.float64)
        out[b] = gqa_attention(qr, keys_k, keys_v, s0 + rows, k_idx, window_of(lt), g)
    return out


def decode(q, gate, qpos, cache_k, cache_v, cache_idx, lt):
    """One decode step for a batch.

    q [B, 16, 256] raw query, gate [B, 16] or None, qpos [B] RoPE positions,
    cache_k/cache_v [B][L_b, 4, 256] cached keys (already roped) and values,
    cache_idx [B][L_b] their sequence indices (any order; the current token
    is in the cache and has the largest index).
    Returns [B, 16, 256] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    B = q.shape[0]
    out = np.zeros(q.shape)
    for b in range(B):
        idx = np.asarray(cache_idx[b])
        qi = int(idx.max())
        qr = rope_layer(q[b][None], np.array([qpos[b]]), lt)      # [1, H, D]
        g = None if gate is None else np.asarray(gate[b], np.float64)[None]
        out[b] = gqa_attention(qr, cache_k[b], cache_v[b], np.array([qi]), idx,
                               window_of(lt), g)[0]
    return out


def decode_group(q_rows, k, v, q_idx, k_idx, lt, gate=None):
    """One decode query for the query heads of a single KV group.

    The same definition as gqa_attention, written per group (the grouping of
    [LAPTOP] §"分组查询注意力" applied by indexing instead of repeating K/V),
    so that a history of ~10^6 keys fits in host memory.
    q_rows [G, D] the group's query heads, already roped; k / v [L, D] that
    KV head's keys (roped) and values; k_idx [L] their sequence indices; the
    query sits at sequence index q_idx.  gate [G] raw gate scores or None.
    Returns [G, D] float64.
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    visible = dense_mask(np.array([q_idx]), np.asarray(k_idx), window_of(lt))[0]
    s = (q_rows @ k.T) / np.sqrt(q_rows.shape[-1])          # [G, L]
    s = np.where(visible[None], s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    p = np.exp(s - m)
    o = (p @ v) / p.sum(axis=-1, keepdims=True)
    if gate is not None:
        o = o * sigmoid(gate)[:, None]
    return o


def decode_partial(q, qpos, cache_k, cache_v, lt):
    """One decode query per sequence against a part of its full-layer history
    (the keys one GPU holds when the history is spread over several), without
    the gate.

    q [B, 16, 256] raw query, qpos [B] RoPE positions, cache_k / cache_v
    [B][L_b, 4, 256] this part's keys (roped) and values.  Every key of a
    full layer precedes the query, so all are visible.
    Returns (o [B, 16, 256], lse2 [B, 16]) float64: o the softmax-normalised
    output over these keys, lse2 = log2 sum_j exp(q . k_j / 16).  A sequence
    with no keys here gives o = 0 and lse2 = -inf.
    """
    assert lt == FULL, "only full layers are spread over several GPUs"
    q = np.asarray(q, dtype=np.float64)
    B, H, D = q.shape
    o = np.zeros((B, H, D))
    lse2 = np.full((B, H), -np.inf)
    for b in range(B):
        k = np.asarray(cache_k[b], np.float64)
        v = np.asarray(cache_v[b], np.float64)
        if k.shape[0] == 0:
            continue
        qr = rope_layer(q[b][None], np.array([qpos[b]]), lt)[0]     # [H, D]
        for h in range(H):
            kv = h // (H // k.shape[1])                              # query head h reads KV head h // 4
            s = (k[:, kv] @ qr[h]) / np.sqrt(D)
            m = s.max()
            p = np.exp(s - m)
            o[b, h] = (p @ v[:, kv]) / p.sum()
            lse2[b, h] = (m + np.log(p.sum())) / np.log(2.0)
    return o, lse2


def merge_partials(o_parts, lse2_parts, gate=None):
    """Attention over the union of the parts from each part's normalised
    output and log-sum-exp: o = sum_p 2^lse2_p o_p / sum_p 2^lse2_p (parts
    with lse2 = -inf hold no keys), then the head-wise sigmoid gate.

    o_parts [P, B, 16, 256], lse2_parts [P, B, 16], gate [B, 16] or None.
    Returns [B, 16, 256] float64.
    """
    o_parts = np.asarray(o_parts, np.float64)
    lse2 = np.asarray(lse2_parts, np.float64)
    m = lse2.max(axis=0)                                             # [B, H]
    safe = np.where(np.isfinite(m), m, 0.0)
    w = np.where(np.isfinite(lse2), np.exp2(lse2 - safe[None]), 0.0)  # [P, B, H]
    den = w.sum(axis=0)
    o = (w[..., None] * o_parts).sum(axis=0) / np.where(den > 0, den, 1.0)[..., None]
    if gate is not None:
        o = o * sigmoid(np.asarray(gate, np.float64))[..., None]
    return o


# ---------------------------------------------------------------------------
# Projections around the attention core
# ---------------------------------------------------------------------------
def linear(x, w):
    """y = x W^T with W in the [out_features, in_features] layout of the
    q_k_v_proj / gate / o_proj weights ([TEARDOWN] §"省显存的第二板斧")."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w, dtype=np.float64).T


def to_bf16(x):
    """Round to bfloat16 (round to nearest even) and back to float64: the
    model's activations between the projections and the attention are bf16
    tensors ([CONFIG] §"模型身份与硬件画像": dtype bfloat16)."""
    import torch
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def attention_layer(hidden, w_qkv, w_gate, w_o, pos, lt, rows=None):
    """One attention layer for prefill ([TEARDOWN] §"省显存的第二板斧"):
    qkv = hidden W_qkv^T, sliced q | k | v; gate = hidden W_g^T; the attention
    of prefill() on them; out = attention(rows) W_o^T.  The three intermediate
    tensors are rounded to bf16, as the model's tensors are.
    hidden [B, T, 2560]; w_qkv [6144, 2560]; w_gate [16, 2560] or None;
    w_o [2560, 4096].  Returns [B, len(rows), 2560] float64."""
    hidden = np.asarray(hidden, dtype=np.float64)
    B, T = hidden.shape[:2]
    qkv = to_bf16(linear(hidden, w_qkv))
    q = qkv[..., :N_Q_HEADS * HEAD_DIM].reshape(B, T, N_Q_HEADS, HEAD_DIM)
    k = qkv[..., N_Q_HEADS * HEAD_DIM:(N_Q_HEADS + N_KV_HEADS) * HEAD_DIM].reshape(B, T, N_KV_HEADS, HEAD_DIM)
    v = qkv[..., (N_Q_HEADS + N_KV_HEADS) * HEAD_DIM:].reshape(B, T, N_KV_HEADS, HEAD_DIM)
    gate = None if w_gate is None else to_bf16(linear(hidden, w_gate))
    o = to_bf16(prefill(q, k, v, gate, pos, lt, rows=rows))
    return linear(o.reshape(B, o.shape[1], N_Q_HEADS * HEAD_DIM), w_o)


def attention_layer_decode(hidden, w_qkv, w_gate, w_o, qpos, hist_k, hist_v, hist_idx, lt):
    """One attention layer for a decode step: the new token of each sequence
    goes through the projections, its K/V join the history, and the query
    attends (the decode definition of decode()).
    hidden [B, 2560] the new tokens, each at sequence index and RoPE position
    qpos[b]; hist_k / hist_v [B][L_b, 4, 256] the cached history (K roped),
    hist_idx [B][L_b] its sequence indices.  Intermediates rounded to bf16 as
    in attention_layer.  Returns [B, 2560] float64."""
    hidden = np.asarray(hidden, dtype=np.float64)
    B = hidden.shape[0]
    qkv = to_bf16(linear(hidden, w_qkv))
    q = qkv[:, :N_Q_HEADS * HEAD_DIM].reshape(B, N_Q_HEADS, HEAD_DIM)
    k = qkv[:, N_Q_HEADS * HEAD_DIM:(N_Q_HEADS + N_KV_HEADS) * HEAD_DIM].reshape(B, N_KV_HEADS, HEAD_DIM)
    v = qkv[:, (N_Q_HEADS + N_KV_HEADS) * HEAD_DIM:].reshape(B, N_KV_HEADS, HEAD_DIM)
    gate = None if w_gate is None else to_bf16(linear(hidden, w_gate))
    keys, vals, idx = [], [], []
    for b in range(B):
        kn = rope_layer(k[b][None], np.array([qpos[b]]), lt)[0]
        keys.append(np.concatenate([np.asarray(hist_k[b], np.float64), kn[None]]))
        vals.append(np.concatenate([np.asarray(hist_v[b], np.float64), v[b][None]]))
        idx.append(np.append(np.asarray(hist_idx[b]), qpos[b]))
    o = to_bf16(decode(q, gate, qpos, keys, vals, idx, lt))
    return linear(o.reshape(B, N_Q_HEADS * HEAD_DIM), w_o)


# ---------------------------------------------------------------------------
# FP8 (e4m3) KV rows
# ---------------------------------------------------------------------------
E4M3_MAX = 448.0


def quantize_e4m3_rows(x):
    """Per-row FP8 e4m3 quantization of KV rows (the 8-bit KV cache the pages'
    deployments use: [LAPTOP] / [12GB] q8_0 KV cache; the e4m3 format and a
    per-row scale are this library's reading).  x [..., 256].
    scale = amax / 448 (fp32); code = e4m3 round-to-nearest-even, saturating
    at +-448, of x * (448 / amax) computed in fp32, as the kernel does (the
    code is an integer decided by floating point, so both sides decide it in
    fp32).  A zero row has scale 0 and zero codes.
    Returns (codes uint8 [..., 256], scale float32 [...])."""
    import torch
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.abs(x32).max(axis=-1)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    inv = np.where(amax > 0, np.float32(E4M3_MAX) / safe, np.float32(0.0)).astype(np.float32)
    scaled = np.clip(x32 * inv[..., None], -E4M3_MAX, E4M3_MAX).astype(np.float32)
    codes = torch.from_numpy(np.ascontiguousarray(scaled)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    return codes, scale


def dequantize_e4m3_rows(codes, scale):
    """code value (e4m3) * scale, in float64."""
    import torch
    vals = torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return vals * np.asarray(scale, dtype=np.float64)[..., None]


# ---------------------------------------------------------------------------
# KV caches: linear (full layers) and the 512-slot ring (sliding layers)
# ---------------------------------------------------------------------------
def linear_slots(length: int, n_new: int) -> np.ndarray:
    """A full-layer cache stores sequence index i at slot i."""
    return np.arange(length, length + n_new)


class RingSim:
    """Host simulator of one sequence's 512-slot ring.

    [LAPTOP] §"百万上下文的真正瓶颈": a sliding layer keeps only the K/V of the
    most recent 512 tokens and drops older ones.  Reading: the write head
    advances one slot per token, modulo 512; each slot is tagged with the
    sequence index it holds (-1 = empty).
    """

    def __init__(self, head0: int = 0, size: int = WINDOW):
        self.size = size
        self.head = head0 % size
        self.length = 0
        self.tag = np.full(size, -1, dtype=np.int64)

    def append(self, n: int) -> np.ndarray:
        """Appends n tokens; returns the slot of each (later writes win)."""
        slots = (self.head + np.arange(n)) % self.size
        for t in range(n):
            self.tag[slots[t]] = self.length + t
        self.head = (self.head + n) % self.size
        self.length += n
        return slots

    @property
    def count(self) -> int:
        return min(self.length, self.size)


# ---------------------------------------------------------------------------
# Closed forms the pages print
# ---------------------------------------------------------------------------
def kv_bytes_per_token_layer(elem_bytes: int = 2) -> int:
    """2 (K and V) x 4 KV heads x 256 dims x 2 bytes = 4096
    ([TEARDOWN] §"先算一笔账：1M 上下文对 4B 模型意味着什么")."""
    return 2 * N_KV_HEADS * HEAD_DIM * elem_bytes


def kv_bytes(n_tokens: int, n_full: int, n_sliding: int) -> int:
    """Hybrid KV bytes: full layers keep every token, sliding ones at most 512."""
    per = kv_bytes_per_token_layer()
    return n_full * per * n_tokens + n_sliding * per * min(n_tokens, WINDOW)


def attention_pairs(n: int, lt: int) -> int:
    """(query, key) pairs one head attends over a causal prefill of n tokens."""
    if lt == FULL or n <= WINDOW:
        return n * (n + 1) // 2
    return WINDOW * (WINDOW + 1) // 2 + (n - WINDOW) * WINDOW


def prefill_flops(n: int, lt: int, n_heads: int = N_Q_HEADS, d: int = HEAD_DIM) -> int:
    """QK^T and PV: 2*d + 2*d flops per (query head, key) pair."""
    return attention_pairs(n, lt) * n_heads * 4 * d
