"""Full-size parity on sampled outputs, in the launch configurations bench.py times.

Each case runs the CUDA path at the workload's full size and compares a
sample of outputs with the fp64 oracle, which computes those rows (or
sequences) one by one from the same seeded inputs:

* the 3-sliding + 1-full group prefill at T=32768 into fresh KV caches:
  first and last 128 rows, rows around the 512-key band edge and tile
  edges, 64 random rows, per layer;
* one full layer at T=131072 without a cache: last 64 rows, first 16 rows,
  tile edges, random rows;
* decode at batch 16 over a 131072-token full-layer cache and a full ring
  (write head at a random offset), after an append: 3 sequences of the full
  layer and all 16 of the sliding layer;
* decode over a 1,048,576-token full-layer cache;
* chunked prefill of 262144 tokens in 8192-token chunks, full and sliding
  layer: rows of the second, a middle and the last chunk.
"""
import numpy as np
import pytest
import torch

import bench
import oracle as O
from full_gqa_attention_partial_b200 import synth

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

MAX_ABS = 2e-2
REL_L2 = 5e-3


def f64(t):
    return t.detach().float().cpu().double().numpy()


def check(got, ref, what):
    got = f64(got) if isinstance(got, torch.Tensor) else got
    assert np.all(np.isfinite(got)), what
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


def sample_rows(T, n_random, seed, head=128, tail=128):
    rng = np.random.default_rng(seed)
    edges = [e + d for e in (63, 64, 127, 128, 511, 512, 1023, 1024, T // 2) for d in (-1, 0, 1)]
    rows = set(range(min(head, T))) | set(range(max(0, T - tail), T)) | {e for e in edges if 0 <= e < T}
    rows |= set(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    return np.array(sorted(rows))


def host_layer(x):
    return {k: f64(x[k]) if k != "pos" else x[k].cpu().numpy() for k in ("q", "k", "v", "gate", "pos")}


def test_group_prefill_T32768_into_caches(lib):
    T = bench.T_MAIN
    for li, lt in enumerate(bench.GROUP_LAYERS):
        x = synth.prefill_inputs(1, T, seed=bench.layer_seed(1, li), device="cuda")
        cache = lib.KVCache(lt, 1, capacity=T)
        out = lib.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], None, lt, cache=cache)
        torch.cuda.synchronize()
        assert lib.hyb_device_error() == 0
        rows = sample_rows(T, 64, seed=li)
        h = host_layer(x)
        ref = O.prefill(h["q"], h["k"], h["v"], h["gate"], h["pos"], lt, rows=rows)
        check(out[:, rows], ref, f"group layer {li} (type {lt})")
        del x, cache, out


def test_full_layer_prefill_T131072(lib):
    T = 131072
    x = synth.prefill_inputs(1, T, seed=bench.layer_seed(1, 3), device="cuda")
    out = lib.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], lib.FULL)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    rows = sample_rows(T, 32, seed=7, head=16, tail=64)
    h = host_layer(x)
    ref = O.prefill(h["q"], h["k"], h["v"], h["gate"], h["pos"], O.FULL, rows=rows)
    check(out[:, rows], ref, "full layer T=131072")


def test_decode_batch16_L131072(lib):
    """Oracle inputs: the seeded cache history (snapshot before any library call
    on it) plus the raw new token, which the oracle rotates itself."""
    B, L = 16, 131072
    cap = L + 2
    r = synth.ring_offset(2)
    full = bench.fill_full_cache(lib, B, L, cap, seed=2)
    ring = bench.fill_ring_cache(lib, B, L, seed=3, head0=r)
    seqs = (0, 7, 15)
    hist_full = {b: (full.k[b, :, :L].permute(1, 0, 2).cpu(), full.v[b, :, :L].permute(1, 0, 2).cpu()) for b in seqs}
    ring_k = ring.k.permute(0, 2, 1, 3).cpu()        # [B, 512, 4, 256], slot-indexed
    ring_v = ring.v.permute(0, 2, 1, 3).cpu()
    x = synth.decode_query(B, seed=1000, device="cuda")
    lib.hyb_kv_append(full, x["k"], x["v"])
    lib.hyb_kv_append(ring, x["k"], x["v"])
    out_f = lib.hyb_attn_decode(x["q"], x["gate"], full, max_len=cap)
    out_r = lib.hyb_attn_decode(x["q"], x["gate"], ring, max_len=512)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    n = L + 1
    q, g = f64(x["q"]), f64(x["gate"])
    knew, vnew = f64(x["k"])[:, 0], f64(x["v"])[:, 0]          # [B, 4, 256] raw
    for lt, out in ((O.FULL, out_f), (O.SLIDING, out_r)):
        kn = O.rope_layer(knew[:, None], np.full((B, 1), n - 1), lt)[:, 0]
        if lt == O.FULL:
            for b in seqs:
                kc = np.concatenate([f64(hist_full[b][0]), kn[b][None]])
                vc = np.concatenate([f64(hist_full[b][1]), vnew[b][None]])
                ref = O.decode(q[b:b + 1], g[b:b + 1], [n - 1], [kc], [vc], [np.arange(n)], lt)
                check(out[b:b + 1], ref, f"full decode seq {b}")
        else:
            # ring: token i (i < L) sits at slot (r + i) % 512; the window is [n - 512, n)
            idx = np.arange(n - 512, n - 1)
            slots = (r + idx) % 512
            kc = [np.concatenate([f64(ring_k[b, slots]), kn[b][None]]) for b in range(B)]
            vc = [np.concatenate([f64(ring_v[b, slots]), vnew[b][None]]) for b in range(B)]
            ref = O.decode(q, g, [n - 1] * B, kc, vc, [np.append(idx, n - 1)] * B, lt)
            check(out, ref, "sliding decode, 16 sequences")


def test_decode_L1M_full_layer(lib):
    L0 = (1 << 20) - 64
    cap = 1 << 20
    full = bench.fill_full_cache(lib, 1, L0, cap, seed=3)
    hist_k = full.k[0, :, :L0].cpu()                     # seeded history, before any library call on it
    hist_v = full.v[0, :, :L0].cpu()
    x = synth.decode_query(1, seed=9000, device="cuda")
    lib.hyb_kv_append(full, x["k"], x["v"])
    out = lib.hyb_attn_decode(x["q"], x["gate"], full, max_len=cap)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    n = L0 + 1
    q, g = f64(x["q"])[0], f64(x["gate"])[0]
    qr = O.rope_layer(q[None], np.array([n - 1]), O.FULL)          # [1, 16, 256]
    kn = O.rope_layer(f64(x["k"])[0], np.array([n - 1]), O.FULL)   # [1, 4, 256]
    vn = f64(x["v"])[0]
    ref = np.zeros((16, 256))
    idx = np.arange(n)
    for kvh in range(4):    # one KV group at a time keeps the fp64 copies at ~4 GB
        kc = np.concatenate([f64(hist_k[kvh]), kn[:, kvh]])[:, None]
        vc = np.concatenate([f64(hist_v[kvh]), vn[:, kvh]])[:, None]
        hs = slice(4 * kvh, 4 * kvh + 4)
        ref[hs] = O.gqa_attention(qr[:, hs], kc, vc, np.array([n - 1]), idx, None, g[None, hs])[0]
        del kc, vc
    check(out[0], ref, "full decode at 1M tokens")


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_chunked_prefill_262144(lib, lt):
    total, C = 262144, 8192
    n_chunks = total // C
    checked = {1, n_chunks // 2, n_chunks - 1}
    cache = lib.KVCache(lt, 1, capacity=total)
    hist_k, hist_v = [], []
    for c in range(n_chunks):
        x = synth.prefill_inputs(1, C, seed=4 + 104729 * c + 7 * lt, device="cuda", start=c * C)
        out = lib.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], None, lt, cache=cache)
        hist_k.append(x["k"].cpu())
        hist_v.append(x["v"].cpu())
        if c in checked:
            torch.cuda.synchronize()
            assert lib.hyb_device_error() == 0
            start = c * C
            lo = 0 if lt == O.FULL else max(0, start - 511)   # keys any row of the chunk can see
            hk = torch.cat(hist_k[:-1], 1)[0, lo:start] if c > 0 else None
            hv = torch.cat(hist_v[:-1], 1)[0, lo:start] if c > 0 else None
            idx = np.arange(lo, start)
            rows = sample_rows(C, 32, seed=c, head=48, tail=48)
            h = host_layer(x)
            ref = O.prefill(h["q"], h["k"], h["v"], h["gate"], h["pos"], lt, rows=rows, start=[start],
                            hist_k=[O.rope_layer(f64(hk), idx, lt)], hist_v=[f64(hv)], hist_idx=[idx])
            check(out[:, rows], ref, f"chunk {c} layer type {lt}")
    assert cache.len.tolist() == [total]
