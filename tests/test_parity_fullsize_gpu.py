"""Full-size parity on sampled outputs, in the launch configurations bench.py times.

Each case runs the CUDA path at the workload's full size and compares a
sample of outputs with the fp64 oracle, which computes those rows (or
decode steps) from the same seeded inputs.  Row samples per prefill layer:
every row within 600 of a band edge (the start of the sequence and the
point where the 512-key window becomes full), the first and last 256 rows,
rows around query-tile edges, and 1024 random rows (fixed seeds):

* the 3-sliding + 1-full group prefill at T=32768 into fresh KV caches;
* one full layer at T=131072 without a cache (the same sample, without the
  band-edge block, which the first 256 rows cover for a full layer);
* decode at batch 16 over a 131072-token full-layer cache and a full ring
  (write head at a random offset), after an append;
* 64 steps of append + decode on a full-layer cache prefilled with
  1,048,512 tokens (ending at 1,048,576) and on a full ring, every step and
  all 16 heads of both layers compared;
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


def sample_rows(T, n_random, seed, head=256, tail=256, band_edges=True):
    rng = np.random.default_rng(seed)
    rows = set(range(min(head, T))) | set(range(max(0, T - tail), T))
    if band_edges:   # within 600 of row 0 and of row 511 (first row with a full window)
        rows |= set(range(0, min(T, O.WINDOW - 1 + 601)))
    edges = [e + d for e in (63, 64, 127, 128, 1023, 1024, T // 2) for d in (-1, 0, 1)]
    rows |= {e for e in edges if 0 <= e < T}
    rows |= set(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    return np.array(sorted(rows))


def host_layer(x):
    return {k: f64(x[k]) if k != "pos" else x[k].cpu().numpy() for k in ("q", "k", "v", "gate", "pos")}


def oracle_rows(h, lt, rows, max_rows=128, max_span=4096):
    """The oracle's prefill rows (sorted), a chunk of rows at a time; each chunk
    passes only the tokens its rows can see (from the first key of the
    earliest row's band to the last row), positioned by `start`."""
    rows = np.sort(np.asarray(rows))
    out = []
    i = 0
    while i < len(rows):
        j = i + 1
        while j < len(rows) and j - i < max_rows and (lt == O.FULL or rows[j] - rows[i] <= max_span):
            j += 1
        chunk = rows[i:j]
        lo = 0 if lt == O.FULL else max(0, int(chunk[0]) - (O.WINDOW - 1))
        hi = int(chunk[-1]) + 1
        sl = slice(lo, hi)
        out.append(O.prefill(h["q"][:, sl], h["k"][:, sl], h["v"][:, sl], h["gate"][:, sl], h["pos"][:, sl], lt,
                             rows=chunk - lo, start=[lo]))
        i = j
    return np.concatenate(out, axis=1)


def test_group_prefill_T32768_into_caches(lib):
    T = bench.T_MAIN
    for li, lt in enumerate(bench.GROUP_LAYERS):
        x = synth.prefill_inputs(1, T, seed=bench.layer_seed(1, li), device="cuda")
        cache = lib.KVCache(lt, 1, capacity=T)
        out = lib.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], None, lt, cache=cache)
        torch.cuda.synchronize()
        assert lib.hyb_device_error() == 0
        rows = sample_rows(T, 1024, seed=li)
        ref = oracle_rows(host_layer(x), lt, rows)
        check(out[:, rows], ref, f"group layer {li} (type {lt}), {len(rows)} rows")
        del x, cache, out


def test_full_layer_prefill_T131072(lib):
    T = 131072
    x = synth.prefill_inputs(1, T, seed=bench.layer_seed(1, 3), device="cuda")
    out = lib.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], lib.FULL)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    rows = sample_rows(T, 1024, seed=7, band_edges=False)
    ref = oracle_rows(host_layer(x), O.FULL, rows, max_rows=64)
    check(out[:, rows], ref, f"full layer T=131072, {len(rows)} rows")


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


def test_decode_batch16_L131072_fp8(lib):
    """The bench's FP8 decode configuration: the oracle attends over the
    seeded codes dequantized (snapshot before any library call) and the new
    token rotated, rounded to bf16 and quantized by the oracle's quantizer."""
    B, L = 16, 131072
    cap = L + 4
    r = synth.ring_offset(2)
    full = bench.fill_full_cache(lib, B, L, cap, seed=2, fp8=True)
    ring = bench.fill_ring_cache(lib, B, L, seed=3, head0=r, fp8=True)
    seqs = (0, 9)

    def deq(c, b, rows):
        kc, vc = c.k[b][:, rows].cpu().numpy(), c.v[b][:, rows].cpu().numpy()
        ks, vs = c.k_scale[b][:, rows].cpu().numpy(), c.v_scale[b][:, rows].cpu().numpy()
        return (O.dequantize_e4m3_rows(kc, ks).transpose(1, 0, 2), O.dequantize_e4m3_rows(vc, vs).transpose(1, 0, 2))

    hist_full = {b: deq(full, b, np.arange(L)) for b in seqs}
    n = L + 1
    idx = np.arange(n - 512, n - 1)
    slots = (r + idx) % 512
    hist_ring = [deq(ring, b, slots) for b in range(B)]
    x = synth.decode_query(B, seed=1001, device="cuda")
    lib.hyb_kv_append(full, x["k"], x["v"])
    lib.hyb_kv_append(ring, x["k"], x["v"])
    out_f = lib.hyb_attn_decode(x["q"], x["gate"], full, max_len=cap)
    out_r = lib.hyb_attn_decode(x["q"], x["gate"], ring, max_len=512)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    q, g = f64(x["q"]), f64(x["gate"])
    knew, vnew = f64(x["k"])[:, 0], f64(x["v"])[:, 0]
    vq, vsc = O.quantize_e4m3_rows(vnew)
    vn = O.dequantize_e4m3_rows(vq, vsc)
    for lt, out in ((O.FULL, out_f), (O.SLIDING, out_r)):
        kr = O.to_bf16(O.rope_layer(knew[:, None], np.full((B, 1), n - 1), lt)[:, 0])
        kq, ksc = O.quantize_e4m3_rows(kr)
        kn = O.dequantize_e4m3_rows(kq, ksc)
        if lt == O.FULL:
            for b in seqs:
                kc = np.concatenate([hist_full[b][0], kn[b][None]])
                vc = np.concatenate([hist_full[b][1], vn[b][None]])
                ref = O.decode(q[b:b + 1], g[b:b + 1], [n - 1], [kc], [vc], [np.arange(n)], lt)
                check(out[b:b + 1], ref, f"FP8 full decode seq {b}")
        else:
            kc = [np.concatenate([hist_ring[b][0], kn[b][None]]) for b in range(B)]
            vc = [np.concatenate([hist_ring[b][1], vn[b][None]]) for b in range(B)]
            ref = O.decode(q, g, [n - 1] * B, kc, vc, [np.append(idx, n - 1)] * B, lt)
            check(out, ref, "FP8 sliding decode, 16 sequences")


def test_decode_1m_64_steps(lib):
    """The 1M-token decode workload's two layer types: 64 steps of append +
    decode, each step compared for all 16 heads.  The oracle keeps its own fp64
    history (the seeded cache content, snapshot before any library call, plus
    each step's raw token rotated by the oracle)."""
    n_steps = 64
    cap = 1 << 20
    L0 = cap - n_steps
    r = synth.ring_offset(3)
    full = bench.fill_full_cache(lib, 1, L0, cap, seed=3)
    ring = bench.fill_ring_cache(lib, 1, L0, seed=5, head0=r)
    hk = np.empty((O.N_KV_HEADS, cap, O.HEAD_DIM))
    hv = np.empty((O.N_KV_HEADS, cap, O.HEAD_DIM))
    for h in range(O.N_KV_HEADS):
        hk[h, :L0] = f64(full.k[0, h, :L0])
        hv[h, :L0] = f64(full.v[0, h, :L0])
    # ring: token i (L0 - 512 <= i < L0) at slot (r + i) % 512
    ring_k = f64(ring.k[0]).transpose(1, 0, 2)       # [512 slots, 4, 256]
    ring_v = f64(ring.v[0]).transpose(1, 0, 2)
    win_idx = list(range(L0 - O.WINDOW, L0))
    win_k = [ring_k[(r + i) % O.WINDOW] for i in win_idx]
    win_v = [ring_v[(r + i) % O.WINDOW] for i in win_idx]
    for step in range(n_steps):
        x = synth.decode_query(1, seed=20000 + step, device="cuda")
        lib.hyb_kv_append(full, x["k"], x["v"])
        lib.hyb_kv_append(ring, x["k"], x["v"])
        out_f = lib.hyb_attn_decode(x["q"], x["gate"], full, max_len=cap)
        out_r = lib.hyb_attn_decode(x["q"], x["gate"], ring, max_len=O.WINDOW)
        torch.cuda.synchronize()
        assert lib.hyb_device_error() == 0
        n = L0 + step + 1                            # tokens after the append; the query is token n - 1
        q, g = f64(x["q"])[0], f64(x["gate"])[0]
        knew, vnew = f64(x["k"])[0, 0], f64(x["v"])[0, 0]
        # full layer
        hk[:, n - 1] = O.rope_layer(knew[None], np.array([n - 1]), O.FULL)[0]
        hv[:, n - 1] = vnew
        qf = O.rope_layer(q[None], np.array([n - 1]), O.FULL)[0]
        ref = np.empty((O.N_Q_HEADS, O.HEAD_DIM))
        idx = np.arange(n)
        for kvh in range(O.N_KV_HEADS):
            hs = slice(O.GROUP * kvh, O.GROUP * (kvh + 1))
            ref[hs] = O.decode_group(qf[hs], hk[kvh, :n], hv[kvh, :n], n - 1, idx, O.FULL, g[hs])
        check(out_f[0], ref, f"1M decode step {step}, full layer")
        # sliding layer
        win_idx = win_idx[1:] + [n - 1]
        win_k = win_k[1:] + [O.rope_layer(knew[None], np.array([n - 1]), O.SLIDING)[0]]
        win_v = win_v[1:] + [vnew]
        qs = O.rope_layer(q[None], np.array([n - 1]), O.SLIDING)[0]
        wk, wv = np.stack(win_k), np.stack(win_v)    # [512, 4, 256]
        for kvh in range(O.N_KV_HEADS):
            hs = slice(O.GROUP * kvh, O.GROUP * (kvh + 1))
            ref[hs] = O.decode_group(qs[hs], wk[:, kvh], wv[:, kvh], n - 1, np.array(win_idx), O.SLIDING, g[hs])
        check(out_r[0], ref, f"1M decode step {step}, sliding layer")


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
            rows = sample_rows(C, 32, seed=c, head=48, tail=48, band_edges=False)
            h = host_layer(x)
            ref = O.prefill(h["q"], h["k"], h["v"], h["gate"], h["pos"], lt, rows=rows, start=[start],
                            hist_k=[O.rope_layer(f64(hk), idx, lt)], hist_v=[f64(hv)], hist_idx=[idx])
            check(out[:, rows], ref, f"chunk {c} layer type {lt}")
    assert cache.len.tolist() == [total]
