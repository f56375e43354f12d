"""Seeded random cases through the whole cache path: two prefill chunks and a
decode step on a cache of random kind (layer type, bf16 or FP8, contiguous
or paged, ring offset), random batch, chunk lengths and gate.  Each call is
compared with the oracle on the history as the cache stores it (read back
and, for FP8, dequantized by the oracle; an FP8 chunk also attends to its
own tokens as stored, which the oracle quantizes itself), so any mismatch in
the tiling, masking, paging or append bookkeeping of an odd size shows up."""
import numpy as np
import pytest
import torch

import oracle as O
from full_gqa_attention_partial_b200 import synth

pytestmark = pytest.mark.gpu

SEEDS = list(range(16))


def f64(t):
    return t.detach().float().cpu().double().numpy()


def check(got, ref, what):
    got = f64(got)
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert max_abs <= 2e-2 and rel <= 5e-3, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


def _case(seed):
    rng = np.random.default_rng(1000 + seed)
    lt = O.FULL if rng.random() < 0.5 else O.SLIDING
    return dict(lt=lt, B=int(rng.integers(1, 4)), T1=int(rng.integers(1, 700)), T2=int(rng.integers(1, 300)),
                fp8=bool(rng.random() < 0.5), paged=bool(lt == O.FULL and rng.random() < 0.5),
                gate=bool(rng.random() < 0.8), head0=[int(h) for h in rng.integers(0, 512, size=3)],
                page=int(rng.choice([64, 128, 256])))


def _make_cache(lib, c):
    kvd = lib.KV_FP8 if c["fp8"] else lib.KV_BF16
    if c["lt"] == O.SLIDING:
        return lib.KVCache(O.SLIDING, c["B"], kv_dtype=kvd, head0=c["head0"][:c["B"]])
    cap = c["T1"] + c["T2"] + 8
    if not c["paged"]:
        return lib.KVCache(O.FULL, c["B"], capacity=cap + (-cap) % 4, kv_dtype=kvd)
    P = c["page"]
    max_pages = (cap + P - 1) // P
    n_pages = c["B"] * max_pages + 2
    g = torch.Generator().manual_seed(7)
    table = torch.randperm(n_pages, generator=g)[: c["B"] * max_pages].view(c["B"], max_pages).to(torch.int32).cuda()
    return lib.KVCache(O.FULL, c["B"], kv_dtype=kvd, page_size=P, n_pages=n_pages, block_table=table)


def _stored_history(cache, c, b):
    """(keys [n, 4, 256], values, sequence indices) the cache holds for sequence b, as stored."""
    n = int(cache.len[b].item())
    if c["lt"] == O.SLIDING:
        tag = cache.tag[b].cpu().numpy()
        slots = np.nonzero(tag >= 0)[0]
        idx = tag[slots]
        where = [(b, s) for s in slots]
    else:
        idx = np.arange(n)
        if c["paged"]:
            P = cache.page_size
            tab = cache.block_table[b].tolist()
            where = [(tab[i // P], i % P) for i in idx]
        else:
            where = [(b, i) for i in idx]
    ks, vs = [], []
    kh, vh = cache.k.cpu(), cache.v.cpu()
    if c["fp8"]:
        ksh, vsh = cache.k_scale.cpu().numpy(), cache.v_scale.cpu().numpy()
    for (lead, row) in where:
        if c["fp8"]:
            ks.append(O.dequantize_e4m3_rows(kh[lead, :, row].numpy(), ksh[lead, :, row]))
            vs.append(O.dequantize_e4m3_rows(vh[lead, :, row].numpy(), vsh[lead, :, row]))
        else:
            ks.append(f64(kh[lead, :, row]))
            vs.append(f64(vh[lead, :, row]))
    shape = (0, 4, 256)
    return (np.stack(ks) if ks else np.zeros(shape)), (np.stack(vs) if vs else np.zeros(shape)), np.asarray(idx)


def _attend_fp8(x, gate, lt, b, start, hk, hv, hidx):
    """The oracle's attention of chunk x over a stored history and the chunk's
    own tokens as an FP8 cache stores them (rotated, rounded to bf16,
    quantized and dequantized by the oracle)."""
    q, k, v, pos = f64(x["q"][b]), f64(x["k"][b]), f64(x["v"][b]), x["pos"][b].cpu().numpy()
    kc = O.dequantize_e4m3_rows(*O.quantize_e4m3_rows(O.to_bf16(O.rope_layer(k, pos, lt))))
    vc = O.dequantize_e4m3_rows(*O.quantize_e4m3_rows(v))
    idx = start + np.arange(q.shape[0])
    return O.gqa_attention(O.rope_layer(q, pos, lt), np.concatenate([hk, kc]), np.concatenate([hv, vc]), idx,
                           np.concatenate([hidx, idx]), O.window_of(lt), None if gate is None else f64(gate[b]))


@pytest.mark.parametrize("seed", SEEDS)
def test_random_cache_path(lib, seed):
    c = _case(seed)
    lt, B = c["lt"], c["B"]
    cache = _make_cache(lib, c)
    start = 0
    for i, T in enumerate((c["T1"], c["T2"])):
        hist = [_stored_history(cache, c, b) for b in range(B)]
        x = synth.prefill_inputs(B, T, seed=5000 + 10 * seed + i, device="cuda", start=start)
        gate = x["gate"] if c["gate"] else None
        out = lib.hyb_attn_prefill(x["q"], x["k"], x["v"], gate, x["pos"], lt, cache=cache)
        torch.cuda.synchronize()
        assert lib.hyb_device_error() == 0
        if c["fp8"]:   # the chunk attends to its own tokens as the FP8 cache stores them
            ref = np.stack([_attend_fp8(x, gate, lt, b, start, *hist[b]) for b in range(B)])
        else:
            ref = O.prefill(f64(x["q"]), f64(x["k"]), f64(x["v"]), None if gate is None else f64(gate),
                            x["pos"].cpu().numpy(), lt, start=[start] * B, hist_k=[h[0] for h in hist],
                            hist_v=[h[1] for h in hist], hist_idx=[h[2] for h in hist])
        check(out, ref, f"{c} chunk {i}")
        start += T
    assert cache.len.tolist() == [start] * B
    # one decode step over the stored history plus the new token, as stored
    xd = synth.decode_query(B, seed=6000 + seed, device="cuda")
    lib.hyb_kv_append(cache, xd["k"], xd["v"])
    gate = xd["gate"] if c["gate"] else None
    out = lib.hyb_attn_decode(xd["q"], gate, cache, max_len=cache.capacity)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    hist = [_stored_history(cache, c, b) for b in range(B)]
    ref = O.decode(f64(xd["q"]), None if gate is None else f64(gate), [start] * B, [h[0] for h in hist],
                   [h[1] for h in hist], [h[2] for h in hist], lt)
    check(out, ref, f"{c} decode")


@pytest.mark.parametrize("seed", SEEDS[:8])
def test_random_cache_path_against_raw_history(lib, seed):
    """The same kind of random case on bf16 caches, but the oracle never reads
    the cache: it gets every raw (unrotated) token of the sequence and applies
    RoPE, masks and the window itself.  A rotation or placement error on the
    append side, which the stored-history comparison above would carry into
    its reference, fails here."""
    c = _case(seed)
    c["fp8"] = False
    lt, B = c["lt"], c["B"]
    cache = _make_cache(lib, c)
    chunks, start = [], 0
    for i, T in enumerate((c["T1"], c["T2"])):
        x = synth.prefill_inputs(B, T, seed=7000 + 10 * seed + i, device="cuda", start=start)
        gate = x["gate"] if c["gate"] else None
        out = lib.hyb_attn_prefill(x["q"], x["k"], x["v"], gate, x["pos"], lt, cache=cache)
        torch.cuda.synchronize()
        assert lib.hyb_device_error() == 0
        chunks.append({k: f64(v) if k != "pos" else v.cpu().numpy() for k, v in x.items() if k != "qkv"})
        whole = {k: np.concatenate([ch[k] for ch in chunks], axis=1) for k in ("q", "k", "v", "gate", "pos")}
        rows = np.arange(start, start + T)
        ref = O.prefill(whole["q"], whole["k"], whole["v"], whole["gate"] if c["gate"] else None, whole["pos"], lt,
                        rows=rows)
        check(out, ref, f"{c} chunk {i} (raw history)")
        start += T
    xd = synth.decode_query(B, seed=8000 + seed, device="cuda")
    lib.hyb_kv_append(cache, xd["k"], xd["v"])
    gate = xd["gate"] if c["gate"] else None
    out = lib.hyb_attn_decode(xd["q"], gate, cache, max_len=cache.capacity)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    n = start + 1
    idx = np.arange(n)
    keys, vals = [], []
    for b in range(B):
        kb = np.concatenate([whole["k"][b], f64(xd["k"])[b]], axis=0)
        keys.append(O.rope_layer(kb, idx, lt))
        vals.append(np.concatenate([whole["v"][b], f64(xd["v"])[b]], axis=0))
    ref = O.decode(f64(xd["q"]), None if gate is None else f64(gate), [start] * B, keys, vals, [idx] * B, lt)
    check(out, ref, f"{c} decode (raw history)")
