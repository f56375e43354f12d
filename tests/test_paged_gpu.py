"""Paged full-layer KV caches (a pool of pages and a block table per
sequence): appends, decode and chunked prefill give the same bits as the
contiguous cache holding the same tokens, whose parity with the oracle the
other suites establish; one decode is also checked against the oracle
directly.  Bad block-table entries raise the page error bit without a fault."""
import numpy as np
import pytest
import torch

import oracle as O
from full_gqa_attention_partial_b200 import synth

pytestmark = pytest.mark.gpu


def f64(t):
    return t.detach().float().cpu().double().numpy()


def _table(B, max_pages, n_pages, seed):
    """Distinct random pool pages for every (sequence, logical page)."""
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g)[: B * max_pages]
    return perm.view(B, max_pages).to(torch.int32).cuda()


def _pair(lib, B, page, max_pages, lens, seed, fp8):
    """A contiguous cache and a paged cache holding the same seeded tokens."""
    kvd = lib.KV_FP8 if fp8 else lib.KV_BF16
    cap = page * max_pages
    flat = lib.KVCache(O.FULL, B, capacity=cap, kv_dtype=kvd)
    n_pages = B * max_pages + 3
    table = _table(B, max_pages, n_pages, seed)
    paged = lib.KVCache(O.FULL, B, kv_dtype=kvd, page_size=page, n_pages=n_pages, block_table=table)
    n = max(lens)
    if fp8:
        synth.fill_cache_fp8_(flat.k, flat.v, flat.k_scale, flat.v_scale, n, seed)
    else:
        synth.fill_cache_randn_(flat.k, flat.v, n, seed)
    _scatter(flat, paged)
    lt = torch.tensor(lens, dtype=torch.int32, device="cuda")
    flat.len.copy_(lt)
    paged.len.copy_(lt)
    return flat, paged


def _scatter(flat, paged):
    """Copies the contiguous cache's rows into the pool through the table."""
    P = paged.page_size
    tab = paged.block_table.cpu().tolist()
    pairs = [(flat.k, paged.k), (flat.v, paged.v)]
    if flat.k_scale is not None:
        pairs += [(flat.k_scale, paged.k_scale), (flat.v_scale, paged.v_scale)]
    for b, row in enumerate(tab):
        for lp, pp in enumerate(row):
            for src, dst in pairs:
                dst[pp].copy_(src[b, :, lp * P:(lp + 1) * P])


def _gather(paged, b, n):
    """Rows [0, n) of sequence b of a paged cache, as [4, n, ...] tensors."""
    P = paged.page_size
    tab = paged.block_table[b].cpu().tolist()
    outs = []
    for t in (paged.k, paged.v) + ((paged.k_scale, paged.v_scale) if paged.k_scale is not None else ()):
        outs.append(torch.cat([t[tab[lp]] for lp in range((n + P - 1) // P)], dim=1)[:, :n])
    return outs


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("page", [64, 256])
def test_paged_decode_equals_contiguous(lib, fp8, page):
    B, max_pages = 3, 40 if page == 64 else 10
    lens = [2500, 777, 1]                      # mixed lengths, one sequence with a single cached token
    flat, paged = _pair(lib, B, page, max_pages, lens, seed=61 + page, fp8=fp8)
    x = synth.decode_query(B, seed=62, device="cuda")
    outs = []
    for c in (flat, paged):
        lib.hyb_kv_append(c, x["k"], x["v"])
        outs.append(lib.hyb_attn_decode(x["q"], x["gate"], c, max_len=c.capacity))
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    assert torch.equal(paged.len, flat.len)
    for b, n in enumerate(lens):
        got = _gather(paged, b, n + 1)
        ref = [flat.k[b, :, :n + 1], flat.v[b, :, :n + 1]]
        if fp8:
            ref += [flat.k_scale[b, :, :n + 1], flat.v_scale[b, :, :n + 1]]
        for g_, r_ in zip(got, ref):
            assert torch.equal(g_, r_)
    assert torch.equal(outs[0], outs[1])
    if not fp8 and page == 64:
        # and the oracle on the tokens as stored (keys already rotated in the cache)
        keys, vals, idx = [], [], []
        for b, n in enumerate(lens):
            k_, v_ = _gather(paged, b, n + 1)
            keys.append(f64(k_).transpose(1, 0, 2))
            vals.append(f64(v_).transpose(1, 0, 2))
            idx.append(np.arange(n + 1))
        ref = O.decode(f64(x["q"]), f64(x["gate"]), lens, keys, vals, idx, O.FULL)
        got = f64(outs[1])
        max_abs = float(np.abs(got - ref).max())
        rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
        assert max_abs <= 2e-2 and rel <= 5e-3, f"max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


def test_paged_decode_noalloc_and_shared_prefix(lib):
    """Two sequences whose block tables share their first pages (a common
    prefix) read them in place; the allocation-free entry point agrees."""
    B, page, max_pages = 2, 64, 12
    flat, paged = _pair(lib, B, page, max_pages, [700, 700], seed=71, fp8=False)
    # sequence 1 takes sequence 0's first 5 pages; the contiguous copy gets the same rows
    tab = paged.block_table.clone()
    tab[1, :5] = tab[0, :5]
    paged.block_table.copy_(tab)
    flat.k[1, :, :5 * page].copy_(flat.k[0, :, :5 * page])
    flat.v[1, :, :5 * page].copy_(flat.v[0, :, :5 * page])
    x = synth.decode_query(B, seed=72, device="cuda")
    for c in (flat, paged):
        lib.hyb_kv_append(c, x["k"], x["v"])
    a = lib.hyb_attn_decode(x["q"], x["gate"], flat, max_len=flat.capacity)
    b = lib.hyb_attn_decode(x["q"], x["gate"], paged, max_len=paged.capacity)
    c = lib.hyb_attn_decode_noalloc(x["q"], x["gate"], paged, max_len=paged.capacity)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    assert torch.equal(a, b) and torch.equal(b, c)


@pytest.mark.parametrize("fp8", [False, True])
def test_paged_chunked_prefill_equals_contiguous(lib, fp8):
    """Two prefill chunks through a paged cache: the outputs and the cached
    rows equal the contiguous cache's bit for bit (pages of 64 keys, so the
    prefill's 64-key tiles come from scattered pool pages; FP8: the history
    is dequantized through the table)."""
    B, page, max_pages = 2, 64, 16
    kvd = lib.KV_FP8 if fp8 else lib.KV_BF16
    flat = lib.KVCache(O.FULL, B, capacity=page * max_pages, kv_dtype=kvd)
    n_pages = B * max_pages + 5
    paged = lib.KVCache(O.FULL, B, kv_dtype=kvd, page_size=page, n_pages=n_pages,
                        block_table=_table(B, max_pages, n_pages, 81))
    start = 0
    for i, T in enumerate((300, 211)):
        x = synth.prefill_inputs(B, T, seed=82 + i, device="cuda", start=start)
        outs = [lib.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], O.FULL, cache=c)
                for c in (flat, paged)]
        torch.cuda.synchronize()
        assert lib.hyb_device_error() == 0
        assert torch.equal(outs[0], outs[1]), f"chunk {i}"
        start += T
    assert paged.len.tolist() == [start] * B
    for b in range(B):
        got = _gather(paged, b, start)
        ref = [flat.k[b, :, :start], flat.v[b, :, :start]]
        if fp8:
            ref += [flat.k_scale[b, :, :start], flat.v_scale[b, :, :start]]
        for g_, r_ in zip(got, ref):
            assert torch.equal(g_, r_)


def test_paged_layer_decode_equals_contiguous(lib):
    """The whole decode layer (projections, append, attention, o_proj) on a
    paged cache gives the contiguous cache's bits."""
    B, page, max_pages = 2, 128, 8
    flat, paged = _pair(lib, B, page, max_pages, [600, 901], seed=91, fp8=False)
    g = torch.Generator(device="cuda").manual_seed(92)
    hid = lib.HIDDEN
    w_qkv = (torch.randn(6144, hid, generator=g, device="cuda") / hid ** 0.5).to(torch.bfloat16)
    w_gate = (torch.randn(16, hid, generator=g, device="cuda") / hid ** 0.5).to(torch.bfloat16)
    w_o = (torch.randn(hid, 4096, generator=g, device="cuda") / 64.0).to(torch.bfloat16)
    h = torch.randn(B, hid, generator=g, device="cuda").to(torch.bfloat16)
    outs = [lib.hyb_attn_layer_decode(h, w_qkv, w_gate, w_o, c, max_len=c.capacity) for c in (flat, paged)]
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    assert torch.equal(outs[0], outs[1])


def test_bad_block_table_entry_raises_page_error(lib):
    """An entry outside the pool: the append skips the row, decode reads
    zeros for that page; the page bit is raised and nothing faults."""
    B, page, max_pages = 1, 64, 4
    n_pages = 4
    table = torch.arange(max_pages, dtype=torch.int32, device="cuda").view(1, max_pages)
    paged = lib.KVCache(O.FULL, B, kv_dtype=lib.KV_BF16, page_size=page, n_pages=n_pages, block_table=table)
    synth.fill_cache_randn_(paged.k, paged.v, page, 101)   # fills every pool page's rows
    paged.len.fill_(130)                                   # tokens 0..129: logical pages 0, 1, 2
    before = paged.k.clone()
    table[0, 2] = n_pages + 7                              # the append's page is outside the pool
    x = synth.decode_query(B, seed=102, device="cuda")
    lib.hyb_kv_append(paged, x["k"], x["v"])
    torch.cuda.synchronize()
    assert lib.hyb_device_error() & lib.DEV_ERR_PAGE
    assert torch.equal(paged.k, before)                    # nothing written anywhere in the pool
    table[0, 1] = -1                                       # a page inside [0, len) not handed out
    out = lib.hyb_attn_decode(x["q"], x["gate"], paged, max_len=paged.capacity)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() & lib.DEV_ERR_PAGE
    assert torch.isfinite(out.float()).all()
    assert lib.hyb_device_error() == 0                     # the previous read cleared the word


def test_paged_chunked_prefill_matches_oracle(lib):
    """Two prefill chunks and a decode step through a paged cache with pages
    of 64 keys scattered over the pool, compared with the oracle on the raw
    tokens (it rotates the keys and builds the history itself)."""
    B, page, max_pages = 2, 64, 12
    n_pages = B * max_pages + 3
    paged = lib.KVCache(O.FULL, B, kv_dtype=lib.KV_BF16, page_size=page, n_pages=n_pages,
                        block_table=_table(B, max_pages, n_pages, 111))
    raw, start = [], 0
    for i, T in enumerate((333, 190)):
        x = synth.prefill_inputs(B, T, seed=112 + i, device="cuda", start=start)
        out = lib.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], O.FULL, cache=paged)
        torch.cuda.synchronize()
        assert lib.hyb_device_error() == 0
        raw.append({k: f64(v) if k != "pos" else v.cpu().numpy() for k, v in x.items() if k != "qkv"})
        w = {k: np.concatenate([r[k] for r in raw], axis=1) for k in ("q", "k", "v", "gate", "pos")}
        ref = O.prefill(w["q"], w["k"], w["v"], w["gate"], w["pos"], O.FULL, rows=np.arange(start, start + T))
        got = f64(out)
        max_abs = float(np.abs(got - ref).max())
        rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
        assert max_abs <= 2e-2 and rel <= 5e-3, f"chunk {i}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"
        start += T
    xd = synth.decode_query(B, seed=115, device="cuda")
    lib.hyb_kv_append(paged, xd["k"], xd["v"])
    out = lib.hyb_attn_decode(xd["q"], xd["gate"], paged, max_len=paged.capacity)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    idx = np.arange(start + 1)
    keys = [O.rope_layer(np.concatenate([w["k"][b], f64(xd["k"])[b]]), idx, O.FULL) for b in range(B)]
    vals = [np.concatenate([w["v"][b], f64(xd["v"])[b]]) for b in range(B)]
    ref = O.decode(f64(xd["q"]), f64(xd["gate"]), [start] * B, keys, vals, [idx] * B, O.FULL)
    got = f64(out)
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert max_abs <= 2e-2 and rel <= 5e-3, f"decode: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"
