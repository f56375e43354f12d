"""FP8 (e4m3) KV caches: the quantizing append against the oracle's
quantizer (values bit-exact, rotated keys within one code), decode over
every code and scale range, and chunked prefill over the stored history,
all against the oracle on the dequantized cache."""
import numpy as np
import pytest
import torch

import oracle as O
from full_gqa_attention_partial_b200 import synth

pytestmark = pytest.mark.gpu


def f64(t):
    return t.detach().float().cpu().double().numpy()


def _check_rows(lib, cache, x, lt, slots, tokens):
    """Rows `tokens` of the appended batch 0 sit at cache slots `slots`."""
    kc = cache.k[0].cpu().numpy()[:, slots]            # [4, n, 256] codes
    vc = cache.v[0].cpu().numpy()[:, slots]
    ks = cache.k_scale[0].cpu().numpy()[:, slots]      # [4, n]
    vs = cache.v_scale[0].cpu().numpy()[:, slots]
    v_raw = f64(x["v"][0, tokens]).transpose(1, 0, 2)   # [4, n, 256]
    codes, scale = O.quantize_e4m3_rows(v_raw)
    np.testing.assert_array_equal(vc, codes)
    np.testing.assert_array_equal(vs, scale)
    # keys: rotated (fp64), rounded to bf16 as the bf16 cache would hold them, then quantized
    pos = x["pos"][0, tokens].cpu().numpy()
    k_rot = O.to_bf16(O.rope_layer(f64(x["k"][0, tokens])[None], pos[None], lt)[0]).transpose(1, 0, 2)
    kcodes, kscale = O.quantize_e4m3_rows(k_rot)
    np.testing.assert_allclose(ks, kscale, rtol=1e-2)
    assert np.mean(kc == kcodes) > 0.99
    got = O.dequantize_e4m3_rows(kc, ks)
    ref = O.dequantize_e4m3_rows(kcodes, kscale)
    # at most one e4m3 step apart: 2^-3 of the value's binade, below 2^-9 * 448 * scale near zero
    tol = np.maximum(np.abs(ref) * 2 ** -3, kscale[..., None] * 2 ** -9 * 2) * 1.01
    assert np.all(np.abs(got - ref) <= tol)


@pytest.mark.parametrize("lt", [O.FULL, O.SLIDING])
def test_fp8_append_matches_quantizer(lib, lt):
    T = 300 if lt == O.FULL else 700
    x = synth.prefill_inputs(1, T, seed=31 + lt, device="cuda", start=0)
    r = synth.ring_offset(31)
    cache = lib.KVCache(lt, 1, capacity=1024, kv_dtype=lib.KV_FP8, head0=None if lt == O.FULL else [r])
    lib.hyb_kv_append(cache, x["k"], x["v"], pos=x["pos"])
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    assert cache.len.tolist() == [T]
    if lt == O.FULL:
        tokens = np.arange(T)
        slots = tokens
    else:
        tokens = np.arange(T - 512, T)
        slots = (r + tokens) % 512
        assert (cache.tag[0].cpu().numpy()[slots] == tokens).all()
    _check_rows(lib, cache, x, lt, slots, tokens)


def as_stored(k_raw, v_raw, pos, lt):
    """A chunk's keys and values as an FP8 cache stores them ([T, 4, 256]
    each): keys rotated, rounded to bf16 and quantized, values quantized; both
    dequantized, all by the oracle."""
    k_rot = O.to_bf16(O.rope_layer(k_raw, pos, lt))
    return (O.dequantize_e4m3_rows(*O.quantize_e4m3_rows(k_rot)),
            O.dequantize_e4m3_rows(*O.quantize_e4m3_rows(v_raw)))


def attend(x, lt, b, start, hist_k=None, hist_v=None, hist_idx=None):
    """The oracle's attention of chunk x's queries (sequence b, token 0 at
    sequence index `start`) over an optional stored history and the chunk's
    own tokens as stored."""
    q, k, v, g, pos = (f64(x["q"][b]), f64(x["k"][b]), f64(x["v"][b]), f64(x["gate"][b]), x["pos"][b].cpu().numpy())
    T = q.shape[0]
    kc, vc = as_stored(k, v, pos, lt)
    idx = start + np.arange(T)
    if hist_k is not None:
        kc, vc, kidx = np.concatenate([hist_k, kc]), np.concatenate([hist_v, vc]), np.concatenate([hist_idx, idx])
    else:
        kidx = idx
    return O.gqa_attention(O.rope_layer(q, pos, lt), kc, vc, idx, kidx, O.window_of(lt), g)


@pytest.mark.parametrize("lt", [O.FULL, O.SLIDING])
def test_fp8_chunked_prefill_matches_oracle(lib, lt):
    """Two prefill chunks through an FP8 cache: each chunk is appended
    quantized and attends to the cached history and to its own tokens as the
    cache stores them (the oracle quantizes the chunk itself and dequantizes
    the history's codes)."""
    B, T1, T2 = 2, 700, 300
    r = synth.ring_offset(51)
    cache = lib.KVCache(lt, B, capacity=1024, kv_dtype=lib.KV_FP8, head0=None if lt == O.FULL else [r, (r + 99) % 512])
    x1 = synth.prefill_inputs(B, T1, seed=52, device="cuda")
    out1 = lib.hyb_attn_prefill(x1["q"], x1["k"], x1["v"], x1["gate"], x1["pos"], lt, cache=cache)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    ref1 = np.stack([attend(x1, lt, b, 0) for b in range(B)])
    assert_close(out1, ref1, f"chunk 1 lt={lt}")
    # the history chunk 2 sees, as stored
    if lt == O.FULL:
        rows = [np.arange(T1)] * B
        idx = rows
    else:
        tag = cache.tag.cpu().numpy()
        rows = [np.nonzero(tag[b] >= 0)[0] for b in range(B)]
        idx = [tag[b][rows[b]] for b in range(B)]
    hk, hv = [], []
    for b in range(B):
        kc = cache.k[b][:, rows[b]].cpu().numpy()
        vc = cache.v[b][:, rows[b]].cpu().numpy()
        ks = cache.k_scale[b][:, rows[b]].cpu().numpy()
        vs = cache.v_scale[b][:, rows[b]].cpu().numpy()
        hk.append(O.dequantize_e4m3_rows(kc, ks).transpose(1, 0, 2))
        hv.append(O.dequantize_e4m3_rows(vc, vs).transpose(1, 0, 2))
    x2 = synth.prefill_inputs(B, T2, seed=53, device="cuda", start=T1)
    out2 = lib.hyb_attn_prefill(x2["q"], x2["k"], x2["v"], x2["gate"], x2["pos"], lt, cache=cache)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    assert cache.len.tolist() == [T1 + T2] * B
    ref2 = np.stack([attend(x2, lt, b, T1, hk[b], hv[b], idx[b]) for b in range(B)])
    assert_close(out2, ref2, f"chunk 2 lt={lt}")


def test_fp8_prefill_workspace_does_not_grow_with_capacity(lib):
    """A full-layer FP8 cache is read in place: the prefill workspace is the
    bf16 cache's (none), whatever the capacity."""
    for cap in (1024, 1 << 20):
        for kvd in (lib.KV_BF16, lib.KV_FP8):
            c = lib.KVCache(O.FULL, 1, capacity=cap, kv_dtype=kvd)
            assert lib.hyb_attn_prefill_cache_workspace_size(c, 8192) == 0
            del c
            torch.cuda.empty_cache()


def assert_close(got, ref, what):
    got = f64(got)
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert max_abs <= 2e-2 and rel <= 5e-3, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


def _fp8_full(lib, B, L, cap, seed):
    c = lib.KVCache(O.FULL, B, capacity=cap, kv_dtype=lib.KV_FP8)
    synth.fill_cache_fp8_(c.k, c.v, c.k_scale, c.v_scale, L, seed)
    c.len.fill_(L)
    return c


def _fp8_ring(lib, B, L, seed, head0):
    c = lib.KVCache(O.SLIDING, B, kv_dtype=lib.KV_FP8, head0=[head0] * B)
    synth.fill_cache_fp8_(c.k, c.v, c.k_scale, c.v_scale, 512, seed)
    idx = torch.arange(L - 512, L, dtype=torch.int64, device="cuda")
    tag = torch.full((512,), -1, dtype=torch.int32, device="cuda")
    tag[(head0 + idx) % 512] = idx.to(torch.int32)
    c.tag.copy_(tag.expand(B, 512))
    c.len.fill_(L)
    c.head.fill_((head0 + L) % 512)
    return c


def _snapshot(c, rows):
    """Host copy of the seeded history rows [B][n, 4, 256] (dequantized by the oracle)."""
    kc = c.k[:, :, rows].cpu().numpy()
    vc = c.v[:, :, rows].cpu().numpy()
    ks = c.k_scale[:, :, rows].cpu().numpy()
    vs = c.v_scale[:, :, rows].cpu().numpy()
    return (O.dequantize_e4m3_rows(kc, ks).transpose(0, 2, 1, 3), O.dequantize_e4m3_rows(vc, vs).transpose(0, 2, 1, 3))


@pytest.mark.parametrize("lt", [O.FULL, O.SLIDING])
@pytest.mark.parametrize("noalloc", [False, True])
def test_fp8_decode_matches_oracle_on_dequantized_cache(lib, lt, noalloc):
    """Decode over an FP8 cache equals the attention of the dequantized keys
    and values: the seeded history (snapshot before any library call) plus
    the new token, which the oracle rotates, rounds to bf16 and quantizes."""
    B = 4
    L = 3000 if lt == O.FULL else 1200
    if lt == O.FULL:
        cap = L + 4
        c = _fp8_full(lib, B, L, cap, seed=41)
        hk, hv = _snapshot(c, np.arange(L))
        hidx = np.arange(L)
        max_len = cap
    else:
        r = synth.ring_offset(42)
        c = _fp8_ring(lib, B, L, seed=43, head0=r)
        hidx = np.arange(L - 511, L)                     # the window after one more token
        hk, hv = _snapshot(c, (r + hidx) % 512)
        max_len = 512
    x = synth.decode_query(B, seed=44 + lt, device="cuda")
    lib.hyb_kv_append(c, x["k"], x["v"])
    if noalloc:
        out = lib.hyb_attn_decode_noalloc(x["q"], x["gate"], c, max_len=max_len)
    else:
        out = lib.hyb_attn_decode(x["q"], x["gate"], c, max_len=max_len)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    n = L + 1
    k_rot = O.to_bf16(O.rope_layer(f64(x["k"]), np.full((B, 1), n - 1), lt)[:, 0])      # [B, 4, 256]
    kq, ksc = O.quantize_e4m3_rows(k_rot)
    vq, vsc = O.quantize_e4m3_rows(f64(x["v"])[:, 0])
    kn, vn = O.dequantize_e4m3_rows(kq, ksc), O.dequantize_e4m3_rows(vq, vsc)
    keys = [np.concatenate([hk[b], kn[b][None]]) for b in range(B)]
    vals = [np.concatenate([hv[b], vn[b][None]]) for b in range(B)]
    idx = [np.append(hidx, n - 1)] * B
    ref = O.decode(f64(x["q"]), f64(x["gate"]), [n - 1] * B, keys, vals, idx, lt)
    got = f64(out)
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert max_abs <= 2e-2 and rel <= 5e-3, f"max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


_FINITE = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)   # every non-NaN code
_SUBNORMAL = np.array([c for c in range(256) if c & 0x78 == 0], dtype=np.uint8)   # exponent field 0


@pytest.mark.parametrize("case", ["every_code", "subnormal_only"])
def test_fp8_decode_code_coverage(lib, case):
    """Decode reads every finite e4m3 code, subnormals included, at row
    scales from 1e-3 to 1e3 (values past 1e5): the widening keeps each code's
    value and the scales reach the output without leaving the fp32 or bf16
    range."""
    B, L = 2, 700
    cap = L + 4
    rng = np.random.default_rng(7 if case == "every_code" else 8)
    pool = _FINITE if case == "every_code" else _SUBNORMAL
    c = lib.KVCache(O.FULL, B, capacity=cap, kv_dtype=lib.KV_FP8)
    kc = rng.choice(pool, size=(B, 4, L, 256))
    vc = rng.choice(pool, size=(B, 4, L, 256))
    if case == "every_code":
        ks = np.full((B, 4, L), 3e-3, np.float32)                        # key values up to 1.3
        vs = (10.0 ** rng.uniform(-3, 3, size=(B, 4, L))).astype(np.float32)
    else:
        ks = np.full((B, 4, L), 100.0, np.float32)                       # subnormal codes are <= 7/512
        vs = (10.0 ** rng.uniform(-1, 1, size=(B, 4, L))).astype(np.float32)
    c.k[:, :, :L].copy_(torch.from_numpy(kc))
    c.v[:, :, :L].copy_(torch.from_numpy(vc))
    c.k_scale[:, :, :L].copy_(torch.from_numpy(ks))
    c.v_scale[:, :, :L].copy_(torch.from_numpy(vs))
    c.len.fill_(L)
    x = synth.decode_query(B, seed=45, device="cuda")
    lib.hyb_kv_append(c, x["k"], x["v"])
    out = lib.hyb_attn_decode(x["q"], x["gate"], c, max_len=cap)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    hk, hv = _snapshot(c, np.arange(L + 1))            # history and the appended row, as stored
    idx = [np.arange(L + 1)] * B
    ref = O.decode(f64(x["q"]), f64(x["gate"]), [L] * B, list(hk), list(hv), idx, O.FULL)
    got = f64(out)
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert np.isfinite(got).all()
    assert rel <= 5e-3, f"rel_l2 {rel:.3e}"
