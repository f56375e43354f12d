"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's own formulas: each checks it against an
independent formulation (complex-number RoPE, scalar triple loops), a closed
form, an invariant, or a figure printed on the pages (tests/golden).
"""
import cmath
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_closed_forms.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16_like(rng, shape):
    """Values representable in bf16 (so the test inputs match what the GPU sees)."""
    x = rng.standard_normal(shape).astype(np.float32)
    u = x.view(np.uint32) & np.uint32(0xFFFF0000)
    return u.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Independent brute force: complex-number RoPE and scalar loops
# ---------------------------------------------------------------------------
def _rope_complex(vec, pos, theta, rdim):
    """Rotation written as z_k = x_k + i x_{k+R/2} times e^{i phi_k}."""
    out = list(vec)
    half = rdim // 2
    for k in range(half):
        phi = pos * theta ** (-2.0 * k / rdim)
        z = complex(vec[k], vec[k + half]) * cmath.exp(1j * phi)
        out[k], out[k + half] = z.real, z.imag
    return out


def _brute_attention(q, k, v, gate, pos, lt, start=0):
    """q [T,16,256], k/v [T,4,256] raw; plain loops, no matrices."""
    T = q.shape[0]
    theta, rdim = O.ROPE_THETA[lt], O.rotary_dim(lt)
    qr = [[_rope_complex(q[t, h], pos[t], theta, rdim) for h in range(16)] for t in range(T)]
    kr = [[_rope_complex(k[t, g], pos[t], theta, rdim) for g in range(4)] for t in range(T)]
    out = np.zeros((T, 16, 256))
    for t in range(T):
        for h in range(16):
            g = h // 4
            scores = []
            for j in range(T):
                ti, tj = start + t, start + j
                visible = tj <= ti and (lt == O.FULL or ti - tj <= 511)
                if visible:
                    dot = 0.0
                    for d in range(256):
                        dot += qr[t][h][d] * kr[j][g][d]
                    scores.append((j, dot / 16.0))
            mx = max(s for _, s in scores)
            w = [(j, math.exp(s - mx)) for j, s in scores]
            tot = sum(x for _, x in w)
            sg = 1.0 / (1.0 + math.exp(-gate[t, h]))
            for d in range(256):
                acc = 0.0
                for j, x in w:
                    acc += x * v[j, g, d]
                out[t, h, d] = acc / tot * sg
    return out


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
@pytest.mark.parametrize("start", [0, 1_000_000])
def test_brute_force_tiny(lt, start):
    rng = _rng(10 + lt)
    T = 4
    q = _bf16_like(rng, (1, T, 16, 256))
    k = _bf16_like(rng, (1, T, 4, 256))
    v = _bf16_like(rng, (1, T, 4, 256))
    gate = _bf16_like(rng, (1, T, 16))
    pos = np.arange(T)[None] + start
    got = O.prefill(q, k, v, gate, pos, lt, start=np.array([start]))[0]
    ref = _brute_attention(q[0], k[0], v[0], gate[0], pos[0], lt, start=start)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


def test_single_token_returns_gated_value():
    rng = _rng(1)
    q = _bf16_like(rng, (1, 1, 16, 256))
    k = _bf16_like(rng, (1, 1, 4, 256))
    v = _bf16_like(rng, (1, 1, 4, 256))
    gate = _bf16_like(rng, (1, 1, 16))
    for lt in (O.SLIDING, O.FULL):
        out = O.prefill(q, k, v, gate, np.array([[7]]), lt)[0, 0]
        for h in range(16):
            sg = 1.0 / (1.0 + math.exp(-gate[0, 0, h]))
            np.testing.assert_allclose(out[h], sg * v[0, 0, h // 4], rtol=0, atol=1e-14)


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_zero_query_averages_the_band(lt):
    """q = 0 gives equal scores: the output is the mean of v over the visible band."""
    rng = _rng(2)
    T = 700
    q = np.zeros((1, T, 16, 256))
    k = _bf16_like(rng, (1, T, 4, 256))
    v = _bf16_like(rng, (1, T, 4, 256))
    rows = np.array([0, 1, 510, 511, 512, 513, 699])
    out = O.prefill(q, k, v, None, np.arange(T)[None], lt, rows=rows)[0]
    for r_i, t in enumerate(rows):
        lo = max(0, t - 511) if lt == O.SLIDING else 0
        for h in (0, 5, 15):
            ref = v[0, lo:t + 1, h // 4].mean(axis=0)
            np.testing.assert_allclose(out[r_i, h], ref, rtol=0, atol=1e-12)


def test_sliding_equals_full_when_window_covers_sequence():
    rng = _rng(3)
    T = 300
    q = _bf16_like(rng, (T, 16, 256))
    k = _bf16_like(rng, (T, 4, 256))
    v = _bf16_like(rng, (T, 4, 256))
    idx = np.arange(T)
    a = O.gqa_attention(q, k, v, idx, idx, 512)
    b = O.gqa_attention(q, k, v, idx, idx, None)
    np.testing.assert_array_equal(a, b)
    # longer sequence: rows below 512 still agree, later ones differ
    T2 = 600
    q2 = _bf16_like(rng, (T2, 16, 256))
    k2 = _bf16_like(rng, (T2, 4, 256))
    v2 = _bf16_like(rng, (T2, 4, 256))
    i2 = np.arange(T2)
    a2 = O.gqa_attention(q2, k2, v2, i2, i2, 512)
    b2 = O.gqa_attention(q2, k2, v2, i2, i2, None)
    np.testing.assert_array_equal(a2[:512], b2[:512])
    assert np.abs(a2[512:] - b2[512:]).max() > 1e-3


def test_gqa_equals_mha_with_repeated_heads_and_grouping_is_contiguous():
    rng = _rng(4)
    T = 40
    q = _bf16_like(rng, (T, 16, 256))
    k = _bf16_like(rng, (T, 4, 256))
    v = _bf16_like(rng, (T, 4, 256))
    idx = np.arange(T)
    gqa = O.gqa_attention(q, k, v, idx, idx, None)
    # MHA written per head with an explicit index map, no repeat helper
    for h in range(16):
        qh = q[:, h:h + 1]
        kh = k[:, h // 4: h // 4 + 1]
        vh = v[:, h // 4: h // 4 + 1]
        mha = O.gqa_attention(qh, kh, vh, idx, idx, None)
        np.testing.assert_allclose(gqa[:, h], mha[:, 0], rtol=1e-13, atol=1e-14)
    # grouping: V of KV head g constant g + 1 -> query head h outputs h // 4 + 1
    vc = np.zeros((T, 4, 256))
    for g in range(4):
        vc[:, g, :] = g + 1
    out = O.gqa_attention(q, k, vc, idx, idx, None)
    for h in range(16):
        np.testing.assert_allclose(out[:, h], h // 4 + 1, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_rope_matches_complex_rotation(lt):
    rng = _rng(5)
    x = _bf16_like(rng, (3, 1, 256))
    pos = np.array([0, 17, 1_048_575])
    got = O.rope_layer(x, pos, lt)
    for t in range(3):
        ref = _rope_complex(list(x[t, 0]), int(pos[t]), O.ROPE_THETA[lt], O.rotary_dim(lt))
        # fp64 angles at pos ~2^20 carry pos * ulp(inv_freq) ~ 2e-10 rad of rounding
        np.testing.assert_allclose(got[t, 0], ref, rtol=0, atol=1e-9)


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_rope_norm_identity_and_passthrough(lt):
    rng = _rng(6)
    x = _bf16_like(rng, (64, 4, 256))
    pos = rng.integers(0, 1 << 20, size=64)
    y = O.rope_layer(x, pos, lt)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)
    z = O.rope_layer(x, np.zeros(64, dtype=np.int64), lt)
    np.testing.assert_array_equal(z, x)
    if lt == O.FULL:
        np.testing.assert_array_equal(y[..., 64:], x[..., 64:])
        assert np.abs(y[..., :64] - x[..., :64]).max() > 1e-3
    else:
        assert np.abs(y[..., 128:] - x[..., 128:]).max() > 1e-3


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_rope_scores_depend_only_on_offset(lt):
    rng = _rng(7)
    q = _bf16_like(rng, (1, 1, 256))
    k = _bf16_like(rng, (1, 1, 256))
    base = None
    for shift in (0, 1000, 900_000):
        qm = O.rope_layer(q, np.array([shift + 40]), lt)
        kn = O.rope_layer(k, np.array([shift + 3]), lt)
        s = float(np.sum(qm * kn))
        if base is None:
            base = s
        assert abs(s - base) < 1e-9 * max(1.0, abs(base))


def test_rope_frequencies_closed_form():
    """At position 1 the pair k rotates by theta^(-2k/R): check two pairs per type."""
    for lt, theta, rdim in ((O.SLIDING, 1e4, 256), (O.FULL, 5e6, 64)):
        for kk in (1, rdim // 2 - 1):
            x = np.zeros((1, 1, 256))
            x[0, 0, kk] = 1.0
            y = O.rope_layer(x, np.array([1]), lt)
            ang = math.atan2(y[0, 0, kk + rdim // 2], y[0, 0, kk])
            assert abs(ang - theta ** (-2.0 * kk / rdim)) < 1e-14


# ---------------------------------------------------------------------------
# Gate
# ---------------------------------------------------------------------------
def test_gate_zero_halves_and_saturates():
    rng = _rng(8)
    T = 9
    q = _bf16_like(rng, (1, T, 16, 256))
    k = _bf16_like(rng, (1, T, 4, 256))
    v = _bf16_like(rng, (1, T, 4, 256))
    pos = np.arange(T)[None]
    ungated = O.prefill(q, k, v, None, pos, O.FULL)
    half = O.prefill(q, k, v, np.zeros((1, T, 16)), pos, O.FULL)
    np.testing.assert_array_equal(half, 0.5 * ungated)
    hi = O.prefill(q, k, v, np.full((1, T, 16), 40.0), pos, O.FULL)
    lo = O.prefill(q, k, v, np.full((1, T, 16), -40.0), pos, O.FULL)
    np.testing.assert_allclose(hi, ungated, rtol=1e-15, atol=1e-15)
    assert np.abs(lo).max() < 1e-16


# ---------------------------------------------------------------------------
# Decode, chunking and caches
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_decode_equals_last_prefill_row(lt):
    rng = _rng(9)
    T = 530
    q = _bf16_like(rng, (1, T, 16, 256))
    k = _bf16_like(rng, (1, T, 4, 256))
    v = _bf16_like(rng, (1, T, 4, 256))
    gate = _bf16_like(rng, (1, T, 16))
    pos = np.arange(T)[None]
    ref = O.prefill(q, k, v, gate, pos, lt, rows=[T - 1])[0, 0]
    kc = O.rope_layer(k[0], pos[0], lt)
    got = O.decode(q[:, T - 1], gate[:, T - 1], [T - 1], [kc], [v[0]], [np.arange(T)], lt)[0]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_chunked_prefill_equals_one_shot(lt):
    rng = _rng(11)
    T, C = 900, 300
    q = _bf16_like(rng, (1, T, 16, 256))
    k = _bf16_like(rng, (1, T, 4, 256))
    v = _bf16_like(rng, (1, T, 4, 256))
    pos = np.arange(T)[None]
    ref = O.prefill(q, k, v, None, pos, lt)
    for c0 in (300, 600):
        hk = [O.rope_layer(k[0, :c0], pos[0, :c0], lt)]
        hv = [v[0, :c0]]
        got = O.prefill(q[:, c0:c0 + C], k[:, c0:c0 + C], v[:, c0:c0 + C], None,
                        pos[:, c0:c0 + C], lt, start=[c0], hist_k=hk, hist_v=hv,
                        hist_idx=[np.arange(c0)])
        np.testing.assert_allclose(got, ref[:, c0:c0 + C], rtol=1e-12, atol=1e-13)


def test_ring_keeps_last_512_and_slot_map():
    head0 = 77
    r = O.RingSim(head0)
    r.append(300)
    assert r.count == 300 and r.head == (77 + 300) % 512
    r.append(700)
    r.append(1)
    n = 1001
    assert r.count == 512 and r.length == n and r.head == (77 + n) % 512
    assert sorted(r.tag.tolist()) == list(range(n - 512, n))
    for i in range(n - 512, n):
        assert r.tag[(head0 + i) % 512] == i


# ---------------------------------------------------------------------------
# Closed forms printed on the pages (tests/golden/page_closed_forms.json)
# ---------------------------------------------------------------------------
def test_page_closed_forms():
    gold = json.load(open(GOLDEN))
    assert O.kv_bytes_per_token_layer() == gold["kv_bytes_per_token_layer"]["printed"]
    per = O.kv_bytes_per_token_layer()
    M1 = 1 << 20
    assert round(36 * per * M1 / 1e9, 1) == gold["kv_all_full_36_layers_1M_GB"]["printed"]
    assert round(36 * per * 32768 / 1e9, 1) == gold["kv_all_full_36_layers_32K_GB"]["printed"]
    assert round(O.kv_bytes(M1, 0, 28) / 1e6, 1) == gold["kv_sliding_28_layers_MB"]["printed"]
    assert round(O.kv_bytes(M1, 8, 0) / 1e9, 1) == gold["kv_full_8_layers_1M_GB"]["printed"]
    assert O.kv_bytes(M1, 0, 1) == 512 * 4096 == 2_097_152
    # the schedule the build uses: 9 full + 27 sliding, 38.65 GB + 56.6 MB at 1M
    assert round(O.kv_bytes(M1, 9, 0) / 1e9, 2) == 38.65
    assert round(O.kv_bytes(M1, 0, 27) / 1e6, 1) == 56.6
    # attention work, in the pages' units (layers x pairs, N^2 for full layers)
    assert round(8 * M1 ** 2 / 1e12, 1) == round(gold["work_full_8_layers_1M"]["printed"] / 1e12, 1)
    # 36 x (2^20)^2 = 3.958e13: the page truncates it to 3.9e13
    printed = gold["work_all_full_36_layers_1M"]["printed"]
    assert printed <= 36 * M1 ** 2 < printed + 0.1e13
    sl = 28 * M1 * 512
    assert round(sl / 1e10, 2) == round(gold["work_sliding_28_layers_1M"]["exact"] / 1e10, 2)
    assert 900 < gold["work_sliding_28_layers_1M"]["printed"] / sl < 1100  # the page's ~1000x slip


def test_layer_schedule():
    gold = json.load(open(GOLDEN))
    types = [O.layer_type(i) for i in range(36)]
    assert types.count(O.FULL) == gold["layer_counts"]["printed_full"]
    assert types.count(O.SLIDING) == gold["layer_counts"]["printed_sliding"]
    for i in gold["full_layer_indices"]["printed"]:
        assert types[i] == O.FULL
    assert types[:4] == [O.SLIDING, O.SLIDING, O.SLIDING, O.FULL]
    assert O.layer_type(36) == O.FULL
    assert O.rotary_dim(O.FULL) == 64 and O.rotary_dim(O.SLIDING) == 256


@pytest.mark.parametrize("n", [1, 5, 511, 512, 513, 1300])
def test_pair_counts_match_dense_mask(n):
    idx = np.arange(n)
    for lt in (O.SLIDING, O.FULL):
        assert O.attention_pairs(n, lt) == int(O.dense_mask(idx, idx, O.window_of(lt)).sum())
    assert O.prefill_flops(1024, O.FULL) == 524_800 * 16 * 1024
    assert O.attention_pairs(1024, O.SLIDING) == 393_472


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_decode_group_equals_gqa_attention(lt):
    """The per-group decode form agrees with the dense GQA definition (itself
    pinned by brute force above) on a history that crosses the window."""
    rng = np.random.default_rng(11)
    L = 700
    k = rng.standard_normal((L, O.N_KV_HEADS, O.HEAD_DIM))
    v = rng.standard_normal((L, O.N_KV_HEADS, O.HEAD_DIM))
    q = rng.standard_normal((1, O.N_Q_HEADS, O.HEAD_DIM))
    g = rng.standard_normal((1, O.N_Q_HEADS))
    idx = rng.permutation(L)            # any order of the history
    ref = O.gqa_attention(q, k, v, np.array([L - 1]), idx, O.window_of(lt), g)[0]
    for kvh in range(O.N_KV_HEADS):
        hs = slice(O.GROUP * kvh, O.GROUP * (kvh + 1))
        got = O.decode_group(q[0, hs], k[:, kvh], v[:, kvh], L - 1, idx, lt, g[0, hs])
        np.testing.assert_allclose(got, ref[hs], rtol=1e-12, atol=1e-12)


def test_linear_matches_scalar_loops():
    """y[m, n] = sum_k x[m, k] w[n, k], written as explicit loops."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 7))
    w = rng.standard_normal((5, 7))
    ref = np.zeros((3, 5))
    for m in range(3):
        for n in range(5):
            for k in range(7):
                ref[m, n] += x[m, k] * w[n, k]
    np.testing.assert_allclose(O.linear(x, w), ref, rtol=1e-13, atol=1e-13)


def test_attention_layer_slices_q_k_v_from_the_fused_projection():
    """With one-hot hidden states, column t of W_qkv is token t's fused
    q | k | v row and column t of W_g its gate scores, so the layer must equal
    the attention of exactly those q, k, v, g, followed by o_proj.  A swapped
    slice or a missing transpose fails."""
    rng = np.random.default_rng(9)
    B, T, Hd = 1, 6, 2560
    hidden = np.zeros((B, T, Hd))
    hidden[0, np.arange(T), np.arange(T)] = 1.0
    q = O.to_bf16(rng.standard_normal((B, T, 16, 256)))
    k = O.to_bf16(rng.standard_normal((B, T, 4, 256)))
    v = O.to_bf16(rng.standard_normal((B, T, 4, 256)))
    g = O.to_bf16(rng.standard_normal((B, T, 16)))
    w_qkv = np.zeros((6144, Hd))
    w_qkv[:, :T] = np.concatenate([q[0].reshape(T, -1), k[0].reshape(T, -1), v[0].reshape(T, -1)], axis=1).T
    w_gate = np.zeros((16, Hd))
    w_gate[:, :T] = g[0].T
    w_o = rng.standard_normal((Hd, 4096)) / 64.0
    pos = np.arange(T)[None]
    for lt in (O.SLIDING, O.FULL):
        got = O.attention_layer(hidden, w_qkv, w_gate, w_o, pos, lt)
        att = O.to_bf16(O.prefill(q, k, v, g, pos, lt)).reshape(B, T, 4096)
        np.testing.assert_allclose(got, att @ w_o.T, rtol=1e-12, atol=1e-12)


def test_to_bf16_rounds_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, 1.0 + 2 ** -9, -2.5, 3.0e38])
    got = O.to_bf16(x)
    # bf16 keeps 8 significant bits: ulp(1) = 2^-7; halfway cases go to even
    np.testing.assert_array_equal(got[:5], [1.0, 1.0, 1.0 + 2 ** -7, 1.0, -2.5])
    assert np.isfinite(got[5]) and abs(got[5] / 3.0e38 - 1) < 2 ** -8


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_layer_decode_equals_last_row_of_layer_prefill(lt):
    """Decoding the last token of a sequence through the layer, with the other
    tokens' projected K/V as history, gives the layer prefill's last row."""
    rng = np.random.default_rng(12)
    T, Hd = 7, 2560
    hidden = O.to_bf16(rng.standard_normal((1, T, Hd)))
    w_qkv = O.to_bf16(rng.standard_normal((6144, Hd)) / np.sqrt(Hd))
    w_gate = O.to_bf16(rng.standard_normal((16, Hd)) / np.sqrt(Hd))
    w_o = O.to_bf16(rng.standard_normal((Hd, 4096)) / 64.0)
    pos = np.arange(T)[None]
    full = O.attention_layer(hidden, w_qkv, w_gate, w_o, pos, lt)
    qkv = O.to_bf16(hidden[0, :T - 1] @ w_qkv.T)
    hk = O.rope_layer(qkv[:, 4096:5120].reshape(T - 1, 4, 256), np.arange(T - 1), lt)
    hv = qkv[:, 5120:].reshape(T - 1, 4, 256)
    got = O.attention_layer_decode(hidden[:, T - 1], w_qkv, w_gate, w_o, [T - 1], [hk], [hv], [np.arange(T - 1)], lt)
    np.testing.assert_allclose(got[0], full[0, T - 1], rtol=1e-10, atol=1e-12)


def test_e4m3_quantizer_known_values_and_bounds():
    """e4m3: 1 sign, 4 exponent (bias 7), 3 mantissa bits, max 448, smallest
    subnormal 2^-9; round to nearest even; saturating at +-448."""
    # a row whose amax is 448 keeps representable values exactly (scale 1)
    row = np.zeros(256)
    row[:8] = [448.0, -448.0, 1.0, 1.125, 0.015625, 2 ** -9, -3.25, 0.0]
    codes, scale = O.quantize_e4m3_rows(row)
    assert scale == np.float32(1.0)
    # bit patterns: 448 = 0 1111 110; 1.0 = 0 0111 000; 1.125 = 0 0111 001;
    # 2^-6 = 0 0001 000; 2^-9 = 0 0000 001 (subnormal); -3.25 = 1 1000 101
    assert codes[:8].tolist() == [0x7E, 0xFE, 0x38, 0x39, 0x08, 0x01, 0xC5, 0x00]
    np.testing.assert_array_equal(O.dequantize_e4m3_rows(codes, scale)[:8], row[:8])
    # halfway cases go to even: 1.0625 lies between 1.0 (even code) and 1.125
    c2, _ = O.quantize_e4m3_rows(np.concatenate([[448.0, 1.0625, 1.1875], np.zeros(253)]))
    assert c2[1] == 0x38 and c2[2] == 0x3A
    # random rows: relative error of normal values <= 2^-4 (half of a 3-bit ulp); amax exact
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 256)) * rng.uniform(0.01, 100, size=(64, 1))
    c, s = O.quantize_e4m3_rows(x)
    d = O.dequantize_e4m3_rows(c, s)
    x32 = x.astype(np.float32).astype(np.float64)
    normal = np.abs(x32) >= (2 ** -6) * (np.abs(x32).max(-1, keepdims=True) / 448)
    assert np.all(np.abs(d - x32)[normal] <= 2 ** -4 * np.abs(x32)[normal] * (1 + 1e-6))
    np.testing.assert_allclose(np.abs(d).max(-1), np.abs(x32).max(-1), rtol=1e-6)
    # a zero row: scale 0, codes 0
    cz, sz = O.quantize_e4m3_rows(np.zeros(256))
    assert sz == 0 and not cz.any()


def test_decode_partial_brute_force_tiny():
    """lse2 and o of one part written out as scalar loops (position 0: no rotation)."""
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 16, 256))
    k = rng.standard_normal((1, 3, 4, 256))
    v = rng.standard_normal((1, 3, 4, 256))
    o, lse2 = O.decode_partial(q, [0], list(k), list(v), O.FULL)
    for h in (0, 5, 15):
        kv = h // 4
        s = [sum(q[0, h, d] * k[0, j, kv, d] for d in range(256)) / 16.0 for j in range(3)]
        z = sum(math.exp(x) for x in s)
        assert abs(lse2[0, h] - math.log2(z)) < 1e-12
        for d in (0, 77, 255):
            ref = sum(math.exp(s[j]) * v[0, j, kv, d] for j in range(3)) / z
            assert abs(o[0, h, d] - ref) < 1e-12


def test_merged_parts_equal_decode_over_the_union():
    """Spreading a full-layer history over parts (one of them empty, keys in
    any order) and merging gives decode over all keys, gate included."""
    rng = np.random.default_rng(6)
    B, L = 2, 90
    q = rng.standard_normal((B, 16, 256))
    gate = rng.standard_normal((B, 16))
    k = rng.standard_normal((B, L, 4, 256))
    v = rng.standard_normal((B, L, 4, 256))
    qpos = [L - 1, L - 1]
    owner = rng.integers(0, 3, size=L)
    owner[owner == 2] = 0                   # part 2 holds nothing
    parts = [O.decode_partial(q, qpos, [k[b][owner == p] for b in range(B)], [v[b][owner == p] for b in range(B)],
                              O.FULL) for p in range(3)]
    assert np.all(parts[2][1] == -np.inf) and np.all(parts[2][0] == 0)
    got = O.merge_partials(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]), gate)
    ref = O.decode(q, gate, qpos, list(k), list(v), [np.arange(L)] * B, O.FULL)
    assert np.abs(got - ref).max() < 1e-12
    # a single part is decode without the gate, and its merge adds the gate
    o1, l1 = O.decode_partial(q, qpos, list(k), list(v), O.FULL)
    assert np.abs(o1 - O.decode(q, None, qpos, list(k), list(v), [np.arange(L)] * B, O.FULL)).max() < 1e-12
    assert np.abs(O.merge_partials(o1[None], l1[None], gate) - ref).max() < 1e-12


# ---------------------------------------------------------------------------
# Randomised identities (hypothesis): shapes, positions and partitions drawn
# at random, each checked against a relation the definition implies.
# ---------------------------------------------------------------------------
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(lt=st.sampled_from([O.FULL, O.SLIDING]), p=st.integers(0, 1 << 20), shift=st.integers(-5000, 5000),
       seed=st.integers(0, 2 ** 31 - 1))
def test_rope_scores_depend_only_on_the_offset(lt, p, shift, seed):
    """q(m) . k(n) after rotation depends on m - n only, at any positions."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 1, 256))
    k = rng.standard_normal((1, 1, 256))
    n = max(0, p - 777)
    a = (O.rope_layer(q, np.array([p]), lt) * O.rope_layer(k, np.array([n]), lt)).sum()
    p2, n2 = max(0, p + shift), max(0, n + shift)
    if p2 - n2 != p - n:
        return
    b = (O.rope_layer(q, np.array([p2]), lt) * O.rope_layer(k, np.array([n2]), lt)).sum()
    assert abs(a - b) <= 1e-9 * (1 + abs(a))


@settings(max_examples=20, deadline=None)
@given(L=st.integers(1, 60), n_parts=st.integers(1, 4), seed=st.integers(0, 2 ** 31 - 1))
def test_any_partition_of_the_history_merges_to_decode(L, n_parts, seed):
    """The log-sum-exp merge of the parts of any partition equals decode."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, 16, 256))
    gate = rng.standard_normal((1, 16))
    k = rng.standard_normal((1, L, 4, 256))
    v = rng.standard_normal((1, L, 4, 256))
    owner = rng.integers(0, n_parts, size=L)
    parts = [O.decode_partial(q, [L - 1], [k[0][owner == p]], [v[0][owner == p]], O.FULL) for p in range(n_parts)]
    got = O.merge_partials(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]), gate)
    ref = O.decode(q, gate, [L - 1], [k[0]], [v[0]], [np.arange(L)], O.FULL)
    assert np.abs(got - ref).max() < 1e-12


@settings(max_examples=20, deadline=None)
@given(codes=st.lists(st.integers(0, 255).filter(lambda c: c & 0x7F != 0x7F), min_size=256, max_size=256),
       scale=st.floats(1e-6, 1e6))
def test_e4m3_requantizing_a_dequantized_row_is_identity(codes, scale):
    """quantize(dequantize(codes, s)) gives the codes back (up to the sign of
    zero) when the row's largest code is 448: the scale is recovered (to the
    fp32 rounding of 448 s) and every value is on the e4m3 grid."""
    c = np.array(codes, dtype=np.uint8).reshape(1, 256)
    c[0, 0] = 0x7E                                  # +448 sets amax
    vals = O.dequantize_e4m3_rows(c, np.array([scale], dtype=np.float32))
    c2, s2 = O.quantize_e4m3_rows(vals)
    s32 = float(np.float32(scale))
    assert abs(float(s2[0]) - s32) <= 2.0 ** -22 * s32
    zero = (c & 0x7F) == 0
    assert np.array_equal(c2[~zero], c[~zero])
    assert np.all((c2[zero] & 0x7F) == 0)
