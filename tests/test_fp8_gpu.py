"""FP8 (e4m3) KV caches: the quantizing append against the oracle's
quantizer (values bit-exact, rotated keys within one code), and the calls
that do not support FP8 yet report it."""
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


def test_fp8_cache_rejected_by_prefill(lib):
    x = synth.prefill_inputs(1, 64, seed=1, device="cuda")
    cache = lib.KVCache(O.FULL, 1, capacity=128, kv_dtype=lib.KV_FP8)
    with pytest.raises(lib.HybError):
        lib.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], None, O.FULL, cache=cache)
