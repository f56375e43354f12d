"""A whole attention layer (q_k_v_proj + gate projection -> attention core ->
o_proj) against the oracle's attention_layer, which rounds the three
intermediate tensors to bf16 as the model does; synthetic weights
N(0, 1/fan_in), hidden states N(0, 1)."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


def f64(t):
    return t.detach().float().cpu().double().numpy()


def weights(seed, gate=True):
    g = torch.Generator(device="cuda").manual_seed(seed)
    w_qkv = (torch.randn(6144, 2560, generator=g, device="cuda") / 2560 ** 0.5).to(torch.bfloat16)
    w_gate = (torch.randn(16, 2560, generator=g, device="cuda") / 2560 ** 0.5).to(torch.bfloat16) if gate else None
    w_o = (torch.randn(2560, 4096, generator=g, device="cuda") / 4096 ** 0.5).to(torch.bfloat16)
    return w_qkv, w_gate, w_o


def hidden_states(B, T, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn(B, T, 2560, generator=g, device="cuda").to(torch.bfloat16)


def check(got, ref, what):
    got = f64(got)
    assert np.all(np.isfinite(got)), what
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


def oracle(h, w_qkv, w_gate, w_o, pos, lt, rows=None):
    return O.attention_layer(f64(h), f64(w_qkv), None if w_gate is None else f64(w_gate), f64(w_o),
                             pos.cpu().numpy(), lt, rows=rows)


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
@pytest.mark.parametrize("gate", [True, False])
def test_layer_prefill_small(lib, lt, gate):
    B, T = 2, 300
    h = hidden_states(B, T, seed=1 + lt)
    w_qkv, w_gate, w_o = weights(10 + lt, gate)
    pos = torch.arange(T, dtype=torch.int32, device="cuda").repeat(B, 1).contiguous()
    out = lib.hyb_attn_layer_prefill(h, w_qkv, w_gate, w_o, pos, lt)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    check(out, oracle(h, w_qkv, w_gate, w_o, pos, lt), f"layer B={B} T={T} type {lt} gate {gate}")


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_layer_prefill_into_cache_then_chunk(lib, lt):
    """Two chunks through a cache: the second chunk's rows see the first's keys."""
    T1, T2 = 700, 260
    h = hidden_states(1, T1 + T2, seed=5 + lt)
    w_qkv, w_gate, w_o = weights(20 + lt)
    cache = lib.KVCache(lt, 1, capacity=T1 + T2) if lt == O.FULL else lib.KVCache(lt, 1)
    pos = torch.arange(T1 + T2, dtype=torch.int32, device="cuda")[None].contiguous()
    out1 = lib.hyb_attn_layer_prefill(h[:, :T1].contiguous(), w_qkv, w_gate, w_o, pos[:, :T1].contiguous(), lt,
                                      cache=cache)
    out2 = lib.hyb_attn_layer_prefill(h[:, T1:].contiguous(), w_qkv, w_gate, w_o, pos[:, T1:].contiguous(), lt,
                                      cache=cache)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    ref = oracle(h, w_qkv, w_gate, w_o, pos, lt)      # one shot over both chunks
    check(out1, ref[:, :T1], f"layer chunk 1 type {lt}")
    check(out2, ref[:, T1:], f"layer chunk 2 type {lt}")


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_layer_prefill_T8192_sampled(lib, lt):
    T = 8192
    h = hidden_states(1, T, seed=30 + lt)
    w_qkv, w_gate, w_o = weights(40 + lt)
    pos = torch.arange(T, dtype=torch.int32, device="cuda")[None].contiguous()
    out = lib.hyb_attn_layer_prefill(h, w_qkv, w_gate, w_o, pos, lt)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    rng = np.random.default_rng(lt)
    rows = np.unique(np.concatenate([np.arange(0, 140), np.arange(T - 140, T), rng.choice(T, 200, replace=False)]))
    check(out[:, rows], oracle(h, w_qkv, w_gate, w_o, pos, lt, rows=rows), f"layer T={T} type {lt}")


def test_layer_rejects_bad_weight_shape(lib):
    h = hidden_states(1, 8, seed=0)
    w_qkv, w_gate, w_o = weights(0)
    with pytest.raises(ValueError):
        lib.hyb_attn_layer_prefill(h, w_qkv[:, :2048].contiguous(), w_gate, w_o, None, O.FULL)


@pytest.mark.parametrize("B", [3, 20])
@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_layer_decode_steps(lib, lt, B):
    """Three decode steps of the layer over a seeded cache (history snapshot
    taken before any library call on it; the oracle projects and rotates the
    new tokens itself).  Up to 16 sequences the projections run on the
    few-row kernel and the append / decode rotate k and q; 20 sequences take
    the tiled GEMM with RoPE in its epilogue."""
    import bench
    from full_gqa_attention_partial_b200 import synth
    L, n_steps = 1500, 3
    w_qkv, w_gate, w_o = weights(50 + lt)
    if lt == O.FULL:
        cap = L + n_steps
        cache = bench.fill_full_cache(lib, B, L, cap, seed=8)
        hist = [(f64(cache.k[b, :, :L]).transpose(1, 0, 2), f64(cache.v[b, :, :L]).transpose(1, 0, 2),
                 np.arange(L)) for b in range(B)]
        max_len = cap
    else:
        r = synth.ring_offset(9)
        cache = bench.fill_ring_cache(lib, B, L, seed=10, head0=r)
        idx = np.arange(L - O.WINDOW, L)
        rk, rv = f64(cache.k), f64(cache.v)           # [B, 4, 512, 256], slot-indexed
        hist = [(rk[b][:, (r + idx) % O.WINDOW].transpose(1, 0, 2), rv[b][:, (r + idx) % O.WINDOW].transpose(1, 0, 2),
                 idx) for b in range(B)]
        max_len = O.WINDOW
    for step in range(n_steps):
        h = hidden_states(1, B, seed=60 + step)[0]    # [B, 2560]
        out = lib.hyb_attn_layer_decode(h, w_qkv, w_gate, w_o, cache, max_len=max_len)
        torch.cuda.synchronize()
        assert lib.hyb_device_error() == 0
        n = L + step                                  # sequence index of the new token
        ref = O.attention_layer_decode(f64(h), f64(w_qkv), f64(w_gate), f64(w_o), [n] * B,
                                       [x[0] for x in hist], [x[1] for x in hist], [x[2] for x in hist], lt)
        check(out, ref, f"layer decode step {step} type {lt}")
        # the oracle's history grows by the token it just computed
        hf = f64(h)
        qkv = O.to_bf16(O.linear(hf, f64(w_qkv)))
        kn = O.rope_layer(qkv[:, 4096:5120].reshape(B, 1, 4, 256), np.full((B, 1), n), lt)[:, 0]
        vn = qkv[:, 5120:].reshape(B, 4, 256)
        new_hist = []
        for b in range(B):
            k_b = np.concatenate([hist[b][0], kn[b][None]])
            v_b = np.concatenate([hist[b][1], vn[b][None]])
            i_b = np.append(hist[b][2], n)
            if lt == O.SLIDING:                       # the window keeps the last 512
                k_b, v_b, i_b = k_b[-O.WINDOW:], v_b[-O.WINDOW:], i_b[-O.WINDOW:]
            new_hist.append((k_b, v_b, i_b))
        hist = new_hist
