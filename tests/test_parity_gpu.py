"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Acceptance (bf16 in, fp32 accumulate): max-abs error <= 2e-2 and relative L2
error <= 5e-3 on the attention outputs; cache slot mapping, tags, lengths and
copied values bit-exact; rotated keys within one bf16 ulp of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
from full_gqa_attention_partial_b200 import synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


def f64(t):
    return t.detach().float().cpu().double().numpy()


def assert_close(got, ref, what=""):
    got = f64(got) if isinstance(got, torch.Tensor) else got
    d = np.abs(got - ref)
    max_abs = float(d.max())
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"
    return max_abs, rel


def to_dev(inp):
    """Moves a prefill batch to the GPU keeping q/k/v as views into the fused qkv rows."""
    qkv = inp["qkv"].cuda()
    return {
        "qkv": qkv,
        "q": qkv[..., :4096].unflatten(-1, (16, 256)),
        "k": qkv[..., 4096:5120].unflatten(-1, (4, 256)),
        "v": qkv[..., 5120:].unflatten(-1, (4, 256)),
        "gate": inp["gate"].cuda(),
        "pos": inp["pos"].cuda(),
    }


def run_prefill(lib, inp, lt, fused=True, with_gate=True, with_pos=True):
    d = to_dev(inp)
    if fused:
        q, k, v = d["q"], d["k"], d["v"]
        assert q.stride(1) == 6144 and k.stride(1) == 6144
    else:
        q, k, v = d["q"].contiguous(), d["k"].contiguous(), d["v"].contiguous()
    out = lib.hyb_attn_prefill(q, k, v, d["gate"] if with_gate else None, d["pos"] if with_pos else None, lt)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    return out


def oracle_prefill(inp, lt, rows=None, with_gate=True):
    return O.prefill(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]),
                     f64(inp["gate"]) if with_gate else None, inp["pos"].numpy(), lt, rows=rows)


# ---------------------------------------------------------------------------
# Prefill without a cache
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_prefill_seq1024_one_layer_each(lib, lt):
    """One sliding and one full layer, B=1, T=1024, N(0,1) inputs, seed 0."""
    inp = synth.prefill_inputs(1, 1024, seed=0)
    out = run_prefill(lib, inp, lt)
    assert_close(out, oracle_prefill(inp, lt), f"T=1024 lt={lt}")


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
@pytest.mark.parametrize("B,T", [(1, 1), (1, 5), (2, 64), (1, 130), (3, 700), (1, 1000)])
def test_prefill_ragged_shapes(lib, lt, B, T):
    inp = synth.prefill_inputs(B, T, seed=100 + T)
    out = run_prefill(lib, inp, lt, fused=(T % 2 == 0))
    assert_close(out, oracle_prefill(inp, lt), f"B={B} T={T} lt={lt}")


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_prefill_no_gate_and_default_positions(lib, lt):
    inp = synth.prefill_inputs(2, 300, seed=7)
    out = run_prefill(lib, inp, lt, with_gate=False, with_pos=False)
    assert_close(out, oracle_prefill(inp, lt, with_gate=False), "no gate")


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_prefill_large_positions(lib, lt):
    """RoPE angles at positions near 2^20 (max_position_embeddings)."""
    inp = synth.prefill_inputs(1, 257, seed=8, start=(1 << 20) - 257)
    out = run_prefill(lib, inp, lt)
    assert_close(out, oracle_prefill(inp, lt), "large positions")


def test_prefill_gate_zero_halves(lib):
    inp = synth.prefill_inputs(1, 200, seed=9)
    d = to_dev(inp)
    ungated = lib.hyb_attn_prefill(d["q"], d["k"], d["v"], None, d["pos"], lib.FULL)
    half = lib.hyb_attn_prefill(d["q"], d["k"], d["v"], torch.zeros_like(d["gate"]), d["pos"], lib.FULL)
    # sigmoid(0) = 0.5 exactly and halving is exact in bf16
    assert torch.equal(half, (ungated.float() * 0.5).to(torch.bfloat16))


# ---------------------------------------------------------------------------
# KV caches: append (bit-exact bookkeeping), decode, chunked prefill
# ---------------------------------------------------------------------------
def test_linear_append_slots_and_rotation(lib):
    B, T1, T2 = 2, 100, 37
    cache = lib.KVCache(lib.FULL, B, capacity=256)
    a = synth.prefill_inputs(B, T1, seed=11)
    b = synth.prefill_inputs(B, T2, seed=12, start=T1)
    lib.hyb_kv_append(cache, a["k"].cuda(), a["v"].cuda())
    lib.hyb_kv_append(cache, b["k"].cuda(), b["v"].cuda(), pos=b["pos"].cuda())
    torch.cuda.synchronize()
    assert cache.len.tolist() == [T1 + T2] * B
    kc = cache.k.permute(0, 2, 1, 3).cpu()   # [B, cap, 4, 256]
    vc = cache.v.permute(0, 2, 1, 3).cpu()
    allk = torch.cat([a["k"], b["k"]], 1)
    allv = torch.cat([a["v"], b["v"]], 1)
    n = T1 + T2
    assert torch.equal(vc[:, :n], allv)                               # V copied bit for bit
    assert torch.count_nonzero(vc[:, n:]) == 0                        # untouched slots stay zero
    ref = O.rope_layer(f64(allk), np.arange(n)[None].repeat(B, 0), O.FULL)
    got = f64(kc[:, :n])
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-6)
    assert torch.equal(kc[:, :n, :, 64:], allk[..., 64:])            # dims 64..255 untouched


def test_ring_append_slot_map_bit_exact(lib):
    B = 3
    head0 = [0, 77, 511]
    cache = lib.KVCache(lib.SLIDING, B, head0=head0)
    sims = [O.RingSim(h) for h in head0]
    steps = [300, 1, 600, 211, 1]
    start = 0
    allk, allv = [], []
    for i, T in enumerate(steps):
        x = synth.prefill_inputs(B, T, seed=20 + i, start=start)
        lib.hyb_kv_append(cache, x["k"].cuda(), x["v"].cuda())
        for s in sims:
            s.append(T)
        allk.append(x["k"])
        allv.append(x["v"])
        start += T
    torch.cuda.synchronize()
    allk, allv = torch.cat(allk, 1), torch.cat(allv, 1)
    assert cache.len.tolist() == [start] * B
    assert cache.head.tolist() == [s.head for s in sims]
    tag = cache.tag.cpu().numpy()
    for b, s in enumerate(sims):
        assert np.array_equal(tag[b], s.tag)
        vc = cache.v[b].permute(1, 0, 2).cpu()   # [512, 4, 256]
        kc = f64(cache.k[b].permute(1, 0, 2))
        for slot in range(512):
            i = int(s.tag[slot])
            assert torch.equal(vc[slot], allv[b, i])
        idx = s.tag.astype(np.int64)
        ref = O.rope_layer(f64(allk[b, idx]), idx, O.SLIDING)
        assert np.all(np.abs(kc - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-6)


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
@pytest.mark.parametrize("lens", [[1, 5], [511, 513], [64, 1000], [2048, 3001]])
def test_decode_matches_oracle(lib, lt, lens):
    """Sequences of different lengths, each in its own single-sequence cache."""
    B = len(lens)
    L = max(lens)
    cap = L if lt == O.FULL else 512
    head0 = [(37 * b) % 512 for b in range(B)]
    hist = synth.prefill_inputs(B, L, seed=31)
    outs, refs = [], []
    for b, Lb in enumerate(lens):
        c1 = lib.KVCache(lt, 1, capacity=cap, head0=[head0[b]] if lt == O.SLIDING else None)
        k = hist["k"][b:b + 1, :Lb].cuda()
        v = hist["v"][b:b + 1, :Lb].cuda()
        lib.hyb_kv_append(c1, k, v)
        qd = synth.decode_query(1, seed=40 + b)
        out = lib.hyb_attn_decode(qd["q"].cuda(), qd["gate"].cuda(), c1, max_len=cap)
        outs.append(out)
        kr = O.rope_layer(f64(hist["k"][b, :Lb]), np.arange(Lb), lt)
        ref = O.decode(f64(qd["q"]), f64(qd["gate"]), [Lb - 1], [kr], [f64(hist["v"][b, :Lb])],
                       [np.arange(Lb)], lt)
        if lt == O.SLIDING:   # the ring only holds the last 512 tokens; the oracle's window agrees
            assert c1.len.tolist() == [Lb]
        refs.append(ref)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    assert_close(torch.cat(outs), np.concatenate(refs), f"decode lt={lt} lens={lens}")


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
def test_decode_batched_after_appends(lib, lt):
    """B=4 sequences decoded together after a prefill-sized append and 3 decode appends."""
    B, L0 = 4, 777
    cap = 1024 if lt == O.FULL else 512
    cache = lib.KVCache(lt, B, capacity=cap, head0=[5, 100, 300, 511] if lt == O.SLIDING else None)
    hist = synth.prefill_inputs(B, L0, seed=50)
    lib.hyb_kv_append(cache, hist["k"].cuda(), hist["v"].cuda())
    ks, vs = [hist["k"]], [hist["v"]]
    for step in range(3):
        qd = synth.decode_query(B, seed=60 + step)
        lib.hyb_kv_append(cache, qd["k"].cuda(), qd["v"].cuda())
        ks.append(qd["k"])
        vs.append(qd["v"])
        out = lib.hyb_attn_decode(qd["q"].cuda(), qd["gate"].cuda(), cache, max_len=cap)
        n = L0 + step + 1
        allk = torch.cat(ks, 1)
        allv = torch.cat(vs, 1)
        lo = 0 if lt == O.FULL else max(0, n - 512)
        idx = np.arange(lo, n)
        kr = [O.rope_layer(f64(allk[b, lo:n]), idx, lt) for b in range(B)]
        ref = O.decode(f64(qd["q"]), f64(qd["gate"]), [n - 1] * B, kr, [f64(allv[b, lo:n]) for b in range(B)],
                       [idx] * B, lt)
        assert_close(out, ref, f"batched decode step {step}")
    assert lib.hyb_device_error() == 0


@pytest.mark.parametrize("lt", [O.SLIDING, O.FULL])
@pytest.mark.parametrize("chunks", [[300, 300, 300], [1000, 24, 700]])
def test_chunked_prefill_with_cache(lib, lt, chunks):
    B = 2
    n = sum(chunks)
    cap = n if lt == O.FULL else 512
    cache = lib.KVCache(lt, B, capacity=cap, head0=[3, 400] if lt == O.SLIDING else None)
    inp = synth.prefill_inputs(B, n, seed=70)
    outs = []
    s0 = 0
    for T in chunks:
        sl = slice(s0, s0 + T)
        qkv = inp["qkv"][:, sl].contiguous().cuda()
        q = qkv[..., :4096].unflatten(-1, (16, 256))
        k = qkv[..., 4096:5120].unflatten(-1, (4, 256))
        v = qkv[..., 5120:].unflatten(-1, (4, 256))
        outs.append(lib.hyb_attn_prefill(q, k, v, inp["gate"][:, sl].contiguous().cuda(), None, lt,
                                         cache=cache))
        s0 += T
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    assert cache.len.tolist() == [n] * B
    got = torch.cat(outs, 1)
    ref = oracle_prefill(inp, lt)
    assert_close(got, ref, f"chunked lt={lt} chunks={chunks}")


def test_full_cache_overflow_sets_flag_and_keeps_state(lib):
    cache = lib.KVCache(lib.FULL, 1, capacity=100)
    a = synth.prefill_inputs(1, 80, seed=80)
    lib.hyb_kv_append(cache, a["k"].cuda(), a["v"].cuda())
    before = cache.k.clone()
    b = synth.prefill_inputs(1, 30, seed=81)
    lib.hyb_kv_append(cache, b["k"].cuda(), b["v"].cuda())
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == lib.DEV_ERR_CAPACITY
    assert cache.len.tolist() == [80]
    assert torch.equal(cache.k, before)
    assert lib.hyb_device_error() == 0   # cleared by the previous read


def test_bounded_wait_times_out_and_context_stays_usable(lib):
    """A device-side wait that nothing satisfies gives up after its limit and
    raises the timeout bit instead of hanging; the next calls work."""
    import time
    lib.hyb_device_error(clear=True)
    t0 = time.perf_counter()
    lib.hyb_selftest_wait_timeout()
    flags = lib.hyb_device_error(clear=True)
    elapsed = time.perf_counter() - t0
    assert flags == lib.DEV_ERR_TIMEOUT
    assert 0.5 < elapsed < 30.0, elapsed
    # the context is usable: a small prefill still matches the oracle
    x = synth.prefill_inputs(1, 300, seed=77, device="cuda")
    out = lib.hyb_attn_prefill(x["q"], x["k"], x["v"], x["gate"], x["pos"], lib.FULL)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    h = {k: x[k].float().cpu().double().numpy() for k in ("q", "k", "v", "gate")}
    ref = O.prefill(h["q"], h["k"], h["v"], h["gate"], x["pos"].cpu().numpy(), O.FULL)
    got = out.float().cpu().double().numpy()
    assert np.abs(got - ref).max() <= 2e-2
