"""hyb_attn_decode_noalloc: decode without a caller workspace.

For callers that may not allocate device memory on their decode path (a
plugin inside an application that owns all device memory, a latency-critical
loop where cudaMalloc would stall the device), the split partials live in a
fixed 4 MiB scratch array inside the library.  These tests call it through
the C ABI and compare it with hyb_attn_decode (the workspace entry point)
on two calls in a row: the second call must not be disturbed by what the
first left in the shared scratch.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle as O
from full_gqa_attention_partial_b200 import synth

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
REL_L2 = 5e-3


def _close(a, b, what):
    a = a.float().cpu().double().numpy()
    b = b.float().cpu().double().numpy()
    max_abs = float(np.abs(a - b).max())
    rel = float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))
    assert np.all(np.isfinite(a)), what
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"{what}: max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


@pytest.mark.parametrize("lt", [0, 1])
def test_noalloc_decode_matches_workspace_decode_twice(lib, lt):
    B = 3
    cap = 4096 if lt == lib.FULL else 512
    cache = lib.KVCache(lt, B, capacity=cap, head0=[7, 300, 511] if lt == lib.SLIDING else None)
    hist = synth.prefill_inputs(B, 3000, seed=900 + lt)
    lib.hyb_kv_append(cache, hist["k"].cuda(), hist["v"].cuda())
    for call in range(2):
        qd = synth.decode_query(B, seed=910 + 10 * lt + call)
        lib.hyb_kv_append(cache, qd["k"].cuda(), qd["v"].cuda())
        q, gate = qd["q"].cuda(), qd["gate"].cuda()
        ref = lib.hyb_attn_decode(q, gate, cache, max_len=cap)
        out = torch.empty_like(q)
        lib.hyb_attn_decode_noalloc(q, gate, cache, max_len=cap, out=out)
        torch.cuda.synchronize()
        _close(out, ref, f"layer type {lt}, call {call}")
    assert lib.hyb_device_error() == 0


def test_noalloc_decode_rejects_batches_beyond_the_fixed_scratch(lib):
    # 300 sequences x 16 heads x 1 split x 1 KB of partials exceed 4 MiB
    cache = lib.KVCache(lib.SLIDING, 300)
    q = torch.zeros(300, 16, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.HybError) as e:
        lib.hyb_attn_decode_noalloc(q, None, cache, max_len=512, out=torch.empty_like(q))
    assert e.value.status == -4
    assert "fixed scratch" in str(e.value)


@pytest.mark.parametrize("lt", [0, 1])
def test_noalloc_decode_matches_oracle(lib, lt):
    """The allocation-free entry point against the oracle directly: the
    oracle gets the raw history and the new token and applies RoPE, the
    window and the gate itself."""
    B, n_hist = 2, 900
    cap = 1024 if lt == lib.FULL else 512
    cache = lib.KVCache(lt, B, capacity=cap, head0=[5, 400] if lt == lib.SLIDING else None)
    hist = synth.prefill_inputs(B, n_hist, seed=930 + lt)
    lib.hyb_kv_append(cache, hist["k"].cuda(), hist["v"].cuda())
    qd = synth.decode_query(B, seed=940 + lt)
    lib.hyb_kv_append(cache, qd["k"].cuda(), qd["v"].cuda())
    out = torch.empty(B, 16, 256, dtype=torch.bfloat16, device="cuda")
    lib.hyb_attn_decode_noalloc(qd["q"].cuda(), qd["gate"].cuda(), cache, max_len=cap, out=out)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    f = lambda t: t.float().double().numpy()
    n = n_hist + 1
    lo = 0 if lt == lib.FULL else n - 512
    idx = np.arange(lo, n)
    keys = [O.rope_layer(np.concatenate([f(hist["k"][b]), f(qd["k"][b])])[lo:], idx, lt) for b in range(B)]
    vals = [np.concatenate([f(hist["v"][b]), f(qd["v"][b])])[lo:] for b in range(B)]
    ref = O.decode(f(qd["q"]), f(qd["gate"]), [n - 1] * B, keys, vals, [idx] * B, lt)
    got = out.float().cpu().double().numpy()
    max_abs = float(np.abs(got - ref).max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    assert max_abs <= MAX_ABS and rel <= REL_L2, f"max_abs {max_abs:.3e} rel_l2 {rel:.3e}"
