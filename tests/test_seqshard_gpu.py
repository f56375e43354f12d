"""Sequence-sharded decode kernels on one GPU: a full-layer history spread
over three caches (one per would-be GPU, one of them empty), each part's
hyb_attn_decode_partial against the oracle's decode_partial, and
hyb_attn_decode_merge of the parts against the oracle's decode over the
whole history.  The ranks are emulated one after another on one device
(their kernels never wait on each other)."""
import numpy as np
import pytest
import torch

import oracle as O
from full_gqa_attention_partial_b200 import synth

pytestmark = pytest.mark.gpu


def f64(t):
    return t.detach().float().cpu().double().numpy()


def _spread(lib, whole, L, owner, n_parts):
    """Caches holding the rows of `whole` whose owner is p, in position order."""
    B = whole.batch
    parts, held = [], []
    for p in range(n_parts):
        rows = np.nonzero(owner == p)[0]
        c = lib.KVCache(O.FULL, B, capacity=max(64, len(rows) + 64 - len(rows) % 64))
        if len(rows):
            idx = torch.from_numpy(rows).cuda()
            c.k[:, :, :len(rows)].copy_(whole.k[:, :, idx])
            c.v[:, :, :len(rows)].copy_(whole.v[:, :, idx])
        c.len.fill_(len(rows))
        parts.append(c)
        held.append(rows)
    return parts, held


def test_partials_and_merge_match_the_oracle(lib):
    B, L = 2, 3000
    whole = lib.KVCache(O.FULL, B, capacity=L + 64)
    synth.fill_cache_randn_(whole.k, whole.v, L, 121)
    whole.len.fill_(L)
    # blocks of 100 tokens dealt to parts 0 and 1; part 2 holds nothing
    owner = (np.arange(L) // 100) % 2
    parts, held = _spread(lib, whole, L, owner, 3)
    x = synth.decode_query(B, seed=122, device="cuda")
    pos = torch.full((B,), L, dtype=torch.int32, device="cuda")
    outs = [lib.hyb_attn_decode_partial(x["q"], c, pos=pos, max_len=c.capacity) for c in parts]
    merged = lib.hyb_attn_decode_merge(torch.stack([o for o, _ in outs]), torch.stack([l for _, l in outs]), x["gate"])
    whole_out = lib.hyb_attn_decode(x["q"], x["gate"], whole, pos=pos, max_len=whole.capacity)
    torch.cuda.synchronize()
    assert lib.hyb_device_error() == 0
    kk, vv = f64(whole.k[:, :, :L]).transpose(0, 2, 1, 3), f64(whole.v[:, :, :L]).transpose(0, 2, 1, 3)
    q64 = f64(x["q"])
    for p, (o, lse) in enumerate(outs):
        ro, rl = O.decode_partial(q64, [L] * B, [kk[b][held[p]] for b in range(B)],
                                  [vv[b][held[p]] for b in range(B)], O.FULL)
        if len(held[p]) == 0:
            assert torch.all(lse == -float("inf")) and torch.all(o == 0)
            continue
        assert np.abs(f64(lse) - rl).max() < 2e-2, p
        err = f64(o) - ro
        assert np.abs(err).max() < 2e-2 and np.linalg.norm(err) / np.linalg.norm(ro) < 5e-3, p
    ref = O.decode(q64, f64(x["gate"]), [L] * B, list(kk), list(vv), [np.arange(L)] * B, O.FULL)
    for got in (f64(merged), f64(whole_out)):
        max_abs = float(np.abs(got - ref).max())
        rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
        assert max_abs <= 2e-2 and rel <= 5e-3, f"max_abs {max_abs:.3e} rel_l2 {rel:.3e}"


def test_sharded_decoder_single_rank_matches_decode(lib):
    """SeqShardedDecoder with one rank (no process group): append, partial,
    merge of one part equals hyb_attn_decode on the same cache."""
    from full_gqa_attention_partial_b200 import seqshard
    B, L = 2, 1000
    a = lib.KVCache(O.FULL, B, capacity=L + 64)
    b = lib.KVCache(O.FULL, B, capacity=L + 64)
    synth.fill_cache_randn_(a.k, a.v, L, 131)
    b.k.copy_(a.k)
    b.v.copy_(a.v)
    a.len.fill_(L)
    b.len.fill_(L)
    dec = seqshard.SeqShardedDecoder(a)
    for s in range(3):
        x = synth.decode_query(B, seed=132 + s, device="cuda")
        pos = torch.full((B,), L + s, dtype=torch.int32, device="cuda")
        got = dec.step(x["q"], x["k"], x["v"], x["gate"], pos, s)
        lib.hyb_kv_append(b, x["k"], x["v"])
        ref = lib.hyb_attn_decode(x["q"], x["gate"], b, max_len=b.capacity)
        torch.cuda.synchronize()
        assert lib.hyb_device_error() == 0
        d = (got.float() - ref.float()).abs().max().item()
        assert d <= 1e-2, (s, d)     # one part through the merge vs the splits' own combine
