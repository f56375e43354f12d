"""Sequence-sharded decode orchestration (seqshard.py) on CPU: two gloo ranks
share a full-layer history.  The attention itself comes from the oracle in
a stand-in for the library binding (this file is test infrastructure), so
what is checked is the orchestration: the history split, which rank stores
each step's token, the all-gather of the partials and their merge.  Every
rank's output must equal the oracle's decode over the whole history."""
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _OracleCache:
    """This rank's part of a full-layer history, held as rotated fp64 rows."""

    def __init__(self, batch, capacity):
        import oracle as O
        self.layer_type = O.FULL
        self.batch = batch
        self.capacity = capacity
        self.k = torch.zeros(1)                      # device of the part: the CPU
        self.keys = [[] for _ in range(batch)]
        self.vals = [[] for _ in range(batch)]
        self.pos = [[] for _ in range(batch)]


class _OracleLib:
    """Stand-in for the binding's decode calls, computed by the oracle."""

    @staticmethod
    def hyb_kv_append(cache, k, v, pos):
        import oracle as O
        for b in range(cache.batch):
            p = pos[b].numpy()
            kr = O.rope_layer(k[b].double().numpy(), p, O.FULL)
            for t in range(k.shape[1]):
                cache.keys[b].append(kr[t])
                cache.vals[b].append(v[b, t].double().numpy())
                cache.pos[b].append(int(p[t]))

    @staticmethod
    def hyb_attn_decode_partial(q, cache, pos, max_len, part_o, part_lse, workspace):
        import oracle as O
        ks = [np.array(cache.keys[b]).reshape(-1, 4, 256) for b in range(cache.batch)]
        vs = [np.array(cache.vals[b]).reshape(-1, 4, 256) for b in range(cache.batch)]
        o, lse2 = O.decode_partial(q.double().numpy(), pos.numpy(), ks, vs, O.FULL)
        part_o.copy_(torch.from_numpy(o))
        part_lse.copy_(torch.from_numpy(lse2))

    @staticmethod
    def hyb_attn_decode_merge_records(records, B, gate):
        import oracle as O
        n = B * 16 * 256
        r = records.double().numpy()
        g = None if gate is None else gate.double().numpy()
        return torch.from_numpy(O.merge_partials(r[:, :n].reshape(-1, B, 16, 256), r[:, n:].reshape(-1, B, 16), g))


def _inputs(B, n, seed):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, n, 4, 256, generator=g)
    v = torch.randn(B, n, 4, 256, generator=g)
    q = torch.randn(B, n, 16, 256, generator=g)
    gate = torch.randn(B, n, 16, generator=g)
    return k, v, q, gate


def _worker(rank, world, port, q_out, n0, steps, block):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import oracle as O
    from full_gqa_attention_partial_b200 import seqshard
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B = 2
        k, v, q, gate = _inputs(B, n0 + steps, seed=11)
        cache = _OracleCache(B, n0 + steps)
        lib = _OracleLib()
        lo, hi = seqshard.history_range(n0, world, rank)
        if hi > lo:
            pos = torch.arange(lo, hi, dtype=torch.int32).expand(B, -1)
            lib.hyb_kv_append(cache, k[:, lo:hi], v[:, lo:hi], pos)
        dec = seqshard.SeqShardedDecoder(cache, block=block, lib=lib)
        worst = 0.0
        for s in range(steps):
            t = n0 + s
            pos = torch.full((B,), t, dtype=torch.int32)
            out = dec.step(q[:, t], k[:, t:t + 1], v[:, t:t + 1], gate[:, t], pos, s)
            if s % 7 == 0 or s == steps - 1:
                ref = O.decode(q[:, t].double().numpy(), gate[:, t].double().numpy(), [t] * B,
                               [O.rope_layer(k[b, :t + 1].double().numpy(), np.arange(t + 1), O.FULL) for b in range(B)],
                               [v[b, :t + 1].double().numpy() for b in range(B)], [np.arange(t + 1)] * B, O.FULL)
                worst = max(worst, float(np.abs(out.numpy() - ref).max()))
        held = [sorted(p) for p in cache.pos]
        q_out.put((rank, worst, held))
    finally:
        dist.destroy_process_group()


def test_two_ranks_share_history_and_steps():
    world, n0, steps, block = 2, 45, 70, 32
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, n0, steps, block)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, worst, _ in res:
        assert worst < 1e-5          # the partials travel as fp32
    # every position is held by exactly one rank; history in contiguous halves, steps in blocks of 32
    for b in range(2):
        allpos = sorted(p for _, _, held in res for p in held[b])
        assert allpos == list(range(n0 + steps))
    r0 = set(res[0][2][0])
    assert set(range(0, 23)) <= r0 and not (set(range(23, 45)) & r0)
    assert set(range(45, 45 + 32)) <= r0 and not (set(range(45 + 32, 45 + 64)) & r0)
    assert set(range(45 + 64, 45 + 70)) <= r0


def test_history_range_partitions():
    sys.path.insert(0, ROOT)
    from full_gqa_attention_partial_b200 import seqshard
    for n in (0, 1, 7, 1 << 20):
        for world in (1, 2, 3, 8):
            parts = [seqshard.history_range(n, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
