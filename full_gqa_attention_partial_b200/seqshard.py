"""Sequence-sharded decode of full-attention layers over several GPUs.

A million-token full-layer history (4.3 GB per layer per sequence in bf16)
can be spread over the GPUs of a node instead of being held by one.  One
process per GPU (torch.distributed, NCCL); each rank's full-layer cache
holds a part of every sequence's history:

* the history present at the start is split into contiguous ranges
  (`history_range`), which the caller appends (or prefills) on each rank
  with the tokens' own positions, so keys are rotated as in one cache;
* each decode step's new token goes to exactly one rank: steps are dealt in
  blocks of `block` steps round-robin over the ranks (`owner`), which keeps
  the parts within one block of each other.

A decode step then runs, on every rank, the attention of the (replicated)
query over the local part (hyb_attn_decode_partial: normalised output and
base-2 log-sum-exp per head, written into one record of 16 heads x (256 +
1) fp32 = 16 KB per sequence), one all-gather of the records, and
hyb_attn_decode_merge over the gathered records, which weighs each part by
2^lse and applies the gate.  Attention over the union equals this merge
exactly (the split-KV identity), so every rank ends the step with the full
layer's output, as the replicated layers after it expect.  Sliding layers
keep their 512-slot rings whole on every rank.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def history_range(n_tokens: int, world: int, rank: int) -> tuple[int, int]:
    """Tokens [start, stop) of an n_tokens history that `rank` holds:
    contiguous ranges, sizes differing by at most one."""
    base, extra = divmod(int(n_tokens), int(world))
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


class SeqShardedDecoder:
    """Decode steps of one full-attention layer whose history is spread over
    the ranks of `group`.

    cache: this rank's full-layer KVCache (its part of every sequence).
    block: decode steps per round-robin block (which rank stores a step's token).
    lib:   the library binding (the package itself; replaceable in tests of
           the orchestration).
    """

    def __init__(self, cache, block: int = 64, group=None, lib=None):
        if lib is None:
            import full_gqa_attention_partial_b200 as lib
        self.lib = lib
        self.cache = cache
        self.block = int(block)
        self.group = group
        if dist.is_available() and dist.is_initialized():
            self.world = dist.get_world_size(group)
            self.rank = dist.get_rank(group)
            self.backend = dist.get_backend(group)
        else:
            self.world, self.rank, self.backend = 1, 0, None
        B = cache.batch
        dev = cache.k.device
        n_o = B * 16 * 256
        # this rank's record (output, then lse) and every rank's, gathered
        self.rec = torch.empty(n_o + B * 16, dtype=torch.float32, device=dev)
        self.part_o = self.rec[:n_o].view(B, 16, 256)
        self.part_lse = self.rec[n_o:].view(B, 16)
        self.all_rec = self.rec.view(1, -1) if self.world == 1 else \
            torch.empty(self.world, n_o + B * 16, dtype=torch.float32, device=dev)
        self.workspace = None
        if dev.type == "cuda":
            need = lib.hyb_attn_decode_workspace_size(cache.layer_type, B, cache.capacity)
            self.workspace = lib.alloc_workspace(need, dev)

    def owner(self, step: int) -> int:
        """Rank that stores the token of decode step `step`."""
        return (int(step) // self.block) % self.world

    def step(self, q, k, v, gate, pos, step: int):
        """One decode step: q [B,16,256] (the same on every rank), the new
        token's k / v [B,1,4,256], gate [B,16] or None, pos int32 [B] the new
        token's position in the whole sequence.  Returns bf16 [B,16,256]."""
        lib = self.lib
        if self.owner(step) == self.rank:
            lib.hyb_kv_append(self.cache, k, v, pos=pos.view(-1, 1))
        lib.hyb_attn_decode_partial(q, self.cache, pos=pos, max_len=self.cache.capacity, part_o=self.part_o,
                                    part_lse=self.part_lse, workspace=self.workspace)
        self._gather()
        return lib.hyb_attn_decode_merge_records(self.all_rec, self.cache.batch, gate)

    def _gather(self):
        if self.world == 1:
            return                      # the only record is this rank's
        if self.backend == "nccl":
            dist.all_gather_into_tensor(self.all_rec, self.rec, group=self.group)
        else:
            dist.all_gather(list(self.all_rec.unbind(0)), self.rec, group=self.group)
