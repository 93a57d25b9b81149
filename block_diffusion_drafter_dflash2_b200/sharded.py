"""Output head sharded by vocabulary across GPUs, one process per GPU (include/dflash2.h,
dflash2_draft_step_head_shard / dflash2_select).

Every rank holds the layers and the rows [v0, v0 + rows) of the output head; its step ends with
its local top-16 per drafted row (vocabulary ids).  The ranks exchange those lists (an all-gather
over torch.distributed: NCCL over NVLink on GPUs, gloo in the CPU tests) and one rank runs the
selector on the gathered lists.  This module partitions the vocabulary, marshals the calls and
performs the exchange; every step of the arithmetic runs in the library's kernels.
"""
from __future__ import annotations

import ctypes as C
from typing import List, Optional, Tuple

import torch

from . import binding


def vocab_shards(V: int, G: int, align: int = 256) -> List[Tuple[int, int]]:
    """Contiguous (v0, rows) ranges of a V-token head over G ranks: boundaries on multiples of
    `align` (whole 256-row head records), sizes within one record of each other, every rank at
    least 16 rows (V and the sizes multiples of 16)."""
    assert V % 16 == 0 and G >= 1 and align % 16 == 0
    units = V // align
    cuts = [round(i * units / G) * align for i in range(G)] + [V]
    shards = [(cuts[i], cuts[i + 1] - cuts[i]) for i in range(G)]
    assert all(r >= 16 and r % 16 == 0 for _, r in shards), shards
    return shards


def exchange_candidates(val: torch.Tensor, ids: torch.Tensor, group=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All-gather of every rank's [rows][16] candidate values and ids into [G][rows][16] each, in rank
    order (one collective: the ids travel bit-cast beside the values)."""
    import torch.distributed as dist
    G = dist.get_world_size(group)
    packed = torch.stack([val.float(), ids.to(torch.int32).view(torch.float32)])  # [2][rows][16]
    out = torch.empty((G * 2,) + tuple(packed.shape[1:]), dtype=packed.dtype, device=packed.device)
    dist.all_gather_into_tensor(out, packed.contiguous(), group=group)  # rank-major [G * 2][rows][16]
    out = out.view((G, 2) + tuple(packed.shape[1:]))
    return out[:, 0].contiguous(), out[:, 1].contiguous().view(torch.int32)


class ShardedDrafter:
    """One rank of a drafter whose output head is split by vocabulary.  `weights` holds the layers
    (prepared on this device like binding.Drafter) and the whole head on the host or device; the
    rank prepares only its shard's rows for the step."""

    def __init__(self, dims, weights: dict, batch: int, rank: int, world: int, group=None, root: int = 0):
        self.lib = binding.load()
        self.base = binding.Drafter(dims, weights, batch)
        self.dims, self.batch, self.rank, self.world, self.group, self.root = dims, batch, rank, world, group, root
        self.v0, self.rows = vocab_shards(dims.vocab, world)[rank]
        dev = self.base.workspace.device
        cfg = self.base.cfg
        n = self.lib.dflash2_head_shard_size(C.byref(cfg), self.rows)
        self.head = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
        lm = weights["lm_head"][self.v0:self.v0 + self.rows].to(dev).contiguous()
        sp = weights["sel_proj"].to(dev).contiguous()
        binding.check(self.lib.dflash2_prepare_head_shard(C.byref(cfg), binding._ptr(lm), self.rows, binding._ptr(sp),
                                                          binding._ptr(self.head), n, binding._stream()),
                      "prepare_head_shard")
        D = dims.block - 1
        self.cand_val = torch.empty((batch * D, 16), dtype=torch.float32, device=dev)
        self.cand_id = torch.empty((batch * D, 16), dtype=torch.int32, device=dev)
        self.z = torch.empty((batch * D, dims.rank), dtype=torch.float32, device=dev)

    def local_step(self, inputs: dict, state: dict, stream=None, kv: Optional[binding.KV] = None):
        """The layers and this rank's head shard: local candidates (vocabulary ids) and z."""
        ins = binding.Inputs(inputs["taps"].data_ptr(), inputs["n_new"].data_ptr(), inputs["block_tokens"].data_ptr())
        kvs = kv if kv is not None else binding.kv_struct(state)
        b = self.base
        binding.check(self.lib.dflash2_draft_step_head_shard(
            C.byref(b.cfg), C.byref(b.w), binding._ptr(self.head), self.v0, self.rows, C.byref(ins), C.byref(kvs),
            self.batch, binding._ptr(self.cand_val), binding._ptr(self.cand_id), binding._ptr(self.z),
            binding._ptr(b.workspace), b.ws_bytes, binding._stream(stream)), "draft_step_head_shard")

    def select(self, vals: torch.Tensor, ids: torch.Tensor, block_tokens: torch.Tensor, out_path, out_scores,
               stream=None):
        """The selector on G gathered lists ([G][rows][16]) with this rank's z."""
        b = self.base
        binding.check(self.lib.dflash2_select(
            C.byref(b.cfg), C.byref(b.w), self.batch, int(vals.shape[0]), binding._ptr(vals), binding._ptr(ids),
            binding._ptr(self.z), binding._ptr(block_tokens), binding._ptr(out_path), binding._ptr(out_scores),
            binding._ptr(b.workspace), b.ws_bytes, binding._stream(stream)), "select")

    def draft_step(self, inputs: dict, state: dict, out_path, out_scores, kv=None):
        """Local step, exchange, selection on the root rank, path and scores broadcast to all ranks."""
        import torch.distributed as dist
        self.local_step(inputs, state, kv=kv)
        vals, ids = exchange_candidates(self.cand_val, self.cand_id, self.group)
        if self.rank == self.root:
            self.select(vals, ids, inputs["block_tokens"], out_path, out_scores)
        dist.broadcast(out_path, self.root, group=self.group)
        dist.broadcast(out_scores, self.root, group=self.group)
