"""Expert parallelism for the ternary MoE block: one process per GPU, the experts split by rank.

Each rank holds a contiguous range of the experts (``expert_range``) in a layer handle created
with ``expert_lo`` / ``n_local_experts``, the full router, and the dense part of the block (shared
expert and correction).  Tokens are data-parallel: every rank brings its own batch of T tokens
(the same T on every rank).  One forward:

  1. all-gather the ranks' batches (bf16 moved as bytes);
  2. each rank computes the routed part of its experts for all gathered tokens (the library's
     forward with SCION_OPT_PARTS = SCION_PART_ROUTED: routing over all experts, grouping and the
     expert GEMMs only for the local ones);
  3. reduce-scatter (sum) returns to each rank the routed output of its own tokens;
  4. each rank adds the dense part for its own tokens (the residual entry point with
     SCION_OPT_PARTS = SCION_PART_DENSE, in place).

Expert parallelism is not on the pages ("Scion: ternary MoE quantization with trained
corrections", Serving notes, places one model's experts on more than one device); this is the
plainest split, by expert.  The collectives are torch.distributed's (NCCL on GPUs, gloo on CPU);
every step of the block's arithmetic runs in the library (or, for the CPU tests, in the backend
they pass).
"""
from __future__ import annotations

from typing import Tuple


def expert_range(n_experts: int, world: int, rank: int) -> Tuple[int, int]:
    """(first expert, number of experts) of `rank`: contiguous ranges, the first n_experts % world
    ranks one expert more."""
    if world < 1 or not 0 <= rank < world or n_experts < world:
        raise ValueError("need 0 <= rank < world <= n_experts")
    base, extra = divmod(n_experts, world)
    lo = rank * base + min(rank, extra)
    return lo, base + (1 if rank < extra else 0)


class LibraryBackend:
    """The two forwards of one rank on its layer handle (experts of its range, dense part)."""

    def __init__(self, layer, stream=None):
        self.layer, self.stream = layer, stream

    def routed(self, x_all, out_all) -> None:
        import ternary_quantized_moe_b200 as tq

        tq.scion_layer_set_option(self.layer, tq.SCION_OPT_PARTS, tq.SCION_PART_ROUTED)
        tq.scion_moe_forward(x_all, x_all.shape[0], self.layer, out_all, self.stream)

    def dense_add(self, x, out) -> None:
        import ternary_quantized_moe_b200 as tq

        tq.scion_layer_set_option(self.layer, tq.SCION_OPT_PARTS, tq.SCION_PART_DENSE)
        tq.scion_moe_forward_residual(x, x.shape[0], self.layer, out, out, self.stream)
        tq.scion_layer_set_option(self.layer, tq.SCION_OPT_PARTS, tq.SCION_PART_ROUTED | tq.SCION_PART_DENSE)


class ExpertParallelBlock:
    """The block over the ranks of `group`: forward(x, out) with this rank's tokens x (bf16
    [T, d]) and out (fp32 [T, d], written).  The handle behind `backend` must accept world * T
    tokens."""

    def __init__(self, backend, d: int, group=None):
        self.backend, self.d, self.group = backend, d, group

    def forward(self, x, out) -> None:
        import torch
        import torch.distributed as dist

        world = dist.get_world_size(self.group)
        T = x.shape[0]
        # 1. all ranks' tokens, in rank order (bf16 moved as bytes)
        x_all = torch.empty((world * T, self.d), dtype=x.dtype, device=x.device)
        dist.all_gather_into_tensor(x_all.view(torch.uint8), x.contiguous().view(torch.uint8), group=self.group)
        # 2. the routed part of this rank's experts for every token
        part = torch.empty((world * T, self.d), dtype=torch.float32, device=x.device)
        self.backend.routed(x_all, part)
        # 3. every token's routed output summed over the ranks, back on its own rank
        dist.reduce_scatter_tensor(out, part, op=dist.ReduceOp.SUM, group=self.group)
        # 4. the dense part of this rank's tokens
        self.backend.dense_add(x, out)
