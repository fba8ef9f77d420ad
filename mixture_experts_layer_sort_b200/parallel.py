"""Tensor parallelism of the MoE layer over the expert intermediate dimension.

The pages deploy the layer at eight-way tensor parallelism (toolboxkart.tech, "AWS
SageMaker MoE kernel optimizations H200", section "3. Removing repeat compilation can
reduce first-token delay"). Rank g of G holds rows [g*I/G, (g+1)*I/G) of every
W_gate[e] and W_up[e] and the matching columns of every W_down[e]
(moe_load_weights_shard). Routing reads only the logits, so every rank routes alike;
each rank's forward is the library's forward of its slice, and the layer's output is
the sum of the ranks' outputs: one all-reduce (NCCL over NVLink between GPUs) per
forward. This module is plumbing only: the forward runs in the library's kernels and
the sum in the collective.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


class TensorParallelMoE:
    """One rank's shard of a layer with full intermediate size I_full, split over
    `world` ranks of `group` (the default process group when None)."""

    def __init__(self, E: int, topk: int, H: int, I_full: int, dtype="bf16", rank: int | None = None,
                 world: int | None = None, group=None, layer=None):
        self.group = group
        self.world = world if world is not None else (dist.get_world_size(group) if dist.is_initialized() else 1)
        self.rank = rank if rank is not None else (dist.get_rank(group) if dist.is_initialized() else 0)
        if I_full % self.world or (I_full // self.world) % 128:
            raise ValueError(f"I_full={I_full} must split into {self.world} shards of a multiple of 128")
        self.I_full = I_full
        if layer is None:
            from .layer import MoELayer
            layer = MoELayer(E, topk, H, I_full // self.world, dtype)
        self.layer = layer

    def load_weights(self, w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor, stream=None):
        """Full bf16 tensors [E,I_full,H], [E,I_full,H], [E,H,I_full] on this rank's device."""
        self.layer.load_weights_shard(w_gate, w_up, w_down, self.rank, self.world, stream=stream)

    def forward(self, x: torch.Tensor, logits: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        """This rank's partial output, then the all-reduce that sums the ranks' partials
        (in place in `out`). Both run on `stream` (a torch.cuda.Stream or a raw
        cudaStream_t handle), or on the current stream when it is None, so the collective
        is ordered after the forward that writes `out`."""
        out = self.layer.forward(x, logits, out=out, stream=stream)
        if self.world > 1:
            if stream is None:
                dist.all_reduce(out, op=dist.ReduceOp.SUM, group=self.group)
            else:
                s = stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.ExternalStream(stream)
                with torch.cuda.stream(s):
                    dist.all_reduce(out, op=dist.ReduceOp.SUM, group=self.group)
        return out

    __call__ = forward

    def close(self):
        self.layer.close()
