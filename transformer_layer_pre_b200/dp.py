"""Data-parallel replicas of the encoder layer: one process per GPU, each on
its own micro-batch, and one all-reduce of the float32 parameter gradients
per step ("Transformer deployment", section on distributed training: data
parallelism with NCCL gradient all-reduce).

The twelve gradient tensors of a layer are views into one flat float32
buffer, so the exchange is a single collective over ~50 MB (BERT-Large)
instead of twelve small ones; NCCL over NVLink/NVSwitch on GPUs, gloo on
CPU for the host-side tests.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

WEIGHT_NAMES = (
    "wqkv", "bqkv", "wo", "bo", "ln1_g", "ln1_b",
    "w1", "b1", "w2", "b2", "ln2_g", "ln2_b",
)


def gradient_shapes(hidden: int, ffn: int) -> dict:
    """Shapes of the twelve parameter gradients (Linear weights are [out, in])."""
    h, f = hidden, ffn
    return {"wqkv": (3 * h, h), "bqkv": (3 * h,), "wo": (h, h), "bo": (h,), "ln1_g": (h,), "ln1_b": (h,),
            "w1": (f, h), "b1": (f,), "w2": (h, f), "b2": (h,), "ln2_g": (h,), "ln2_b": (h,)}


class FlatGrads:
    """The gradients of one layer as views into one contiguous float32 buffer
    (16-byte aligned views, as the C ABI requires)."""

    def __init__(self, hidden: int, ffn: int, device):
        shapes = gradient_shapes(hidden, ffn)
        sizes = {n: int(torch.Size(s).numel()) for n, s in shapes.items()}
        offs, o = {}, 0
        for n in WEIGHT_NAMES:
            offs[n] = o
            o += (sizes[n] + 3) // 4 * 4      # keep every view 16-byte aligned
        self.flat = torch.zeros(o, dtype=torch.float32, device=device)
        self.views = {n: self.flat[offs[n]:offs[n] + sizes[n]].view(shapes[n]) for n in WEIGHT_NAMES}

    def __getitem__(self, name):
        return self.views[name]

    def as_dict(self) -> dict:
        return dict(self.views)


def allreduce_mean(grads: FlatGrads, group=None) -> None:
    """Averages the gradients over the ranks of `group` in place (one
    collective).  No-op without an initialised process group of size > 1."""
    if not (dist.is_available() and dist.is_initialized()):
        return
    world = dist.get_world_size(group)
    if world == 1:
        return
    dist.all_reduce(grads.flat, op=dist.ReduceOp.SUM, group=group)
    grads.flat.mul_(1.0 / world)
