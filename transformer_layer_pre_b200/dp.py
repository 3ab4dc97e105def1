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


class GradExchanger:
    """Per-layer gradient all-reduce overlapped with the rest of a backward
    pass: `submit(grads)` right after a layer's backward enqueues the mean
    over ranks of that layer's flat buffer on a side stream that first waits
    for the layer's kernels, so the collective runs while the next (lower)
    layer's backward computes; `finish()` makes the caller's stream wait for
    every submitted exchange.  Every rank must submit the same buffers in the
    same order (in a stack with layer dropping the decisions are equal on all
    ranks).  Without a process group of size > 1 both calls do nothing; CPU
    tensors (gloo) are reduced synchronously.

    `allreduce` (with `world`) replaces the collective: a callable that sums
    a tensor over `world` ranks in place, enqueued on the current stream (by
    default torch.distributed's all_reduce over `group`)."""

    def __init__(self, group=None, allreduce=None, world: int | None = None):
        self.group = group
        if allreduce is not None:
            if world is None:
                raise ValueError("a replacement collective needs the world size")
            self.world = int(world)
            self.allreduce = allreduce
        else:
            self.world = (dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1)
            self.allreduce = lambda t: dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)
        self.stream = None
        self.pending = 0

    def submit(self, grads: FlatGrads, stream=None) -> None:
        """`stream`: the stream the layer's backward was enqueued on (None:
        the current stream)."""
        if self.world == 1:
            return
        t = grads.flat
        if t.device.type != "cuda":
            self.allreduce(t)
            t.mul_(1.0 / self.world)
            return
        if self.stream is None:
            self.stream = torch.cuda.Stream(device=t.device)
        ev = torch.cuda.Event()
        ev.record(stream if stream is not None else torch.cuda.current_stream(t.device))
        self.stream.wait_event(ev)
        with torch.cuda.stream(self.stream):
            self.allreduce(t)
            t.mul_(1.0 / self.world)
        self.pending += 1

    def finish(self, stream=None) -> None:
        """Makes `stream` (None: the current stream) wait for the exchanges."""
        if self.stream is not None and self.pending:
            (stream if stream is not None else torch.cuda.current_stream(self.stream.device)).wait_stream(self.stream)
        self.pending = 0
