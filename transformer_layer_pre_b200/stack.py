"""A stack of encoder layers run as one training step, with optional
Progressive Layer Dropping.

"DeepSpeed Transformer Kernel usage guide", Step 1: a model is a stack of
layer objects, one per encoder layer, each holding its own buffers; layer l
takes philox_offset = l so that every layer draws its own dropout bits
(the handle-level configuration of the C ABI).  "Progressive Layer Dropping"
page, schedule section: at global step t the keep level is
theta(t) = (1 - theta_bar) exp(-gamma t) + theta_bar and each layer runs or is
skipped (the identity in forward and backward) by a seeded draw whose keep
probability falls linearly with depth to theta(t) at the last layer; the
decisions come from the library (tl_pld_keep), equal on every rank that
shares the seed and the step.  A skipped layer gets no gradients (None).

Every layer's output and input gradient live in buffers of their own, so
the inputs each layer's backward needs stay valid through the step.  The
layers' per-call scratch (Step 3's memory concern: what lives only within
one layer's forward or backward) is one buffer shared by all of them, since
they run one at a time (share_scratch=False gives each its own).

Data parallelism: with a process group of size > 1, `backward(...,
exchange=True)` averages each layer's gradients over the ranks as soon as
that layer's backward is enqueued, on a side stream, so the collective
overlaps the backward of the layers below it (one bucket per layer, the
layer's flat float32 gradient buffer).
"""
from __future__ import annotations

import torch

from . import Layer, pld_keep, pld_theta
from .dp import FlatGrads, GradExchanger


class EncoderStack:
    """`num_layers` layers of one configuration (see Layer for the arguments)."""

    def __init__(self, num_layers: int, batch: int, seq: int, hidden: int, heads: int, ffn: int = 0,
                 attn_dropout: float = 0.0, hidden_dropout: float = 0.0, pre_layer_norm: bool = True,
                 seed: int = 1234, dtype=torch.float16, device=None, **options):
        if num_layers <= 0:
            raise ValueError("a stack needs at least one layer")
        self.num_layers, self.seed = num_layers, seed
        self.shape = (batch, seq, hidden)
        self.dtype = dtype
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.normalize_invertible = bool(options.get("normalize_invertible", False))
        self.pre_layer_norm = pre_layer_norm
        share = bool(options.pop("share_scratch", True))
        self.layers = [Layer(batch, seq, hidden, heads, ffn, attn_dropout, hidden_dropout, pre_layer_norm, seed,
                             dtype=dtype, philox_offset=l, **options) for l in range(num_layers)]
        # the layers run one at a time on one stream: one scratch serves them all
        self.scratch = None
        if share and num_layers > 1:
            need = max(layer.scratch_bytes for layer in self.layers)
            self.scratch = torch.empty(need, dtype=torch.uint8, device=self.device)
            for layer in self.layers:
                layer.share_scratch(self.scratch)
        self.ffn = self.layers[0].ffn
        self.grads = [FlatGrads(hidden, self.ffn, self.device) for _ in range(num_layers)]
        self.ys = [torch.empty(self.shape, dtype=dtype, device=self.device) for _ in range(num_layers)]
        self.dxs = [torch.empty(self.shape, dtype=dtype, device=self.device) for _ in range(num_layers)]
        self.inputs: list = [None] * num_layers
        self.dys: list = [None] * num_layers
        self.keep: list = [True] * num_layers

    def set_step(self, step: int) -> None:
        """Dropout masks of global step `step`: layer l draws with
        philox_offset = step * num_layers + l (step 0 is the construction's
        offset l), so no two (step, layer) pairs share masks."""
        for l, layer in enumerate(self.layers):
            layer.set_rng(self.seed, step * self.num_layers + l)

    def keep_decisions(self, step: int, theta_bar: float, gamma: float) -> list:
        """Progressive Layer Dropping: which layers run at global step `step`."""
        theta = pld_theta(theta_bar, gamma, step)
        return [pld_keep(self.seed, step, l, self.num_layers, theta) for l in range(self.num_layers)]

    def forward(self, x: torch.Tensor, mask, weights: list, keep: list | None = None, stream=None) -> torch.Tensor:
        """Runs the kept layers in order; returns the stack's output (x itself
        when every layer is skipped).  weights[l] is layer l's weight dict."""
        if len(weights) != self.num_layers:
            raise ValueError("one weight dict per layer")
        self.keep = [True] * self.num_layers if keep is None else [bool(k) for k in keep]
        if len(self.keep) != self.num_layers:
            raise ValueError("one keep decision per layer")
        h = x
        for l, layer in enumerate(self.layers):
            self.inputs[l] = h
            if self.keep[l]:
                h = layer.forward(h, mask, weights[l], y=self.ys[l], stream=stream)
        return h

    def backward(self, dy: torch.Tensor, weights: list, exchange=False, stream=None):
        """Backward of the last forward, layers in reverse.  Returns (dx,
        grads) with grads[l] a dict of float32 gradients (views of the stack's
        per-layer flat buffer, overwritten by the next backward) for a layer
        that ran and None for a skipped one.  With `exchange`, each layer's
        gradients are averaged over the data-parallel ranks (see the module
        docstring); they are final once the caller's stream reaches the end
        of this call's work.  `exchange` may also be a GradExchanger to use
        (e.g. one with its own collective)."""
        out = [None] * self.num_layers
        ex = exchange if isinstance(exchange, GradExchanger) else (GradExchanger() if exchange else None)
        g = dy
        for l in reversed(range(self.num_layers)):
            self.dys[l] = g
            if not self.keep[l]:
                continue
            x_in = None if (self.normalize_invertible and self.pre_layer_norm) else self.inputs[l]
            g, out[l] = self.layers[l].backward(x_in, g, weights[l], grads=self.grads[l].as_dict(), dx=self.dxs[l],
                                                stream=stream)
            if ex is not None:
                ex.submit(self.grads[l], stream)
        if ex is not None:
            ex.finish(stream)
        return g, out

    @property
    def workspace_bytes(self) -> int:
        """Device bytes the stack's layers hold, the shared scratch included."""
        shared = 0 if self.scratch is None else self.scratch.numel()
        return sum(layer.workspace_bytes for layer in self.layers) + shared

    def close(self) -> None:
        for layer in self.layers:
            layer.close()
