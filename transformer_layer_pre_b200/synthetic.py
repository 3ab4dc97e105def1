"""Seeded synthetic inputs for the encoder layer (no arithmetic of the layer).

The workloads are shaped like the BERT setups of the "DeepSpeed Transformer
Kernel usage guide" (Step 1: BERT-Large, 24 layers, hidden 1024, 16 heads,
sequence 128, batch 64).  No dataset is involved: weights are N(0, 0.02)
(initializer_range, Step 2), biases 0, LayerNorm gamma 1 / beta 0, the layer
input x and the upstream gradient dY are N(0, 1), and padded workloads draw
each sequence's valid length uniformly from a range; keys beyond it get an
additive -inf mask.

Draw order (numpy PCG64, one generator per workload): for each layer wqkv,
wo, w1, w2 (biases are zeros and draw nothing), then x, then dY, then the
valid lengths.  Values are drawn in float64 and rounded to the storage dtype;
both the CUDA path and the oracle consume the same rounded values.
"""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
WEIGHT_NAMES = (
    "wqkv", "bqkv", "wo", "bo", "ln1_g", "ln1_b",
    "w1", "b1", "w2", "b2", "ln2_g", "ln2_b",
)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seq: int
    hidden: int
    heads: int
    ffn: int
    dtype: str            # 'f32' | 'f16' | 'bf16'
    attn_dropout: float
    hidden_dropout: float
    pre_layer_norm: bool = True
    lengths: tuple | None = None   # (lo, hi) valid-length range, None = no padding
    layers: int = 1
    gelu_checkpoint: bool = False
    seed: int = 1234
    gelu: str = "erf"              # 'erf' | 'tanh' (the approximation)

    @property
    def tokens(self) -> int:
        return self.batch * self.seq


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny-f32", 2, 16, 64, 4, 256, "f32", 0.0, 0.0),
        Workload("bert-base-bf16", 8, 128, 768, 12, 3072, "bf16", 0.1, 0.1, lengths=(64, 128)),
        Workload("bert-large-f16", 64, 128, 1024, 16, 4096, "f16", 0.1, 0.1),
        Workload("bert-large-stack-f16", 16, 512, 1024, 16, 4096, "f16", 0.1, 0.1,
                 lengths=(256, 512), layers=24, gelu_checkpoint=True),
        Workload("long-postln-bf16", 4, 2048, 1024, 16, 4096, "bf16", 0.1, 0.1,
                 pre_layer_norm=False, lengths=(1024, 2048)),
    ]
}


@dataclasses.dataclass
class Inputs:
    workload: Workload
    weights: list          # one dict name -> CPU tensor (storage dtype) per layer
    x: torch.Tensor        # (B, S, H) storage dtype, CPU
    dy: torch.Tensor       # (B, S, H) storage dtype, CPU
    mask: torch.Tensor | None   # (B, S) float32 additive, CPU
    lengths: np.ndarray | None


def _store(a: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DTYPES[dtype])


def make_weights(rng: np.random.Generator, h: int, f: int, dtype: str, std: float = 0.02) -> dict:
    w = {
        "wqkv": rng.normal(0.0, std, (3 * h, h)),
        "wo": rng.normal(0.0, std, (h, h)),
        "w1": rng.normal(0.0, std, (f, h)),
        "w2": rng.normal(0.0, std, (h, f)),
    }
    w.update(bqkv=np.zeros(3 * h), bo=np.zeros(h), b1=np.zeros(f), b2=np.zeros(h),
             ln1_g=np.ones(h), ln1_b=np.zeros(h), ln2_g=np.ones(h), ln2_b=np.zeros(h))
    return {n: _store(w[n], dtype) for n in WEIGHT_NAMES}


def make_mask(lengths: np.ndarray, seq: int) -> torch.Tensor:
    pos = np.arange(seq)[None, :]
    m = np.where(pos < lengths[:, None], 0.0, -np.inf).astype(np.float32)
    return torch.from_numpy(m)


def make_inputs(w: Workload, batch: int | None = None, seed: int | None = None,
                layers: int | None = None) -> Inputs:
    """Draws one workload's inputs; `batch` / `layers` override the sizes for
    reduced cases (the draw order is unchanged)."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    b = w.batch if batch is None else batch
    nl = w.layers if layers is None else layers
    weights = [make_weights(rng, w.hidden, w.ffn, w.dtype) for _ in range(nl)]
    x = _store(rng.normal(0.0, 1.0, (b, w.seq, w.hidden)), w.dtype)
    dy = _store(rng.normal(0.0, 1.0, (b, w.seq, w.hidden)), w.dtype)
    lengths = mask = None
    if w.lengths is not None:
        lengths = rng.integers(w.lengths[0], w.lengths[1] + 1, b)
        mask = make_mask(lengths, w.seq)
    return Inputs(w, weights, x, dy, mask, lengths)


def with_random_affine(inp: Inputs, seed: int = 4321, bias_std: float = 0.02) -> Inputs:
    """A copy of `inp` whose biases are N(0, bias_std) and whose LayerNorm
    parameters are gamma = 1 + N(0, 0.1), beta = N(0, 0.1) (so that no
    parameter takes its neutral value); drawn from a separate generator, per
    layer in the order bqkv, bo, b1, b2, ln1_g, ln1_b, ln2_g, ln2_b."""
    rng = np.random.default_rng(seed)
    dt = inp.workload.dtype
    out = []
    for w in inp.weights:
        w = dict(w)
        for n in ("bqkv", "bo", "b1", "b2"):
            w[n] = _store(rng.normal(0.0, bias_std, tuple(w[n].shape)), dt)
        for n in ("ln1", "ln2"):
            h = tuple(w[n + "_g"].shape)
            w[n + "_g"] = _store(1.0 + rng.normal(0.0, 0.1, h), dt)
            w[n + "_b"] = _store(rng.normal(0.0, 0.1, h), dt)
        out.append(w)
    return dataclasses.replace(inp, weights=out)


def to_f64(t: torch.Tensor | None) -> np.ndarray | None:
    """The exact values of a stored tensor, widened to float64."""
    return None if t is None else t.to(torch.float64).numpy()
