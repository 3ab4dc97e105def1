"""Shared helpers of the parity tests: run the CUDA layer through the C ABI
and the oracle on the same seeded inputs, and compare with the stated bars.

Bars (what the layer must meet against the float64 oracle):
  * float32 storage: max|gpu - oracle| / max|oracle| <= 1e-5 per tensor;
  * float16 / bfloat16 storage: relative Frobenius error <= 1e-2 against the
    pure float64 oracle for every tensor, and a max-abs bar of 2e-2 against
    the oracle in storage-rounded mode (float64 arithmetic, rounded to the
    storage type where the CUDA path stores a tensor):
      - y and dx (unit-scale tensors): max |gpu - oracle| <= 2e-2 plus two
        units in the last place of their own 16-bit storage at the value: one
        for the output's own rounding and one for a one-unit flip of the
        stored tensor that feeds the last step (a residual sum or a LayerNorm
        input of similar magnitude).  Both sides round values that can fall
        on either side of a rounding boundary; for bfloat16 magnitudes >= 4
        one such unit, 2^-5, exceeds 2e-2 by itself;
      - weight and bias gradients (float32 sums over all T tokens, whose
        magnitude and rounding noise grow like sqrt(T)): max |gpu - oracle|
        <= 2e-2 * max(1, max |oracle|), i.e. the bar relative to the
        tensor's own scale.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from transformer_layer_pre_b200 import Layer, WEIGHT_NAMES
from transformer_layer_pre_b200.synthetic import Inputs, Workload, to_f64

TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
ULP_BITS = {"f16": 10, "bf16": 7}


def oracle_config(w: Workload, batch: int, philox_offset: int = 0) -> oracle.LayerConfig:
    return oracle.LayerConfig(batch=batch, seq=w.seq, hidden=w.hidden, heads=w.heads, ffn=w.ffn,
                              attn_dropout=float(np.float32(w.attn_dropout)),
                              hidden_dropout=float(np.float32(w.hidden_dropout)),
                              pre_layer_norm=w.pre_layer_norm, seed=w.seed, philox_offset=philox_offset,
                              storage=w.dtype, gelu_form=w.gelu)


def run_gpu(inp: Inputs, layer: int = 0, gelu_checkpoint: bool | None = None, normalize_invertible=False,
            philox_offset: int = 0, keep_x: bool = True) -> dict:
    """Forward + backward of one layer on cuda:0; returns float64 numpy arrays."""
    w = inp.workload
    b = inp.x.shape[0]
    dev = torch.device("cuda", 0)
    ck = w.gelu_checkpoint if gelu_checkpoint is None else gelu_checkpoint
    L = Layer(b, w.seq, w.hidden, w.heads, w.ffn, w.attn_dropout, w.hidden_dropout, w.pre_layer_norm, w.seed,
              dtype=TORCH_DT[w.dtype], philox_offset=philox_offset, gelu_checkpoint=ck,
              normalize_invertible=normalize_invertible, gelu_tanh=w.gelu == "tanh")
    try:
        wt = {n: inp.weights[layer][n].to(dev) for n in WEIGHT_NAMES}
        x = inp.x.to(dev)
        dy = inp.dy.to(dev)
        mask = None if inp.mask is None else inp.mask.to(dev)
        y = L.forward(x, mask, wt)
        dx, g = L.backward(x if keep_x else None, dy, wt)
        torch.cuda.synchronize()
        out = dict(y=to_f64(y.cpu()), dx=to_f64(dx.cpu()),
                   grads={n: g[n].cpu().double().numpy() for n in WEIGHT_NAMES})
    finally:
        L.close()
    return out


def run_oracle(inp: Inputs, layer: int = 0, storage_rounded: bool = False, seq_index=None,
               philox_offset: int = 0) -> dict:
    w = inp.workload
    b = inp.x.shape[0]
    idx = np.arange(b) if seq_index is None else np.asarray(seq_index)
    cfg = oracle_config(w, b, philox_offset)
    mask = None if inp.mask is None else to_f64(inp.mask)[idx]
    wt = {n: to_f64(inp.weights[layer][n]) for n in WEIGHT_NAMES}
    return oracle.layer_forward_backward(cfg, to_f64(inp.x)[idx], mask, wt, to_f64(inp.dy)[idx],
                                         seq_index=idx, storage_rounded=storage_rounded)


def ulp(ref: np.ndarray, dtype: str) -> np.ndarray:
    """One unit in the last place of `dtype` at each reference value."""
    if dtype not in ULP_BITS:
        return np.zeros_like(ref)
    _, e = np.frexp(np.abs(ref))
    return np.ldexp(1.0, e - 1 - ULP_BITS[dtype])


def errors(gpu: np.ndarray, pure: np.ndarray, rounded: np.ndarray | None, dtype: str, stored: bool) -> dict:
    gpu, pure = np.asarray(gpu), np.asarray(pure)
    assert gpu.shape == pure.shape
    assert np.all(np.isfinite(gpu)), "non-finite values"
    out = {"rel_max": float(np.abs(gpu - pure).max() / max(np.abs(pure).max(), 1e-300)),
           "rel_frob": float(np.linalg.norm(gpu - pure) / max(np.linalg.norm(pure), 1e-300))}
    if rounded is not None:
        d = np.abs(gpu - rounded)
        out["max_abs"] = float(d.max())
        if stored:
            allow = 2e-2 + 2.0 * ulp(rounded, dtype)
        else:
            allow = 2e-2 * max(1.0, float(np.abs(rounded).max()))
        out["excess"] = float((d - allow).max())
    return out


def check_tensor(name: str, gpu, pure, rounded, dtype: str, stored: bool) -> dict:
    e = errors(gpu, pure, rounded, dtype, stored)
    if dtype == "f32":
        assert e["rel_max"] <= 1e-5, (name, e)
    else:
        assert e["rel_frob"] <= 1e-2, (name, e)
        assert e["excess"] <= 0.0, (name, e)
    return e


def check_layer(gpu: dict, pure: dict, rounded: dict | None, dtype: str) -> dict:
    report = {}
    for k in ("y", "dx"):
        report[k] = check_tensor(k, gpu[k], pure[k], None if rounded is None else rounded[k], dtype, True)
    for n in WEIGHT_NAMES:
        report[n] = check_tensor(n, gpu["grads"][n], pure["grads"][n],
                                 None if rounded is None else rounded["grads"][n], dtype, False)
    return report
