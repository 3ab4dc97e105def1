"""The relaxed-determinism option (tl_options.stochastic_mode; "DeepSpeed
Transformer Kernel usage guide", Step 2: faster, not reproducible run to run).

With it the backward adds the column sums of the bias and LayerNorm
gradients, and the split-K partials of a weight gradient whose K is split,
straight into the gradient outputs with float32 atomics instead of summing
them in a fixed order in a closing launch.  So:
  * against the oracle it meets the same bars as the default mode;
  * y, dx and every gradient that is not such a sum are bitwise the same as
    in the default mode;
  * the summed gradients differ from the default mode's only by float32
    summation order (a dropped or doubled partial row would move them by
    several percent of their largest entry, far above the bound used here).
"""
import dataclasses

import numpy as np
import pytest

from parity import check_layer, run_gpu, run_oracle
from transformer_layer_pre_b200.synthetic import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

# gradients a stochastic-mode backward sums with atomics (dWo: its K = tokens
# is split across CTA pairs at BERT-Large from 1024 tokens up)
SUMMED = ("bqkv", "bo", "ln1_g", "ln1_b", "b1", "b2", "ln2_g", "ln2_b")
SPLIT_K_LARGE = ("wo",)

MULTITILE_F16 = Workload("multitile-f16", 2, 200, 128, 2, 256, "f16", 0.1, 0.1, lengths=(150, 200))
RAGGED_POST_BF16 = Workload("ragged-post-bf16", 2, 40, 128, 2, 264, "bf16", 0.1, 0.1, pre_layer_norm=False,
                            lengths=(17, 40))
RAGGED_F32 = Workload("ragged-f32", 2, 24, 96, 6, 200, "f32", 0.1, 0.2, lengths=(9, 24))


def _against_oracle(w: Workload, batch=None, **kw):
    inp = make_inputs(w, batch=batch)
    gpu = run_gpu(inp, stochastic_mode=True, **kw)
    pure = run_oracle(inp)
    rounded = None if w.dtype == "f32" else run_oracle(inp, storage_rounded=True)
    check_layer(gpu, pure, rounded, w.dtype)
    return inp, gpu


def _against_default(inp, relaxed: dict, summed, **kw):
    det = run_gpu(inp, **kw)
    assert np.array_equal(det["y"], relaxed["y"])
    assert np.array_equal(det["dx"], relaxed["dx"])
    for n, a in det["grads"].items():
        b = relaxed["grads"][n]
        if n in summed:
            # float32 sums of at most a few hundred partial rows in another order
            bound = 1e-4 * float(np.max(np.abs(a))) + 1e-6
            assert float(np.max(np.abs(a - b))) <= bound, n
        else:
            assert np.array_equal(a, b), n


@pytest.mark.parametrize("w", [MULTITILE_F16, RAGGED_POST_BF16, RAGGED_F32], ids=lambda w: w.name)
def test_stochastic_mode_matches_oracle_and_default(w):
    inp, gpu = _against_oracle(w)
    _against_default(inp, gpu, SUMMED)


def test_stochastic_mode_gelu_checkpoint():
    w = dataclasses.replace(MULTITILE_F16, gelu_checkpoint=True)
    inp, gpu = _against_oracle(w)
    _against_default(inp, gpu, SUMMED)


def test_stochastic_mode_split_k_weight_gradient_bert_large_batch16():
    """2048 tokens: the dWo GEMM splits K four ways, each split adding its
    tiles into the gradient by TMA reduce-add."""
    inp, gpu = _against_oracle(WORKLOADS["bert-large-f16"], batch=16)
    _against_default(inp, gpu, SUMMED + SPLIT_K_LARGE)


def test_stochastic_mode_full_batch_bert_large_against_default():
    """The benchmarked workload (B64 S128 H1024 fp16) in both modes."""
    inp = make_inputs(WORKLOADS["bert-large-f16"])
    relaxed = run_gpu(inp, stochastic_mode=True)
    _against_default(inp, relaxed, SUMMED + SPLIT_K_LARGE)
