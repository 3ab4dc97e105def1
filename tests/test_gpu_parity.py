"""Parity of the CUDA layer (through the C ABI) with the float64 oracle on
the same seeded inputs, element by element.

Cases: the tiny float32 layer; ragged shapes (token counts, widths and FFN
sizes that are not multiples of any tile) in both layer orders; the
BERT-base bf16 workload at full size; the BERT-Large fp16 workload at a
reduced batch and at its full batch of 64 (every gradient); the
long-sequence post-LN bf16 workload at batch 1 and, on sampled sequences,
at its full batch."""
import dataclasses

import numpy as np
import pytest
import torch

from parity import check_layer, run_gpu, run_oracle
from transformer_layer_pre_b200.synthetic import WORKLOADS, Workload, make_inputs, with_random_affine

pytestmark = pytest.mark.gpu

RAGGED_F16 = Workload("ragged-f16", 3, 72, 192, 3, 520, "f16", 0.1, 0.1, lengths=(40, 72))
RAGGED_POST_BF16 = Workload("ragged-post-bf16", 2, 40, 128, 2, 264, "bf16", 0.1, 0.1, pre_layer_norm=False,
                            lengths=(17, 40))
RAGGED_F32 = Workload("ragged-f32", 2, 24, 96, 6, 200, "f32", 0.1, 0.2, lengths=(9, 24))
# S = 96: whole 32-row output boxes, the last query quarter of the 128-row tile empty
RAGGED96_F16 = Workload("ragged96-f16", 3, 96, 128, 2, 256, "f16", 0.1, 0.1, lengths=(50, 96))
# sequences spanning two 128-key tiles with a ragged second tile
MULTITILE_F16 = Workload("multitile-f16", 2, 200, 128, 2, 256, "f16", 0.1, 0.1, lengths=(150, 200))
MULTITILE_POST_BF16 = Workload("multitile-post-bf16", 2, 264, 192, 3, 384, "bf16", 0.1, 0.1, pre_layer_norm=False,
                               lengths=(130, 264))


def _parity(w: Workload, batch=None, affine=False, **kw):
    inp = make_inputs(w, batch=batch)
    if affine:
        inp = with_random_affine(inp)
    gpu = run_gpu(inp, **kw)
    pure = run_oracle(inp)
    rounded = None if w.dtype == "f32" else run_oracle(inp, storage_rounded=True)
    return check_layer(gpu, pure, rounded, w.dtype)


def test_tiny_f32():
    _parity(WORKLOADS["tiny-f32"])


def test_ragged_f32_with_dropout_and_mask():
    _parity(RAGGED_F32)


def test_ragged_f16_pre_ln():
    _parity(RAGGED_F16)


def test_ragged96_f16_pre_ln():
    _parity(RAGGED96_F16)


def test_ragged_bf16_post_ln():
    _parity(RAGGED_POST_BF16)


def test_multitile_f16_pre_ln():
    _parity(MULTITILE_F16)


def test_multitile_bf16_post_ln():
    _parity(MULTITILE_POST_BF16)


def test_bert_base_bf16_full_size():
    _parity(WORKLOADS["bert-base-bf16"])


def test_bert_large_f16_batch4():
    _parity(WORKLOADS["bert-large-f16"], batch=4)


def test_long_post_ln_bf16_batch1():
    _parity(WORKLOADS["long-postln-bf16"], batch=1)


def test_gelu_checkpoint_is_bitwise_identical():
    w = dataclasses.replace(WORKLOADS["bert-large-stack-f16"], batch=2, seq=128, layers=1)
    inp = make_inputs(w)
    a = run_gpu(inp, gelu_checkpoint=False)
    b = run_gpu(inp, gelu_checkpoint=True)
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["dx"], b["dx"])
    for n in a["grads"]:
        assert np.array_equal(a["grads"][n], b["grads"][n]), n


def test_philox_offset_changes_masks_and_matches_oracle():
    w = dataclasses.replace(RAGGED_F16, batch=2)
    inp = make_inputs(w)
    gpu = run_gpu(inp, philox_offset=7)
    pure = run_oracle(inp, philox_offset=7)
    rounded = run_oracle(inp, storage_rounded=True, philox_offset=7)
    check_layer(gpu, pure, rounded, w.dtype)
    other = run_gpu(inp, philox_offset=0)
    assert not np.array_equal(gpu["y"], other["y"])


# Non-zero biases and LayerNorm parameters away from gamma = 1, beta = 0, so
# that every bias add and affine step of the forward is exercised.
def test_random_affine_f16_pre_ln():
    _parity(RAGGED_F16, affine=True)


def test_random_affine_bf16_post_ln():
    _parity(MULTITILE_POST_BF16, affine=True)


def test_random_affine_f32():
    _parity(RAGGED_F32, affine=True)


# normalize_invertible: LayerNorm backward from the LayerNorm output
# ("DeepSpeed Transformer Kernel usage guide", Step 3: the input of the
# normalisation is not kept; x-hat is recovered as (y - beta) / gamma).
def test_normalize_invertible_pre_ln_without_x():
    _parity(RAGGED_F16, affine=True, normalize_invertible=True, keep_x=False)


def test_normalize_invertible_pre_ln_multitile_bf16():
    w = dataclasses.replace(MULTITILE_F16, dtype="bf16", name="multitile-bf16")
    _parity(w, affine=True, normalize_invertible=True, keep_x=False)


def test_normalize_invertible_post_ln():
    _parity(MULTITILE_POST_BF16, affine=True, normalize_invertible=True)


def test_normalize_invertible_f32():
    _parity(RAGGED_F32, affine=True, normalize_invertible=True, keep_x=False)


def test_normalize_invertible_bert_large_batch2():
    _parity(WORKLOADS["bert-large-f16"], batch=2, affine=True, normalize_invertible=True, keep_x=False)


# GELU in its tanh approximation (tl_options.gelu_tanh) against the oracle's
# tanh form, forward and backward, and bitwise under gelu_checkpoint.
def test_gelu_tanh_f16_pre_ln():
    _parity(dataclasses.replace(RAGGED_F16, gelu="tanh"), affine=True)


def test_gelu_tanh_f32_post_ln():
    _parity(dataclasses.replace(RAGGED_F32, gelu="tanh", pre_layer_norm=False), affine=True)


def test_gelu_tanh_checkpoint_is_bitwise_identical():
    w = dataclasses.replace(RAGGED_F16, gelu="tanh")
    inp = make_inputs(w)
    a = run_gpu(inp, gelu_checkpoint=False)
    b = run_gpu(inp, gelu_checkpoint=True)
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["dx"], b["dx"])
    for n in a["grads"]:
        assert np.array_equal(a["grads"][n], b["grads"][n]), n


# Valid lengths that end well before the sequence does: the long-sequence
# attention kernels skip key tiles past the last unmasked key (forward,
# dQ) and write zero dK, dV for key tiles that hold only masked keys; the
# result must not change (2^-inf = 0 exactly).  Lengths 37 (one partly valid
# tile of three), 128 (exactly one tile), 129 (one key into the second) and
# 384 (no padding).
SHORT_LEN_F16 = Workload("short-lengths-f16", 4, 384, 128, 2, 256, "f16", 0.1, 0.1)


@pytest.mark.parametrize("pre_ln", [True, False])
def test_long_sequence_skips_padded_key_tiles_exactly(pre_ln):
    from transformer_layer_pre_b200.synthetic import make_mask
    w = dataclasses.replace(SHORT_LEN_F16, pre_layer_norm=pre_ln)
    inp = make_inputs(w)
    lengths = np.array([37, 128, 129, 384])
    inp = dataclasses.replace(inp, mask=make_mask(lengths, w.seq), lengths=lengths)
    gpu = run_gpu(inp)
    check_layer(gpu, run_oracle(inp), run_oracle(inp, storage_rounded=True), w.dtype)


def _sampled_full_size(w: Workload, idx):
    """Whole-batch run on the GPU at the workload's full size; y and dx of the
    sampled sequences against the oracle run on those sequences alone (their
    global indices fix their dropout bits)."""
    inp = make_inputs(w)
    gpu = run_gpu(inp)
    idx = np.asarray(idx)
    pure = run_oracle(inp, seq_index=idx)
    rounded = run_oracle(inp, storage_rounded=True, seq_index=idx)
    from parity import check_tensor
    check_tensor("y", gpu["y"][idx], pure["y"], rounded["y"], w.dtype, True)
    check_tensor("dx", gpu["dx"][idx], pure["dx"], rounded["dx"], w.dtype, True)


def test_bert_large_f16_full_batch_every_gradient():
    """The benchmarked workload itself (B64 S128 H1024, fp16, dropout 0.1;
    "DeepSpeed Transformer Kernel usage guide", Step 1's BERT-Large) at its
    full batch, in the launch configuration the benchmark times: y, dx and
    all twelve parameter gradients element by element against the oracle,
    pure and storage-rounded.  This is where the GEMM tile plans, the
    split-K weight gradients, the keep bits drawn by the idle CTA pairs of
    the QKV GEMM and the persistent attention's multi-round schedule run at
    the sizes the benchmark uses."""
    _parity(WORKLOADS["bert-large-f16"])


def test_long_post_ln_bf16_full_batch_sampled_sequences():
    _sampled_full_size(WORKLOADS["long-postln-bf16"], [1, 3])
