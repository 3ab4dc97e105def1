"""A stack of layers on the GPU (through the C ABI, one handle per layer,
philox_offset = layer id, GELU recomputed in backward) against the oracle's
stack, with Progressive Layer Dropping skipping layers; and the 24-layer
BERT-Large stack at full size (B16, S512, fp16, padded), checked per layer on
sampled sequences at layers 0, 11 and 23."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from parity import TORCH_DT, check_tensor, oracle_config
from transformer_layer_pre_b200 import WEIGHT_NAMES
from transformer_layer_pre_b200.stack import EncoderStack
from transformer_layer_pre_b200.synthetic import WORKLOADS, Workload, make_inputs, to_f64, with_random_affine

pytestmark = pytest.mark.gpu

SMALL_STACK = Workload("small-stack-f16", 2, 128, 256, 4, 1024, "f16", 0.1, 0.1, lengths=(64, 128), layers=4,
                       gelu_checkpoint=True)


def _run_stack(inp, keep, **options):
    w = inp.workload
    dev = torch.device("cuda", 0)
    st = EncoderStack(w.layers, inp.x.shape[0], w.seq, w.hidden, w.heads, w.ffn, w.attn_dropout, w.hidden_dropout,
                      w.pre_layer_norm, w.seed, dtype=TORCH_DT[w.dtype], gelu_checkpoint=w.gelu_checkpoint,
                      **options)
    try:
        wts = [{n: inp.weights[l][n].to(dev) for n in WEIGHT_NAMES} for l in range(w.layers)]
        mask = None if inp.mask is None else inp.mask.to(dev)
        y = st.forward(inp.x.to(dev), mask, wts, keep=keep)
        dx, grads = st.backward(inp.dy.to(dev), wts)
        torch.cuda.synchronize()
        return dict(y=to_f64(y.cpu()), dx=to_f64(dx.cpu()),
                    grads=[None if g is None else {n: g[n].cpu().double().numpy() for n in WEIGHT_NAMES}
                           for g in grads])
    finally:
        st.close()


def _oracle_stack(inp, keep, storage_rounded):
    w = inp.workload
    cfg = oracle_config(w, inp.x.shape[0])
    ws = [{n: to_f64(inp.weights[l][n]) for n in WEIGHT_NAMES} for l in range(w.layers)]
    mask = None if inp.mask is None else to_f64(inp.mask)
    return oracle.stack_forward_backward(cfg, to_f64(inp.x), mask, ws, to_f64(inp.dy), keep,
                                         storage_rounded=storage_rounded)


@pytest.mark.parametrize("keep", [[True, True, True, True], [True, False, True, False]])
def test_small_stack_with_skipped_layers(keep):
    inp = with_random_affine(make_inputs(SMALL_STACK))
    gpu = _run_stack(inp, keep)
    pure = _oracle_stack(inp, keep, False)
    rnd = _oracle_stack(inp, keep, True)
    check_tensor("y", gpu["y"], pure["y"], rnd["y"], "f16", True)
    check_tensor("dx", gpu["dx"], pure["dx"], rnd["dx"], "f16", True)
    for l in range(SMALL_STACK.layers):
        assert (gpu["grads"][l] is None) == (not keep[l])
        if keep[l]:
            for n in WEIGHT_NAMES:
                check_tensor(f"{n}[{l}]", gpu["grads"][l][n], pure["grads"][l][n], rnd["grads"][l][n], "f16", False)


def test_stack_keep_decisions_follow_the_schedule():
    inp = make_inputs(dataclasses.replace(SMALL_STACK, layers=2), batch=1)
    w = inp.workload
    st = EncoderStack(4, 1, w.seq, w.hidden, w.heads, w.ffn, seed=77)
    try:
        for step in (0, 10, 500, 4000):
            th = oracle.pld_theta(0.5, 0.001, step)
            assert st.keep_decisions(step, 0.5, 0.001) == [oracle.pld_keep(77, step, l, 4, th) for l in range(4)]
        assert st.keep_decisions(0, 0.5, 0.001) == [True] * 4
    finally:
        st.close()


def test_all_layers_skipped_is_the_identity():
    inp = make_inputs(dataclasses.replace(SMALL_STACK, layers=2), batch=1)
    gpu = _run_stack(inp, [False, False])
    assert np.array_equal(gpu["y"], to_f64(inp.x)) and np.array_equal(gpu["dx"], to_f64(inp.dy))
    assert gpu["grads"] == [None, None]


def test_bert_large_stack_full_size_sampled_layers():
    """24 layers at B16 S512 fp16 with padding and GELU recompute: every
    layer's forward output and input gradient on two sampled sequences at
    layers 0, 11 and 23, against the oracle run on the GPU stack's own input
    and upstream gradient of that layer (float64, the sequences' global
    indices fixing their dropout bits)."""
    w = WORKLOADS["bert-large-stack-f16"]
    inp = make_inputs(w)
    dev = torch.device("cuda", 0)
    st = EncoderStack(w.layers, w.batch, w.seq, w.hidden, w.heads, w.ffn, w.attn_dropout, w.hidden_dropout,
                      w.pre_layer_norm, w.seed, dtype=TORCH_DT[w.dtype], gelu_checkpoint=True)
    try:
        wts = [{n: inp.weights[l][n].to(dev) for n in WEIGHT_NAMES} for l in range(w.layers)]
        mask = inp.mask.to(dev)
        st.forward(inp.x.to(dev), mask, wts)
        st.backward(inp.dy.to(dev), wts)
        torch.cuda.synchronize()
        idx = np.array([3, 12])
        for l in (0, 11, 23):
            x_l = to_f64(st.inputs[l].cpu())[idx]
            dy_l = to_f64(st.dys[l].cpu())[idx]
            y_gpu = to_f64(st.ys[l].cpu())[idx]
            dx_gpu = to_f64(st.dxs[l].cpu())[idx]
            cfg = dataclasses.replace(oracle_config(w, len(idx)), philox_offset=l)
            wl = {n: to_f64(inp.weights[l][n]) for n in WEIGHT_NAMES}
            m = to_f64(inp.mask)[idx]
            pure = oracle.layer_forward_backward(cfg, x_l, m, wl, dy_l, seq_index=idx)
            rnd = oracle.layer_forward_backward(cfg, x_l, m, wl, dy_l, seq_index=idx, storage_rounded=True)
            check_tensor(f"y[{l}]", y_gpu, pure["y"], rnd["y"], "f16", True)
            check_tensor(f"dx[{l}]", dx_gpu, pure["dx"], rnd["dx"], "f16", True)
    finally:
        st.close()
