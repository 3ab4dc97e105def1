"""layer_set_rng: the dropout generator's key and 4th counter word change
between steps without a reallocation, and a backward keeps the masks of the
forward before it.  Compared bitwise with layers created with those values
(whose masks the oracle pins in test_gpu_parity and test_gpu_dropout)."""
import numpy as np
import pytest
import torch

from parity import TORCH_DT
from transformer_layer_pre_b200 import Layer, WEIGHT_NAMES
from transformer_layer_pre_b200.synthetic import Workload, make_inputs

pytestmark = pytest.mark.gpu

W = Workload("rng-f16", 2, 128, 128, 2, 256, "f16", 0.1, 0.1, lengths=(90, 128))


def _step(inp, seed, offset, rng_before_fwd=None, rng_before_bwd=None):
    w = inp.workload
    dev = torch.device("cuda", 0)
    L = Layer(w.batch, w.seq, w.hidden, w.heads, w.ffn, w.attn_dropout, w.hidden_dropout, w.pre_layer_norm, seed,
              dtype=TORCH_DT[w.dtype], philox_offset=offset)
    try:
        wt = {n: inp.weights[0][n].to(dev) for n in WEIGHT_NAMES}
        x, dy = inp.x.to(dev), inp.dy.to(dev)
        mask = None if inp.mask is None else inp.mask.to(dev)
        if rng_before_fwd:
            L.set_rng(*rng_before_fwd)
        y = L.forward(x, mask, wt)
        if rng_before_bwd:
            L.set_rng(*rng_before_bwd)
        dx, g = L.backward(x, dy, wt)
        torch.cuda.synchronize()
        return [y.cpu().float().numpy(), dx.cpu().float().numpy()] + [g[n].cpu().numpy() for n in WEIGHT_NAMES]
    finally:
        L.close()


def _same(a, b):
    return all(np.array_equal(u, v) for u, v in zip(a, b))


def test_set_rng_before_forward_equals_a_layer_created_with_it():
    inp = make_inputs(W)
    moved = _step(inp, W.seed, 0, rng_before_fwd=(W.seed + 17, 5))
    fresh = _step(inp, W.seed + 17, 5)
    assert _same(moved, fresh)
    assert not np.array_equal(moved[0], _step(inp, W.seed, 0)[0])   # other masks


def test_backward_keeps_the_masks_of_its_forward():
    inp = make_inputs(W)
    plain = _step(inp, W.seed, 3)
    changed = _step(inp, W.seed, 3, rng_before_bwd=(W.seed + 1, 4))
    assert _same(plain, changed)


def test_stack_set_step_gives_each_layer_its_own_offset():
    import ctypes
    import transformer_layer_pre_b200 as tlp
    from transformer_layer_pre_b200.stack import EncoderStack
    st = EncoderStack(3, 1, 64, 128, 2, 256, 0.1, 0.1, True, seed=5, dtype=torch.float16)
    try:
        def offsets():
            out = []
            for layer in st.layers:
                opt = tlp.Options()
                assert layer.lib.layer_get_options(layer.handle, ctypes.byref(opt)) == 0
                out.append(opt.philox_offset)
            return out
        assert offsets() == [0, 1, 2]
        st.set_step(4)
        assert offsets() == [12, 13, 14]
    finally:
        st.close()
