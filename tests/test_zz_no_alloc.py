"""The allocation-free bias-gradient entry point (tl_bias_grad_noalloc).

It serves callers that cannot allocate device memory: its partial sums live
in a fixed array inside the library.  Its result must equal what the
existing entry point computes for the same quantity: layer_backward's
gradient of the FFN output bias, which in pre-LN form with hidden dropout 0
is the column sum of dY; and it must equal that column sum computed in
float64 on the host from the stored dY.  Two calls in a row check that the shared array's
leftover contents do not leak into the next result.  This file is collected
last so that a run stopping at its first failure has run everything else.
"""
import ctypes

import numpy as np
import pytest
import torch

import transformer_layer_pre_b200 as tlp

pytestmark = pytest.mark.gpu

TL_OK, TL_EINVAL = 0, 1


def _layer_b2(dtype, x, dy, w, B, S, H, F):
    layer = tlp.Layer(B, S, H, H // 64, F, 0.1, 0.0, True, 1234, dtype=dtype)
    try:
        layer.forward(x, None, w)
        _, g = layer.backward(x, dy, w)
        torch.cuda.synchronize()
        return g["b2"].clone()
    finally:
        layer.close()


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_noalloc_bias_grad_matches_layer_backward(dtype):
    lib = tlp.load_library()
    dev = torch.device("cuda", 0)
    B, S, H, F = 4, 128, 512, 1024
    gen = torch.Generator().manual_seed(7)
    w = {n: (torch.randn(s, generator=gen) * 0.02) for n, s in [
        ("wqkv", (3 * H, H)), ("bqkv", (3 * H,)), ("wo", (H, H)), ("bo", (H,)), ("w1", (F, H)), ("b1", (F,)),
        ("w2", (H, F)), ("b2", (H,))]}
    w.update(ln1_g=torch.ones(H), ln1_b=torch.zeros(H), ln2_g=torch.ones(H), ln2_b=torch.zeros(H))
    w = {n: v.to(dtype).to(dev) for n, v in w.items()}
    x = torch.randn(B, S, H, generator=gen).to(dtype).to(dev)
    code = tlp.DTYPE_CODES[dtype]
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        dy = (torch.randn(B, S, H, generator=gen) * (1.0 + call)).to(dtype).to(dev)
        ref = _layer_b2(dtype, x, dy, w, B, S, H, F)
        out = torch.full((H,), float("nan"), dtype=torch.float32, device=dev)
        st = lib.tl_bias_grad_noalloc(code, ctypes.c_void_p(dy.data_ptr()), B * S, H,
                                      ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(stream))
        assert st == TL_OK
        torch.cuda.synchronize()
        a, r = out.double().cpu().numpy(), ref.double().cpu().numpy()
        assert np.all(np.isfinite(a))
        assert np.abs(a - r).max() <= 1e-5 * max(1.0, np.abs(r).max()), (call, np.abs(a - r).max())
        # and the column sum itself, in float64 on the host from the stored values
        exact = dy.double().cpu().numpy().reshape(B * S, H).sum(axis=0)
        assert np.abs(a - exact).max() <= 1e-5 * max(1.0, np.abs(exact).max()), (call, np.abs(a - exact).max())


def test_noalloc_rejects_sizes_beyond_its_array():
    lib = tlp.load_library()
    dev = torch.device("cuda", 0)
    dz = torch.zeros(16, 8200, dtype=torch.float16, device=dev)
    out = torch.zeros(8200, dtype=torch.float32, device=dev)
    st = lib.tl_bias_grad_noalloc(1, ctypes.c_void_p(dz.data_ptr()), 16, 8200, ctypes.c_void_p(out.data_ptr()), None)
    assert st == TL_EINVAL
