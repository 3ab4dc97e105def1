"""Dropout masks are bit-exact against the oracle's Philox contract.

1. The library's own device Philox (tl_dropout_keep_mask) against the oracle.
2. Through the whole layer: weights chosen so that the layer output exposes
   the keep bits of each dropout site exactly (the hidden sites through
   constant biases, the attention site through uniform attention
   probabilities over one-hot value vectors)."""
import numpy as np
import pytest
import torch

import oracle
from transformer_layer_pre_b200 import Layer, WEIGHT_NAMES, dropout_keep_mask

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seed,offset,site,p", [
    (1234, 0, 0, 0.1), (1234, 5, 1, 0.1), (0xDEADBEEFCAFEF00D, 23, 2, 0.3), (7, 1 << 31, 0, 0.5)])
def test_device_philox_matches_oracle(seed, offset, site, p):
    p32 = float(np.float32(p))
    for e0 in (0, (1 << 35) + 8 * 977):
        n = 1 << 20
        gpu = dropout_keep_mask(seed, offset, site, p32, e0, n).cpu().numpy().astype(bool)
        ref = oracle.dropout_keep(e0, n, site, offset, seed, p32)
        assert np.array_equal(gpu, ref)


def _zero_weights(h, f, dtype, dev):
    z = lambda *s: torch.zeros(*s, dtype=dtype, device=dev)
    return dict(wqkv=z(3 * h, h), bqkv=z(3 * h), wo=z(h, h), bo=z(h), ln1_g=torch.ones(h, dtype=dtype, device=dev),
                ln1_b=z(h), w1=z(f, h), b1=z(f), w2=z(h, f), b2=z(h), ln2_g=torch.ones(h, dtype=dtype, device=dev),
                ln2_b=z(h))


@pytest.mark.parametrize("dtype,B,S,H,heads,F", [
    (torch.float16, 2, 64, 256, 4, 512), (torch.bfloat16, 2, 64, 256, 4, 512), (torch.float32, 2, 64, 256, 4, 512),
    # BERT-Large shape: the QKV GEMM has CTA pairs without a tile in its last
    # round, which draw the keep bits of sites 1 and 2
    (torch.float16, 64, 128, 1024, 16, 1024)])
def test_hidden_site_masks_through_layer(dtype, B, S, H, heads, F):
    # x = 0, Wqkv = Wo = W2 = 0, bo = 1, b2 = 2: y = keep1 * 1/(1-p) + keep2 * 2/(1-p)
    p, seed, off = 0.1, 4321, 3
    dev = torch.device("cuda", 0)
    w = _zero_weights(H, F, dtype, dev)
    w["bo"].fill_(1.0)
    w["b2"].fill_(2.0)
    L = Layer(B, S, H, heads, F, 0.0, p, True, seed, dtype=dtype, philox_offset=off)
    try:
        x = torch.zeros(B, S, H, dtype=dtype, device=dev)
        y = L.forward(x, None, w).double().cpu().numpy().reshape(-1)
    finally:
        L.close()
    sc = 1.0 / (1.0 - float(np.float32(p)))
    keep2 = y > 1.5 * sc
    keep1 = (y - keep2 * 2 * sc) > 0.5 * sc
    p32 = float(np.float32(p))
    assert np.array_equal(keep1, oracle.dropout_keep(0, B * S * H, 1, off, seed, p32))
    assert np.array_equal(keep2, oracle.dropout_keep(0, B * S * H, 2, off, seed, p32))


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("S", [64, 128])
def test_attention_site_mask_through_layer(dtype, S):
    # One head with d = S: Q = K = 0 makes P uniform (1/S); V = LN1(x) with
    # x[b, s] = e_s gives V_j[c] = (S*[j == c] - 1) / sqrt(S - 1), so
    # ctx_i[c] = (1/(1-p)) / sqrt(S-1) * keep_ic - (a constant per row).
    # Wo = I, no hidden dropout, FFN zero: y = x + ctx.
    B, H, F, p, seed, off = 2, S, 64, 0.1, 99, 11
    dev = torch.device("cuda", 0)
    w = _zero_weights(H, F, dtype, dev)
    w["wqkv"][2 * H:] = torch.eye(H, dtype=dtype, device=dev)
    w["wo"].copy_(torch.eye(H, dtype=dtype, device=dev))
    x = torch.eye(S, H, dtype=dtype, device=dev).expand(B, S, H).contiguous()
    L = Layer(B, S, H, 1, F, p, 0.0, True, seed, dtype=dtype, philox_offset=off)
    try:
        y = L.forward(x, None, w)
    finally:
        L.close()
    ctx = (y.double() - x.double()).cpu().numpy()          # (B, S, S): row i, column c = key c
    step = (1.0 / (1.0 - float(np.float32(p)))) / np.sqrt(S - 1.0)
    rel = ctx - ctx.min(axis=-1, keepdims=True)
    keep = rel > 0.5 * step
    ref = oracle.dropout_keep(0, B * S * S, 0, off, seed, float(np.float32(p))).reshape(B, S, S)
    # rows with no dropped key have no zero baseline: only compare rows where
    # the reference drops at least one key (all rows here, with overwhelming odds)
    rows = ~ref.all(axis=-1)
    assert rows.mean() > 0.9
    assert np.array_equal(keep[rows], ref[rows])
