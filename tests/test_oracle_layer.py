"""Pins of the oracle's whole layer (forward and backward):

* PyTorch's float64 nn.TransformerEncoderLayer (a library routine) with
  dropout 0, erf GELU, eps 1e-12, weights mapped one to one, norm_first for
  pre-LN and not for post-LN, key padding masks, autograd for every gradient;
* central finite differences of L = sum(y * dY) with dropout on (the masks
  are fixed by the seed), for x and every parameter, pre-LN and post-LN;
* the zero-weight closed form (pre-LN y = x, dx = dY, bias grads = sum dY);
* running a subset of the sequences reproduces the full batch's rows.
"""
import numpy as np
import pytest
import torch

from oracle import LayerConfig, WEIGHT_NAMES, layer_forward, layer_forward_backward


def _weights(rng, h, f, std=0.2):
    return dict(
        wqkv=rng.normal(0, std, (3 * h, h)), bqkv=rng.normal(0, 0.1, 3 * h),
        wo=rng.normal(0, std, (h, h)), bo=rng.normal(0, 0.1, h),
        ln1_g=rng.normal(1, 0.2, h), ln1_b=rng.normal(0, 0.1, h),
        w1=rng.normal(0, std, (f, h)), b1=rng.normal(0, 0.1, f),
        w2=rng.normal(0, std, (h, f)), b2=rng.normal(0, 0.1, h),
        ln2_g=rng.normal(1, 0.2, h), ln2_b=rng.normal(0, 0.1, h),
    )


def _mask(lengths, s):
    return np.where(np.arange(s)[None, :] < np.asarray(lengths)[:, None], 0.0, -np.inf)


def _torch_layer(cfg, w, x, mask, dy):
    h, nh, f = cfg.hidden, cfg.heads, cfg.ffn_dim
    act = "gelu" if cfg.gelu_form == "erf" else (lambda v: torch.nn.functional.gelu(v, approximate="tanh"))
    layer = torch.nn.TransformerEncoderLayer(
        d_model=h, nhead=nh, dim_feedforward=f, dropout=0.0, activation=act,
        layer_norm_eps=cfg.ln_eps, batch_first=True, norm_first=cfg.pre_layer_norm,
        dtype=torch.float64)
    T = lambda a: torch.tensor(a, dtype=torch.float64)
    with torch.no_grad():
        layer.self_attn.in_proj_weight.copy_(T(w["wqkv"]))
        layer.self_attn.in_proj_bias.copy_(T(w["bqkv"]))
        layer.self_attn.out_proj.weight.copy_(T(w["wo"]))
        layer.self_attn.out_proj.bias.copy_(T(w["bo"]))
        layer.linear1.weight.copy_(T(w["w1"])); layer.linear1.bias.copy_(T(w["b1"]))
        layer.linear2.weight.copy_(T(w["w2"])); layer.linear2.bias.copy_(T(w["b2"]))
        layer.norm1.weight.copy_(T(w["ln1_g"])); layer.norm1.bias.copy_(T(w["ln1_b"]))
        layer.norm2.weight.copy_(T(w["ln2_g"])); layer.norm2.bias.copy_(T(w["ln2_b"]))
    layer.train()
    xt = T(x).requires_grad_(True)
    kpm = None if mask is None else torch.tensor(~np.isfinite(mask))
    y = layer(xt, src_key_padding_mask=kpm)
    y.backward(T(dy))
    p = {
        "wqkv": layer.self_attn.in_proj_weight, "bqkv": layer.self_attn.in_proj_bias,
        "wo": layer.self_attn.out_proj.weight, "bo": layer.self_attn.out_proj.bias,
        "ln1_g": layer.norm1.weight, "ln1_b": layer.norm1.bias,
        "w1": layer.linear1.weight, "b1": layer.linear1.bias,
        "w2": layer.linear2.weight, "b2": layer.linear2.bias,
        "ln2_g": layer.norm2.weight, "ln2_b": layer.norm2.bias,
    }
    return y.detach().numpy(), xt.grad.numpy(), {n: p[n].grad.numpy() for n in WEIGHT_NAMES}


@pytest.mark.parametrize("pre_ln", [True, False])
@pytest.mark.parametrize("masked", [False, True])
@pytest.mark.parametrize("gelu_form", ["erf", "tanh"])
def test_matches_torch_encoder_layer_float64(pre_ln, masked, gelu_form):
    rng = np.random.default_rng(11)
    cfg = LayerConfig(batch=3, seq=16, hidden=32, heads=4, ffn=48, pre_layer_norm=pre_ln, gelu_form=gelu_form)
    w = _weights(rng, 32, 48)
    x = rng.normal(0, 1, (3, 16, 32))
    dy = rng.normal(0, 1, (3, 16, 32))
    mask = _mask([16, 9, 12], 16) if masked else None
    out = layer_forward_backward(cfg, x, mask, w, dy)
    ty, tdx, tg = _torch_layer(cfg, w, x, mask, dy)
    assert np.allclose(out["y"], ty, atol=1e-12, rtol=0)
    assert np.allclose(out["dx"], tdx, atol=1e-11, rtol=0)
    for n in WEIGHT_NAMES:
        assert np.allclose(out["grads"][n], tg[n], atol=1e-10, rtol=1e-10), n


@pytest.mark.parametrize("pre_ln", [True, False])
def test_finite_differences_with_dropout(pre_ln):
    rng = np.random.default_rng(12)
    cfg = LayerConfig(batch=2, seq=8, hidden=16, heads=2, ffn=24, attn_dropout=0.25,
                      hidden_dropout=0.2, pre_layer_norm=pre_ln, seed=77, philox_offset=5)
    w = _weights(rng, 16, 24, std=0.3)
    x = rng.normal(0, 1, (2, 8, 16))
    dy = rng.normal(0, 1, (2, 8, 16))
    mask = _mask([8, 5], 8)
    out = layer_forward_backward(cfg, x, mask, w, dy)
    # dropout actually dropped something in every site
    from oracle.layer import _hidden_keep
    assert not _hidden_keep(cfg, [0, 1], 1).all() and not _hidden_keep(cfg, [0, 1], 2).all()

    def loss(x_, w_):
        return float((layer_forward(cfg, x_, mask, w_)[0] * dy).sum())

    h = 1e-6
    pick = np.random.default_rng(13)
    for _ in range(8):
        idx = tuple(pick.integers(0, n) for n in x.shape)
        xp, xm = x.copy(), x.copy(); xp[idx] += h; xm[idx] -= h
        fd = (loss(xp, w) - loss(xm, w)) / (2 * h)
        assert abs(fd - out["dx"][idx]) <= 1e-6 * max(1.0, abs(fd)), ("x", idx)
    for n in WEIGHT_NAMES:
        for _ in range(4):
            idx = tuple(pick.integers(0, s) for s in w[n].shape)
            wp = {k: v.copy() for k, v in w.items()}; wp[n][idx] += h
            wm = {k: v.copy() for k, v in w.items()}; wm[n][idx] -= h
            fd = (loss(x, wp) - loss(x, wm)) / (2 * h)
            assert abs(fd - out["grads"][n][idx]) <= 1e-6 * max(1.0, abs(fd)), (n, idx)


def test_zero_weights_closed_form():
    rng = np.random.default_rng(14)
    h, f = 32, 64
    w = {n: np.zeros(s) for n, s in [("wqkv", (3 * h, h)), ("bqkv", 3 * h), ("wo", (h, h)), ("bo", h),
                                     ("w1", (f, h)), ("b1", f), ("w2", (h, f)), ("b2", h)]}
    w.update(ln1_g=np.ones(h), ln1_b=np.zeros(h), ln2_g=np.ones(h), ln2_b=np.zeros(h))
    cfg = LayerConfig(batch=2, seq=8, hidden=h, heads=4, ffn=f)
    x = rng.normal(0, 1, (2, 8, h))
    dy = rng.normal(0, 1, (2, 8, h))
    out = layer_forward_backward(cfg, x, None, w, dy)
    assert np.array_equal(out["y"], x)
    assert np.array_equal(out["dx"], dy)
    for n in ("wqkv", "bqkv", "wo", "w1", "b1", "w2", "ln1_g", "ln1_b", "ln2_g", "ln2_b"):
        assert np.all(out["grads"][n] == 0), n
    assert np.allclose(out["grads"]["b2"], dy.sum((0, 1)), atol=1e-13)
    assert np.allclose(out["grads"]["bo"], dy.sum((0, 1)), atol=1e-13)


@pytest.mark.parametrize("storage_rounded", [False, True])
def test_sequence_subset_reproduces_rows(storage_rounded):
    rng = np.random.default_rng(15)
    cfg = LayerConfig(batch=4, seq=8, hidden=16, heads=2, ffn=32, attn_dropout=0.1,
                      hidden_dropout=0.1, storage="f16")
    w = _weights(rng, 16, 32)
    x = rng.normal(0, 1, (4, 8, 16))
    dy = rng.normal(0, 1, (4, 8, 16))
    mask = _mask([8, 6, 7, 8], 8)
    full = layer_forward_backward(cfg, x, mask, w, dy, storage_rounded=storage_rounded)
    sub = layer_forward_backward(cfg, x[[1, 3]], mask[[1, 3]], w, dy[[1, 3]], seq_index=[1, 3],
                                 storage_rounded=storage_rounded)
    assert np.array_equal(sub["y"], full["y"][[1, 3]])
    assert np.array_equal(sub["dx"], full["dx"][[1, 3]])


def test_storage_rounding_stays_close_to_pure():
    rng = np.random.default_rng(16)
    cfg = LayerConfig(batch=2, seq=16, hidden=32, heads=2, ffn=64, attn_dropout=0.1,
                      hidden_dropout=0.1, storage="f16")
    w = _weights(rng, 32, 64, std=0.05)
    x = rng.normal(0, 1, (2, 16, 32))
    dy = rng.normal(0, 1, (2, 16, 32))
    a = layer_forward_backward(cfg, x, None, w, dy)
    b = layer_forward_backward(cfg, x, None, w, dy, storage_rounded=True)
    rel = lambda u, v: np.linalg.norm(u - v) / np.linalg.norm(v)
    assert 0 < rel(b["y"], a["y"]) < 3e-3
    assert 0 < rel(b["dx"], a["dx"]) < 3e-3
    for n in WEIGHT_NAMES:
        assert rel(b["grads"][n], a["grads"][n]) < 1e-2, n
