"""fp64 oracle of one BERT-style encoder layer, forward and backward.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.  Plain float64 numpy; numpy's matmul is the only library step.

Notation: T = B*S tokens, H hidden, nh heads, d = H/nh, F FFN width.
Tensors are row-major, weights are [out, in] (a Linear layer's convention,
"AI-infra engineers and the Transformer", section 2.1 Step 2).

Parity status: every function below is pinned by a test under ``tests/``
(test_oracle_*.py); none is "parity unpinned".
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np
from scipy.special import erf

WEIGHT_NAMES = (
    "wqkv", "bqkv", "wo", "bo", "ln1_g", "ln1_b",
    "w1", "b1", "w2", "b2", "ln2_g", "ln2_b",
)

# Dropout sites: the Philox counter's third word says which dropout a bit
# belongs to (attention probabilities, attention-block output, FFN output).
SITE_ATTN, SITE_ATTN_OUT, SITE_FFN_OUT = 0, 1, 2


@dataclasses.dataclass
class LayerConfig:
    """The layer's configuration surface ("DeepSpeed Transformer Kernel usage
    guide", Step 2: batch_size, max_seq_length, hidden_size, heads,
    attn_dropout_ratio, hidden_dropout_ratio, pre_layer_norm, seed,
    intermediate_size, layer_norm_eps)."""

    batch: int
    seq: int
    hidden: int
    heads: int
    ffn: int = 0                 # <= 0 means 4 * hidden (Step 2, extra parameters)
    attn_dropout: float = 0.0
    hidden_dropout: float = 0.0
    pre_layer_norm: bool = True
    seed: int = 1234
    philox_offset: int = 0       # the layer's id in a stack
    ln_eps: float = 1e-12
    storage: str = "f32"        # 'f32' | 'f16' | 'bf16': what the GPU stores in HBM
    gelu_form: str = "erf"      # 'erf' (exact) | 'tanh' (the approximation of section 2.3)

    @property
    def ffn_dim(self) -> int:
        return self.ffn if self.ffn > 0 else 4 * self.hidden

    @property
    def head_dim(self) -> int:
        return self.hidden // self.heads


# --------------------------------------------------------------------------
# Philox4x32-10 (Salmon, Moraes, Dror, Shaw: "Parallel Random Numbers: As Easy
# as 1, 2, 3", SC'11), written from the paper's definition: ten rounds of two
# 32x32->64 multiplies with a Weyl-sequence key schedule.
# --------------------------------------------------------------------------
_PHILOX_M0 = np.uint64(0xD2511F53)
_PHILOX_M1 = np.uint64(0xCD9E8D57)
_PHILOX_W0 = np.uint64(0x9E3779B9)
_PHILOX_W1 = np.uint64(0xBB67AE85)
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0, k1):
    """Philox4x32 with 10 rounds.  Counter words c0..c3 and key words k0, k1
    are arrays (or scalars) of 32-bit values; returns the four output words as
    uint64 arrays holding 32-bit values."""
    c = [np.asarray(v, dtype=np.uint64) & _MASK32 for v in (c0, c1, c2, c3)]
    k = [np.asarray(v, dtype=np.uint64) & _MASK32 for v in (k0, k1)]
    for rnd in range(10):
        if rnd > 0:  # key bump before every round after the first
            k = [(k[0] + _PHILOX_W0) & _MASK32, (k[1] + _PHILOX_W1) & _MASK32]
        p0 = _PHILOX_M0 * c[0]            # < 2^64, exact in uint64
        p1 = _PHILOX_M1 * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c = [hi1 ^ c[1] ^ k[0], lo1, hi0 ^ c[3] ^ k[1], lo0]
    return c


def dropout_threshold(p: float) -> int:
    """An element is dropped when its 16-bit random lane is below
    floor(p * 65536); p = 0 drops nothing."""
    return int(math.floor(float(p) * 65536.0))


def dropout_lanes(e0: int, n: int, site: int, offset: int, seed: int) -> np.ndarray:
    """16-bit random lanes for the flat element indices e0 .. e0+n-1.

    Counter contract (the pages only say that dropout is seeded): element e
    uses Philox counter (g mod 2^32, g div 2^32, site, offset) with g = e div 8
    and key (seed mod 2^32, seed div 2^32); lane e mod 8 = k takes the
    16-bit half (k mod 2) of output word (k div 2), low half first."""
    assert e0 % 8 == 0 and n % 8 == 0
    g = np.arange(e0 // 8, (e0 + n) // 8, dtype=np.uint64)
    w = philox4x32_10(g & _MASK32, g >> np.uint64(32), site, offset,
                      seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF)
    lanes = np.empty((g.size, 8), dtype=np.uint64)
    for k in range(8):
        lanes[:, k] = (w[k >> 1] >> np.uint64(16 * (k & 1))) & np.uint64(0xFFFF)
    return lanes.reshape(-1)


def dropout_keep(e0: int, n: int, site: int, offset: int, seed: int, p: float) -> np.ndarray:
    """Boolean keep mask for flat elements e0 .. e0+n-1 (see dropout_lanes)."""
    return dropout_lanes(e0, n, site, offset, seed) >= np.uint64(dropout_threshold(p))


def _apply_dropout(v: np.ndarray, keep: np.ndarray, p: float) -> np.ndarray:
    """Inverted dropout ("AI-infra engineers and the Transformer", section
    5.1): kept values are scaled by 1/(1-p), dropped ones become 0."""
    return np.where(keep, v * (1.0 / (1.0 - p)), 0.0)


# --------------------------------------------------------------------------
# Storage rounding: round-to-nearest-even to a binary floating format, written
# from IEEE 754's definition (significand of `prec` bits incl. the implicit
# one, minimum normal exponent `emin`, gradual underflow, overflow to inf).
# --------------------------------------------------------------------------
_FORMATS = {"f16": (11, -14, 15), "bf16": (8, -126, 127), "f32": (24, -126, 127)}


def round_to_storage(v: np.ndarray, kind: str | None) -> np.ndarray:
    """Round float64 values to the nearest value of format `kind` (ties to
    even) and return them widened back to float64.  kind None / 'f64' is the
    identity."""
    if kind is None or kind == "f64":
        return np.asarray(v, dtype=np.float64)
    prec, emin, emax = _FORMATS[kind]
    v = np.asarray(v, dtype=np.float64)
    _, e = np.frexp(v)                    # v = m * 2^e, 0.5 <= |m| < 1
    ulp = np.ldexp(1.0, np.maximum(e, emin + 1) - prec)
    r = np.round(v / ulp) * ulp           # np.round rounds halves to even
    max_finite = (2.0 - 2.0 ** (1 - prec)) * 2.0 ** emax
    r = np.where(np.abs(r) > max_finite, np.copysign(np.inf, v), r)
    return np.where(np.isfinite(v), r, v)


# --------------------------------------------------------------------------
# Elementary steps
# --------------------------------------------------------------------------
def layer_norm_forward(x: np.ndarray, gamma: np.ndarray, beta: np.ndarray, eps: float):
    """LayerNorm over the last (hidden) axis of each token: biased variance,
    eps inside the square root, affine gamma/beta.  Returns (y, mean, rstd)."""
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = (x - mean) * rstd
    return gamma * xhat + beta, mean[..., 0], rstd[..., 0]


def layer_norm_backward(dy: np.ndarray, x: np.ndarray, mean: np.ndarray, rstd: np.ndarray,
                        gamma: np.ndarray):
    """Gradient of LayerNorm: returns (dx, dgamma, dbeta); dgamma and dbeta
    are summed over every token."""
    xhat = (x - mean[..., None]) * rstd[..., None]
    g = dy * gamma
    dx = rstd[..., None] * (g - g.mean(axis=-1, keepdims=True)
                            - xhat * (g * xhat).mean(axis=-1, keepdims=True))
    red = tuple(range(dy.ndim - 1))
    return dx, (dy * xhat).sum(axis=red), dy.sum(axis=red)


def layer_norm_backward_from_output(dy: np.ndarray, y: np.ndarray, rstd: np.ndarray, gamma: np.ndarray,
                                    beta: np.ndarray):
    """The same gradient computed from the LayerNorm output instead of its
    input ("DeepSpeed Transformer Kernel usage guide", Step 3,
    normalize_invertible): x-hat = (y - beta) / gamma, which needs every
    gamma to be non-zero; only rstd of the forward statistics is used."""
    xhat = (y - beta) / gamma
    g = dy * gamma
    dx = rstd[..., None] * (g - g.mean(axis=-1, keepdims=True)
                            - xhat * (g * xhat).mean(axis=-1, keepdims=True))
    red = tuple(range(dy.ndim - 1))
    return dx, (dy * xhat).sum(axis=red), dy.sum(axis=red)


def gelu(u: np.ndarray) -> np.ndarray:
    """GELU in its exact (erf) form: u * Phi(u)."""
    return 0.5 * u * (1.0 + erf(u / math.sqrt(2.0)))


def gelu_grad(u: np.ndarray) -> np.ndarray:
    """d GELU / du = Phi(u) + u * phi(u)."""
    return 0.5 * (1.0 + erf(u / math.sqrt(2.0))) + u * np.exp(-0.5 * u * u) / math.sqrt(2.0 * math.pi)


_SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)
_TANH_CUBIC = 0.044715


def gelu_tanh(u: np.ndarray) -> np.ndarray:
    """GELU in the tanh approximation ("AI-infra engineers and the
    Transformer", section 2.3): 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))."""
    return 0.5 * u * (1.0 + np.tanh(_SQRT_2_OVER_PI * (u + _TANH_CUBIC * u ** 3)))


def gelu_tanh_grad(u: np.ndarray) -> np.ndarray:
    """Derivative of gelu_tanh: with z = sqrt(2/pi) (u + 0.044715 u^3) and
    t = tanh(z), 0.5 (1 + t) + 0.5 u (1 - t^2) sqrt(2/pi) (1 + 3 * 0.044715 u^2)."""
    t = np.tanh(_SQRT_2_OVER_PI * (u + _TANH_CUBIC * u ** 3))
    return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * _SQRT_2_OVER_PI * (1.0 + 3.0 * _TANH_CUBIC * u * u)


def _gelu_pair(cfg):
    return (gelu_tanh, gelu_tanh_grad) if cfg.gelu_form == "tanh" else (gelu, gelu_grad)


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Softmax over the last axis with the row maximum subtracted; a row whose
    entries are all -inf (every key masked) is defined to be all zeros."""
    m = s.max(axis=-1, keepdims=True)
    dead = ~np.isfinite(m)
    e = np.exp(s - np.where(dead, 0.0, m))
    e = np.where(dead, 0.0, e)
    tot = e.sum(axis=-1, keepdims=True)
    return np.where(dead, 0.0, e / np.where(dead, 1.0, tot))


# --------------------------------------------------------------------------
# Attention (per sequence; the mask is additive over keys)
# --------------------------------------------------------------------------
def _heads(m: np.ndarray, nh: int) -> np.ndarray:
    """(S, H) -> (nh, S, d): head h owns columns h*d .. h*d+d-1."""
    s, h = m.shape
    return m.reshape(s, nh, h // nh).transpose(1, 0, 2)


def _merge(m: np.ndarray) -> np.ndarray:
    """(nh, S, d) -> (S, H): heads concatenated in head order."""
    nh, s, d = m.shape
    return m.transpose(1, 0, 2).reshape(s, nh * d)


def _attn_probs(q, k, mask_row, cfg: LayerConfig, b_global: int):
    """Scores Q K^T / sqrt(d) + mask, softmax over keys, and the dropout keep
    mask of the attention site for sequence b_global.  q, k: (nh, S, d)."""
    nh, s, d = q.shape
    scores = (q @ k.transpose(0, 2, 1)) / math.sqrt(d)
    if mask_row is not None:
        scores = scores + mask_row[None, None, :]
    p = softmax_rows(scores)
    e0 = b_global * nh * s * s
    keep = dropout_keep(e0, nh * s * s, SITE_ATTN, cfg.philox_offset, cfg.seed,
                        cfg.attn_dropout).reshape(nh, s, s)
    return p, keep


def attention_forward(qkv: np.ndarray, mask, cfg: LayerConfig, seq_index, rnd):
    """Multi-head attention of every sequence.  qkv: (nb, S, 3H) holding
    [Q | K | V] column blocks.  ctx = dropout(softmax(Q K^T/sqrt(d) + mask)) V,
    heads merged back to (nb, S, H).  Dropout acts on the probabilities,
    before the product with V."""
    nb, s, h3 = qkv.shape
    h = h3 // 3
    nh = cfg.heads
    ctx = np.empty((nb, s, h))
    for i in range(nb):
        q = _heads(qkv[i, :, :h], nh)
        k = _heads(qkv[i, :, h:2 * h], nh)
        v = _heads(qkv[i, :, 2 * h:], nh)
        p, keep = _attn_probs(q, k, None if mask is None else mask[i], cfg, seq_index[i])
        pd = _apply_dropout(p, keep, cfg.attn_dropout)
        ctx[i] = _merge(pd @ v)
    return rnd(ctx)


def attention_backward(dctx: np.ndarray, qkv: np.ndarray, mask, cfg: LayerConfig, seq_index, rnd):
    """Gradient of attention_forward with respect to qkv, (nb, S, 3H).
    Softmax backward from its Jacobian: dS = P * (dP - rowsum(P * dP))."""
    nb, s, h3 = qkv.shape
    h = h3 // 3
    nh = cfg.heads
    d = h // nh
    scale = 1.0 / (1.0 - cfg.attn_dropout)
    dqkv = np.empty_like(qkv)
    for i in range(nb):
        q = _heads(qkv[i, :, :h], nh)
        k = _heads(qkv[i, :, h:2 * h], nh)
        v = _heads(qkv[i, :, 2 * h:], nh)
        p, keep = _attn_probs(q, k, None if mask is None else mask[i], cfg, seq_index[i])
        pd = np.where(keep, p * scale, 0.0)
        do = _heads(dctx[i], nh)
        dv = pd.transpose(0, 2, 1) @ do
        dpd = do @ v.transpose(0, 2, 1)
        dp = np.where(keep, dpd * scale, 0.0)
        ds = p * (dp - (p * dp).sum(axis=-1, keepdims=True))
        dq = (ds @ k) / math.sqrt(d)
        dk = (ds.transpose(0, 2, 1) @ q) / math.sqrt(d)
        dqkv[i, :, :h] = _merge(dq)
        dqkv[i, :, h:2 * h] = _merge(dk)
        dqkv[i, :, 2 * h:] = _merge(dv)
    return rnd(dqkv)


# --------------------------------------------------------------------------
# The layer
# --------------------------------------------------------------------------
def _hidden_keep(cfg: LayerConfig, seq_index, site: int) -> np.ndarray:
    """Keep mask of a hidden-state dropout site for the given sequences; the
    flat index of token t = b*S + s, column c is t*H + c."""
    s, h = cfg.seq, cfg.hidden
    return np.stack([
        dropout_keep(b * s * h, s * h, site, cfg.philox_offset, cfg.seed,
                     cfg.hidden_dropout).reshape(s, h)
        for b in seq_index])


def _rounder(cfg: LayerConfig, storage_rounded: bool):
    kind = cfg.storage if storage_rounded else None
    return lambda v: round_to_storage(v, kind)


def layer_forward(cfg: LayerConfig, x, mask, w, seq_index=None, storage_rounded=False):
    """Forward pass of one encoder layer for the sequences in x (nb, S, H).

    Pre-LN (the default, "DeepSpeed Transformer Kernel usage guide", Step 2
    pre_layer_norm): h1 = LN1(x); attention on h1; x2 = x + drop(ctx Wo^T + bo);
    h2 = LN2(x2); y = x2 + drop(GELU(h2 W1^T + b1) W2^T + b2).
    Post-LN ("Forward-pass compute-graph optimisation", section 2 steps 1-6):
    x2 = LN1(x + drop(attn(x) Wo^T + bo)); y = LN2(x2 + drop(FFN(x2))).

    seq_index gives each row's global sequence number (dropout counters use
    it), so a subset of a batch reproduces the full batch's values exactly.
    With storage_rounded, every tensor the CUDA path keeps in HBM is rounded
    to cfg.storage where the path materialises it.  Returns (y, saved)."""
    x = np.asarray(x, dtype=np.float64)
    nb = x.shape[0]
    seq_index = np.arange(nb) if seq_index is None else np.asarray(seq_index)
    R = _rounder(cfg, storage_rounded)
    W = {n: np.asarray(w[n], dtype=np.float64) for n in WEIGHT_NAMES}
    mask = None if mask is None else np.asarray(mask, dtype=np.float64)
    ph = cfg.hidden_dropout
    keep1 = _hidden_keep(cfg, seq_index, SITE_ATTN_OUT)
    keep2 = _hidden_keep(cfg, seq_index, SITE_FFN_OUT)
    sv = dict(x=x, mask=mask, seq_index=seq_index, keep1=keep1, keep2=keep2, R=R, W=W)

    if cfg.pre_layer_norm:
        h1, m1, r1 = layer_norm_forward(x, W["ln1_g"], W["ln1_b"], cfg.ln_eps)
        h1 = R(h1)
        qkv = R(h1 @ W["wqkv"].T + W["bqkv"])
        ctx = attention_forward(qkv, mask, cfg, seq_index, R)
        x2 = R(x + _apply_dropout(ctx @ W["wo"].T + W["bo"], keep1, ph))
        h2, m2, r2 = layer_norm_forward(x2, W["ln2_g"], W["ln2_b"], cfg.ln_eps)
        h2 = R(h2)
        u = R(h2 @ W["w1"].T + W["b1"])
        g = R(_gelu_pair(cfg)[0](u))
        y = R(x2 + _apply_dropout(g @ W["w2"].T + W["b2"], keep2, ph))
        sv.update(h1=h1, mean1=m1, rstd1=r1, qkv=qkv, ctx=ctx, x2=x2,
                  h2=h2, mean2=m2, rstd2=r2, u=u, g=g)
    else:
        qkv = R(x @ W["wqkv"].T + W["bqkv"])
        ctx = attention_forward(qkv, mask, cfg, seq_index, R)
        res1 = R(x + _apply_dropout(ctx @ W["wo"].T + W["bo"], keep1, ph))
        x2, m1, r1 = layer_norm_forward(res1, W["ln1_g"], W["ln1_b"], cfg.ln_eps)
        x2 = R(x2)
        u = R(x2 @ W["w1"].T + W["b1"])
        g = R(_gelu_pair(cfg)[0](u))
        res2 = R(x2 + _apply_dropout(g @ W["w2"].T + W["b2"], keep2, ph))
        y, m2, r2 = layer_norm_forward(res2, W["ln2_g"], W["ln2_b"], cfg.ln_eps)
        y = R(y)
        sv.update(qkv=qkv, ctx=ctx, res1=res1, mean1=m1, rstd1=r1, x2=x2,
                  u=u, g=g, res2=res2, mean2=m2, rstd2=r2)
    return y, sv


def _colsum(m: np.ndarray) -> np.ndarray:
    return m.reshape(-1, m.shape[-1]).sum(axis=0)


def _wgrad(dz: np.ndarray, a: np.ndarray) -> np.ndarray:
    """dW[n, k] = sum over tokens of dZ[t, n] * A[t, k]."""
    return dz.reshape(-1, dz.shape[-1]).T @ a.reshape(-1, a.shape[-1])


def layer_backward(cfg: LayerConfig, sv: dict, dy):
    """Backward pass of layer_forward: returns (dx, grads) where grads holds
    the gradient of every weight in WEIGHT_NAMES, summed over the sequences
    of the forward.  Bias gradients are column sums of the stored output
    gradient of their Linear.  In storage-rounded mode GELU'(U) is rounded
    to the storage type before it scales dU (the CUDA path keeps it in HBM
    from the forward, or rounds it so when it recomputes it from U)."""
    dy = np.asarray(dy, dtype=np.float64)
    R, W, mask, seq_index = sv["R"], sv["W"], sv["mask"], sv["seq_index"]
    ph = cfg.hidden_dropout
    gr = {}
    if cfg.pre_layer_norm:
        dz2 = R(_apply_dropout(dy, sv["keep2"], ph))
        gr["b2"] = _colsum(dz2)
        gr["w2"] = _wgrad(dz2, sv["g"])
        du = R((dz2 @ W["w2"]) * R(_gelu_pair(cfg)[1](sv["u"])))
        gr["b1"] = _colsum(du)
        gr["w1"] = _wgrad(du, sv["h2"])
        dh2 = R(du @ W["w1"])
        dln2, gr["ln2_g"], gr["ln2_b"] = layer_norm_backward(dh2, sv["x2"], sv["mean2"], sv["rstd2"], W["ln2_g"])
        dx2 = R(dln2 + dy)
        da = R(_apply_dropout(dx2, sv["keep1"], ph))
        gr["bo"] = _colsum(da)
        gr["wo"] = _wgrad(da, sv["ctx"])
        dctx = R(da @ W["wo"])
        dqkv = attention_backward(dctx, sv["qkv"], mask, cfg, seq_index, R)
        gr["bqkv"] = _colsum(dqkv)
        gr["wqkv"] = _wgrad(dqkv, sv["h1"])
        dh1 = R(dqkv @ W["wqkv"])
        dln1, gr["ln1_g"], gr["ln1_b"] = layer_norm_backward(dh1, sv["x"], sv["mean1"], sv["rstd1"], W["ln1_g"])
        dx = R(dln1 + dx2)
    else:
        dres2, gr["ln2_g"], gr["ln2_b"] = layer_norm_backward(dy, sv["res2"], sv["mean2"], sv["rstd2"], W["ln2_g"])
        dres2 = R(dres2)
        dz2 = R(_apply_dropout(dres2, sv["keep2"], ph))
        gr["b2"] = _colsum(dz2)
        gr["w2"] = _wgrad(dz2, sv["g"])
        du = R((dz2 @ W["w2"]) * R(_gelu_pair(cfg)[1](sv["u"])))
        gr["b1"] = _colsum(du)
        gr["w1"] = _wgrad(du, sv["x2"])
        dx2 = R(du @ W["w1"] + dres2)
        dres1, gr["ln1_g"], gr["ln1_b"] = layer_norm_backward(dx2, sv["res1"], sv["mean1"], sv["rstd1"], W["ln1_g"])
        dres1 = R(dres1)
        da = R(_apply_dropout(dres1, sv["keep1"], ph))
        gr["bo"] = _colsum(da)
        gr["wo"] = _wgrad(da, sv["ctx"])
        dctx = R(da @ W["wo"])
        dqkv = attention_backward(dctx, sv["qkv"], mask, cfg, seq_index, R)
        gr["bqkv"] = _colsum(dqkv)
        gr["wqkv"] = _wgrad(dqkv, sv["x"])
        dx = R(dqkv @ W["wqkv"] + dres1)
    return dx, gr


def layer_forward_backward(cfg: LayerConfig, x, mask, w, dy, seq_index=None, storage_rounded=False):
    """Forward then backward; returns dict(y=..., dx=..., grads={...})."""
    y, sv = layer_forward(cfg, x, mask, w, seq_index=seq_index, storage_rounded=storage_rounded)
    dx, grads = layer_backward(cfg, sv, dy)
    return dict(y=y, dx=dx, grads=grads)
