"""B200 (sm_100a) fused Transformer encoder layer: Python binding of libtlp.so.

The binding only marshals arguments: every step of the layer runs in the
CUDA kernels behind the C ABI declared in include/tlp.h.  PyTorch supplies
device memory and streams.  There is no fallback: if the library is missing,
LibraryMissing is raised.
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["Layer", "Options", "TlError", "LibraryMissing", "load_library", "dropout_keep_mask",
           "WEIGHT_NAMES", "DTYPE_CODES", "EXPORTED_SYMBOLS", "device_check",
           "profile_enable", "profile_read", "launch_count", "PROFILE_CLASSES",
           "pld_theta", "pld_keep_prob", "pld_keep", "set_wait_limit", "wait_probe"]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtlp.so")

WEIGHT_NAMES = (
    "wqkv", "bqkv", "wo", "bo", "ln1_g", "ln1_b",
    "w1", "b1", "w2", "b2", "ln2_g", "ln2_b",
)
DTYPE_CODES = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
EXPORTED_SYMBOLS = (
    "layer_create", "layer_default_options", "layer_set_options", "layer_get_options", "layer_set_rng",
    "layer_forward", "layer_backward", "layer_workspace_bytes", "layer_last_error",
    "layer_destroy", "tl_dropout_keep_mask", "tl_device_check", "tl_profile_enable",
    "tl_profile_read", "tl_launch_count", "tl_bias_grad_noalloc", "tl_gelu_eval", "tl_status_string",
    "tl_pld_theta", "tl_pld_keep_prob", "tl_pld_keep", "tl_gelu_tanh_eval",
    "tl_set_wait_limit_ns", "tl_wait_probe", "layer_scratch_bytes", "layer_share_scratch",
)
PROFILE_CLASSES = ("gemm", "attn_fwd", "attn_bwd", "ln_fwd", "ln_bwd", "rowwise")


class LibraryMissing(RuntimeError):
    pass


class TlError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"tlp status {status}: {msg}")
        self.status = status


class Options(ctypes.Structure):
    _fields_ = [
        ("dtype", ctypes.c_int),
        ("ln_eps", ctypes.c_float),
        ("philox_offset", ctypes.c_uint64),
        ("gelu_checkpoint", ctypes.c_int),
        ("attn_dropout_checkpoint", ctypes.c_int),
        ("normalize_invertible", ctypes.c_int),
        ("training", ctypes.c_int),
        ("gelu_tanh", ctypes.c_int),
        ("stochastic_mode", ctypes.c_int),
    ]


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_NAMES]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libtlp.so once.  Raises LibraryMissing when it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise LibraryMissing(f"{path} not found: build it with `python -m transformer_layer_pre_b200.build_ext`")
    lib = ctypes.CDLL(path)
    vp, i, f, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint64
    lib.layer_create.argtypes = [i, i, i, i, i, f, f, i, u64, ctypes.POINTER(vp)]
    lib.layer_create.restype = i
    lib.layer_default_options.argtypes = [ctypes.POINTER(Options)]
    lib.layer_default_options.restype = None
    lib.layer_set_options.argtypes = [vp, ctypes.POINTER(Options)]
    lib.layer_set_options.restype = i
    lib.layer_get_options.argtypes = [vp, ctypes.POINTER(Options)]
    lib.layer_set_rng.argtypes = [vp, u64, u64]
    lib.layer_set_rng.restype = i
    lib.layer_get_options.restype = i
    lib.layer_forward.argtypes = [vp, vp, vp, ctypes.POINTER(_Weights), vp, vp]
    lib.layer_forward.restype = i
    lib.layer_backward.argtypes = [vp, vp, vp, ctypes.POINTER(_Weights), ctypes.POINTER(_Weights), vp, vp]
    lib.layer_backward.restype = i
    lib.layer_workspace_bytes.argtypes = [vp]
    lib.layer_workspace_bytes.restype = ctypes.c_size_t
    lib.layer_scratch_bytes.argtypes = [vp]
    lib.layer_scratch_bytes.restype = ctypes.c_size_t
    lib.layer_share_scratch.argtypes = [vp, vp, ctypes.c_size_t]
    lib.layer_share_scratch.restype = i
    lib.layer_last_error.argtypes = [vp]
    lib.layer_last_error.restype = ctypes.c_char_p
    lib.layer_destroy.argtypes = [vp]
    lib.layer_destroy.restype = None
    lib.tl_dropout_keep_mask.argtypes = [u64, u64, i, f, u64, u64, vp, vp]
    lib.tl_dropout_keep_mask.restype = i
    lib.tl_device_check.argtypes = []
    lib.tl_device_check.restype = i
    lib.tl_profile_enable.argtypes = [i]
    lib.tl_profile_enable.restype = None
    lib.tl_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_longlong), i]
    lib.tl_profile_read.restype = i
    lib.tl_launch_count.argtypes = []
    lib.tl_launch_count.restype = ctypes.c_longlong
    lib.tl_bias_grad_noalloc.argtypes = [i, vp, i, i, vp, vp]
    lib.tl_bias_grad_noalloc.restype = i
    lib.tl_gelu_eval.argtypes = [vp, vp, vp, u64, vp]
    lib.tl_gelu_eval.restype = i
    lib.tl_gelu_tanh_eval.argtypes = [vp, vp, vp, u64, vp]
    lib.tl_gelu_tanh_eval.restype = i
    lib.tl_status_string.argtypes = [i]
    lib.tl_status_string.restype = ctypes.c_char_p
    d = ctypes.c_double
    lib.tl_pld_theta.argtypes = [d, d, u64]
    lib.tl_pld_theta.restype = d
    lib.tl_pld_keep_prob.argtypes = [i, i, d]
    lib.tl_pld_keep_prob.restype = d
    lib.tl_pld_keep.argtypes = [u64, u64, i, i, d]
    lib.tl_pld_keep.restype = i
    lib.tl_set_wait_limit_ns.argtypes = [u64]
    lib.tl_set_wait_limit_ns.restype = i
    lib.tl_wait_probe.argtypes = [vp]
    lib.tl_wait_probe.restype = i
    _lib = lib
    return lib


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


class Layer:
    """One encoder layer (a handle of the C ABI).

    Layer(batch, seq, hidden, heads, ffn=0, attn_dropout=0., hidden_dropout=0.,
    pre_layer_norm=True, seed=1234, dtype=torch.float16, ...options)
    """

    def __init__(self, batch, seq, hidden, heads, ffn=0, attn_dropout=0.0, hidden_dropout=0.0,
                 pre_layer_norm=True, seed=1234, dtype=torch.float16, ln_eps=1e-12, philox_offset=0,
                 gelu_checkpoint=False, attn_dropout_checkpoint=False, normalize_invertible=False,
                 training=True, gelu_tanh=False, stochastic_mode=False):
        self.lib = load_library()
        self.handle = None
        h = ctypes.c_void_p()
        st = self.lib.layer_create(batch, seq, hidden, heads, ffn, attn_dropout, hidden_dropout,
                                   int(pre_layer_norm), seed, ctypes.byref(h))
        if st != 0:
            raise TlError(st, self.lib.tl_status_string(st).decode())
        self.handle = h
        self.batch, self.seq, self.hidden, self.heads = batch, seq, hidden, heads
        self.ffn = ffn if ffn > 0 else 4 * hidden
        self.dtype = dtype
        opt = Options()
        self.lib.layer_default_options(ctypes.byref(opt))
        opt.dtype = DTYPE_CODES[dtype]
        opt.ln_eps = ln_eps
        opt.philox_offset = philox_offset
        opt.gelu_checkpoint = int(gelu_checkpoint)
        opt.attn_dropout_checkpoint = int(attn_dropout_checkpoint)
        opt.normalize_invertible = int(normalize_invertible)
        opt.training = int(training)
        opt.gelu_tanh = int(gelu_tanh)
        opt.stochastic_mode = int(stochastic_mode)
        self._check(self.lib.layer_set_options(self.handle, ctypes.byref(opt)))

    def _check(self, st: int) -> None:
        if st != 0:
            msg = self.lib.layer_last_error(self.handle).decode() if self.handle else ""
            raise TlError(st, msg or self.lib.tl_status_string(st).decode())

    @staticmethod
    def _weights(w: dict) -> _Weights:
        return _Weights(*[_ptr(w[n]) for n in WEIGHT_NAMES])

    def set_rng(self, seed: int, philox_offset: int) -> None:
        """Dropout key and 4th Philox counter word of the next forward (its
        backward keeps the forward's); nothing is reallocated."""
        self._check(self.lib.layer_set_rng(self.handle, seed, philox_offset))

    def forward(self, x, mask, weights, y=None, stream=None):
        """x (B, S, H) storage dtype on the device; mask (B, S) float32 or None."""
        if y is None:
            y = torch.empty_like(x)
        wt = self._weights(weights)
        self._check(self.lib.layer_forward(self.handle, _ptr(x), _ptr(mask), ctypes.byref(wt), _ptr(y),
                                           _stream(stream)))
        return y

    def backward(self, x, dy, weights, grads=None, dx=None, stream=None):
        """Returns (dx, grads) with grads a dict of float32 tensors."""
        if dx is None:
            dx = torch.empty_like(dy)
        if grads is None:
            grads = {n: torch.empty(tuple(weights[n].shape), dtype=torch.float32, device=dy.device)
                     for n in WEIGHT_NAMES}
        wt = self._weights(weights)
        gt = self._weights(grads)
        self._check(self.lib.layer_backward(self.handle, _ptr(x), _ptr(dy), ctypes.byref(wt), ctypes.byref(gt),
                                            _ptr(dx), _stream(stream)))
        return dx, grads

    @property
    def workspace_bytes(self) -> int:
        """Device bytes the layer holds (saved activations + its own scratch)."""
        return int(self.lib.layer_workspace_bytes(self.handle))

    @property
    def scratch_bytes(self) -> int:
        """Bytes of the per-call scratch this layer needs."""
        return int(self.lib.layer_scratch_bytes(self.handle))

    def share_scratch(self, buf: torch.Tensor) -> None:
        """Use `buf` (a device tensor of >= scratch_bytes bytes, 256-byte
        aligned; the caller keeps it alive) as this layer's scratch; layers
        sharing one must not run concurrently."""
        self._check(self.lib.layer_share_scratch(self.handle, _ptr(buf), buf.numel() * buf.element_size()))
        self._scratch_ref = buf

    def close(self) -> None:
        if self.handle:
            self.lib.layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def device_check() -> None:
    """Synchronises the device; raises TlError on a pending CUDA error or a
    bounded device-side wait that gave up."""
    lib = load_library()
    st = lib.tl_device_check()
    if st != 0:
        raise TlError(st, lib.tl_status_string(st).decode())


def set_wait_limit(ns: int) -> None:
    """Limit (ns; 0 = the default 2 s) of every bounded device-side wait on
    the current device."""
    lib = load_library()
    st = lib.tl_set_wait_limit_ns(int(ns))
    if st != 0:
        raise TlError(st, lib.tl_status_string(st).decode())


def wait_probe(stream=None) -> None:
    """Enqueues a kernel whose one bounded wait is never satisfied; the next
    device_check raises TlError with status 5 (TL_ETIMEOUT)."""
    lib = load_library()
    st = lib.tl_wait_probe(_stream(stream))
    if st != 0:
        raise TlError(st, lib.tl_status_string(st).decode())


def gelu_eval(u: torch.Tensor, tanh_form: bool = False):
    """(GELU(u), GELU'(u)) from the library's device GELU (erf form, or the
    tanh approximation); u float32 on the device."""
    lib = load_library()
    u = u.contiguous()
    g = torch.empty_like(u)
    dg = torch.empty_like(u)
    fn = lib.tl_gelu_tanh_eval if tanh_form else lib.tl_gelu_eval
    st = fn(_ptr(u), _ptr(g), _ptr(dg), u.numel(), _stream(None))
    if st != 0:
        raise TlError(st, lib.tl_status_string(st).decode())
    return g, dg


def profile_enable(on: bool) -> None:
    load_library().tl_profile_enable(int(on))


def profile_read() -> dict:
    """{class: (milliseconds, bracketed launch groups)} since the last read."""
    lib = load_library()
    n = len(PROFILE_CLASSES)
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_longlong * n)()
    lib.tl_profile_read(ms, cnt, n)
    return {c: (ms[i], cnt[i]) for i, c in enumerate(PROFILE_CLASSES)}


def attention_uses_tensor_cores(dtype: str, heads: int, head_dim: int, seq: int) -> bool:
    """Whether the library runs attention on tensor cores for this shape
    (16-bit storage and head dim 64); the exact-float32 SIMT kernels serve
    the rest."""
    return dtype in ("f16", "bf16") and head_dim == 64 and seq >= 8


def pld_theta(theta_bar: float, gamma: float, step: int) -> float:
    """Progressive Layer Dropping keep level at a global step."""
    return float(load_library().tl_pld_theta(theta_bar, gamma, step))


def pld_keep_prob(layer: int, num_layers: int, theta: float) -> float:
    return float(load_library().tl_pld_keep_prob(layer, num_layers, theta))


def pld_keep(seed: int, step: int, layer: int, num_layers: int, theta: float) -> bool:
    """Whether `layer` runs at `step` (False: the layer is the identity)."""
    r = load_library().tl_pld_keep(seed, step, layer, num_layers, theta)
    if r < 0:
        raise ValueError(f"layer {layer} outside a stack of {num_layers}")
    return bool(r)


def launch_count() -> int:
    return int(load_library().tl_launch_count())


def dropout_keep_mask(seed: int, offset: int, site: int, p: float, e0: int, n: int, device="cuda") -> torch.Tensor:
    """Keep bits computed on the device by the layer's own Philox code."""
    lib = load_library()
    out = torch.empty(n, dtype=torch.uint8, device=device)
    st = lib.tl_dropout_keep_mask(seed, offset, site, p, e0, n, _ptr(out), _stream(None))
    if st != 0:
        raise TlError(st, lib.tl_status_string(st).decode())
    return out
