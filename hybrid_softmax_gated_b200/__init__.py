"""ARL2 hybrid attention layer on B200: Python binding of libarl2.so.

Argument marshalling only: every step of the layer runs in the CUDA
kernels of ``libarl2.so`` (C ABI in ``include/arl2.h``).  PyTorch supplies
device memory and streams.  If the library is missing, importing this
package raises; there is no other implementation to fall back on.

The layer ("Attend Locally, Remember Linearly", technical summary §2.1 and
§2.2), per stream b and head h of one latent frame and denoising pass:

    out = softmax(Q K^T / sqrt(d)) V + (Q W_q[h]) S_{N-1}
    clean pass only, after the read:
    S_N = alpha S_{N-1} + K'^T diag(beta) (V' - K' S_{N-1}),
    K' = rownorm(K W_k[h]), V' = V W_v[h]

and the softmax teacher layer it replaces (TeacherLayer, technical summary
§1 "KV Cache Growth"): frame N attends to the clean keys/values of frames
0..N-1, kept in a KV cache, and bidirectionally to its own.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libarl2.so")

ARL2_OK = 0
ARL2_ERR_TIMEOUT = -6
ARL2_BF16, ARL2_FP32 = 0, 1
ARL2_IMPL_AUTO, ARL2_IMPL_SIMT = 0, 1
ARL2_GATE_HEADWISE, ARL2_GATE_ELEMENTWISE = 0, 1
ARL2_ACCESS_FRAME, ARL2_ACCESS_TOKEN = 0, 1

EXPORTED = (
    "arl2_create", "arl2_frame_forward", "arl2_frame_forward_host", "arl2_state_reset",
    "arl2_state_get", "arl2_state_set", "arl2_phi_apply", "arl2_device_status",
    "arl2_device_bytes", "arl2_kernel_launches", "arl2_state_update_noalloc", "arl2_destroy",
    "arl2_status_string", "arl2_version", "arl2_gates_apply", "arl2_frame_forward_hidden",
    "arl2_frame_forward_hidden_host", "arl2_selftest_wait_timeout",
    "arl2_kv_create", "arl2_kv_frame_forward", "arl2_kv_frame_forward_host", "arl2_kv_reset",
    "arl2_kv_frames", "arl2_kv_cache_get", "arl2_kv_cache_set", "arl2_kv_device_status", "arl2_kv_device_bytes",
    "arl2_kv_cache_bytes", "arl2_kv_kernel_launches", "arl2_kv_destroy",
)
NOALLOC_MAX_ELEMENTS = 1 << 22


class Arl2Config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("tokens_per_frame", ctypes.c_int), ("dtype", ctypes.c_int),
        ("w_q", ctypes.c_void_p), ("w_k", ctypes.c_void_p), ("w_v", ctypes.c_void_p),
        ("softmax_scale", ctypes.c_float), ("host_staging", ctypes.c_int), ("impl", ctypes.c_int),
        ("max_ctas", ctypes.c_int), ("gating", ctypes.c_int), ("access", ctypes.c_int),
        ("hidden_dim", ctypes.c_int), ("w_gate", ctypes.c_void_p), ("b_gate", ctypes.c_void_p),
    ]


class Arl2KvConfig(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("tokens_per_frame", ctypes.c_int), ("max_frames", ctypes.c_int), ("dtype", ctypes.c_int),
        ("softmax_scale", ctypes.c_float), ("host_staging", ctypes.c_int), ("impl", ctypes.c_int),
        ("max_ctas", ctypes.c_int),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python hybrid_softmax_gated_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    H = ctypes.c_void_p
    sig = {
        "arl2_create": ([ctypes.POINTER(Arl2Config), P, ctypes.POINTER(H)], I),
        "arl2_frame_forward": ([H, P, P, P, P, P, I, P, P], I),
        "arl2_frame_forward_host": ([H, P, P, P, P, P, I, P, P], I),
        "arl2_state_reset": ([H, P], I),
        "arl2_state_get": ([H, P, P], I),
        "arl2_state_set": ([H, P, P], I),
        "arl2_phi_apply": ([H, I, P, P, P], I),
        "arl2_device_status": ([H, P], I),
        "arl2_device_bytes": ([H], S),
        "arl2_kernel_launches": ([H], ctypes.c_ulonglong),
        "arl2_state_update_noalloc": ([I, I, I, I, I, P, P, P, P, P, P, P, P], I),
        "arl2_destroy": ([H], None),
        "arl2_status_string": ([I], ctypes.c_char_p),
        "arl2_version": ([], I),
        "arl2_gates_apply": ([H, P, P, P, P], I),
        "arl2_frame_forward_hidden": ([H, P, P, P, P, I, P, P], I),
        "arl2_frame_forward_hidden_host": ([H, P, P, P, P, I, P, P], I),
        "arl2_selftest_wait_timeout": ([H, ctypes.c_uint, P], I),
        "arl2_kv_create": ([ctypes.POINTER(Arl2KvConfig), P, ctypes.POINTER(H)], I),
        "arl2_kv_frame_forward": ([H, P, P, P, I, P, P], I),
        "arl2_kv_frame_forward_host": ([H, P, P, P, I, P, P], I),
        "arl2_kv_reset": ([H], I),
        "arl2_kv_frames": ([H], I),
        "arl2_kv_cache_get": ([H, P, P, P], I),
        "arl2_kv_cache_set": ([H, P, P, I, P], I),
        "arl2_kv_device_status": ([H, P], I),
        "arl2_kv_device_bytes": ([H], S),
        "arl2_kv_cache_bytes": ([H], S),
        "arl2_kv_kernel_launches": ([H], ctypes.c_ulonglong),
        "arl2_kv_destroy": ([H], None),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()


class Arl2Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_lib.arl2_status_string(status).decode()} ({status})")


def _check(status: int, what: str) -> None:
    if status != ARL2_OK:
        raise Arl2Error(status, what)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def state_update_noalloc(k, v, w_k, w_v, alpha, beta, state, stream=None) -> None:
    """arl2_state_update_noalloc: the clean-pass update in place on a
    caller-owned fp32 state [B, H, d, d], allocating no device memory."""
    B, L, H, d = k.shape
    dt = ARL2_BF16 if k.dtype == torch.bfloat16 else ARL2_FP32
    _check(_lib.arl2_state_update_noalloc(B, H, d, L, dt, _ptr(k), _ptr(v), _ptr(w_k), _ptr(w_v),
                                          _ptr(alpha), _ptr(beta), _ptr(state), _stream(stream)),
           "arl2_state_update_noalloc")


def library_path() -> str:
    return LIB_PATH


def version() -> int:
    return _lib.arl2_version()


class Arl2Layer:
    """One ARL2 hybrid attention layer: B streams, H heads, width d, L tokens.

    w_q, w_k, w_v: CUDA tensors [H, d, d] in the layer dtype (bf16 or fp32),
    row = input feature.  The handle copies them and owns the fp32 state
    S [B, H, d, d] (zero at creation).  host_staging: 0 none, 1 staging
    buffers for the host-buffer calls, 2 two sets of them whose copies
    overlap the neighbouring calls' work (arl2_config.host_staging).
    """

    def __init__(self, batch: int, heads: int, head_dim: int, tokens: int, w_q, w_k, w_v, *,
                 dtype: torch.dtype = torch.bfloat16, softmax_scale: float = 0.0,
                 host_staging: int = 0, impl: str = "auto", max_ctas: int = 0,
                 gating: str = "headwise", access: str = "frame", gate_weights=None, stream=None):
        if dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("dtype must be torch.bfloat16 or torch.float32")
        for w in (w_q, w_k, w_v):
            if not (w.is_cuda and w.is_contiguous() and w.dtype == dtype):
                raise ValueError("feature maps must be contiguous CUDA tensors of the layer dtype")
            if tuple(w.shape) != (heads, head_dim, head_dim):
                raise ValueError("feature maps must be [H, d, d]")
        self.shape = (batch, tokens, heads, head_dim)
        self.dtype = dtype
        self.device = w_q.device
        self.hidden_dim = 0
        w_gate = b_gate = None
        if gate_weights is not None:
            w_gate, b_gate = gate_weights
            if not (w_gate.is_cuda and w_gate.is_contiguous() and w_gate.dtype == dtype and w_gate.dim() == 2
                    and w_gate.shape[1] == 2 * heads):
                raise ValueError("gate weights must be a contiguous CUDA tensor [D, 2H] of the layer dtype")
            if not (b_gate.is_cuda and b_gate.is_contiguous() and b_gate.dtype == torch.float32
                    and tuple(b_gate.shape) == (2 * heads,)):
                raise ValueError("gate bias must be a contiguous fp32 CUDA tensor [2H]")
            self.hidden_dim = int(w_gate.shape[0])
        cfg = Arl2Config(batch, heads, head_dim, tokens,
                         ARL2_BF16 if dtype == torch.bfloat16 else ARL2_FP32,
                         w_q.data_ptr(), w_k.data_ptr(), w_v.data_ptr(), float(softmax_scale),
                         int(host_staging),
                         {"auto": ARL2_IMPL_AUTO, "simt": ARL2_IMPL_SIMT}[impl], int(max_ctas),
                         {"headwise": ARL2_GATE_HEADWISE, "elementwise": ARL2_GATE_ELEMENTWISE}[gating],
                         {"frame": ARL2_ACCESS_FRAME, "token": ARL2_ACCESS_TOKEN}[access],
                         self.hidden_dim, None if w_gate is None else w_gate.data_ptr(),
                         None if b_gate is None else b_gate.data_ptr())
        self.token_level = access == "token"
        self.alpha_shape = lambda B, H: (B, H, head_dim) if gating == "elementwise" else (B, H)
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(_lib.arl2_create(ctypes.byref(cfg), _stream(stream), ctypes.byref(h)), "arl2_create")
        self._h = h

    # -- helpers --------------------------------------------------------
    def _tok(self, t, name):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == self.dtype):
            raise ValueError(f"{name} must be a contiguous CUDA tensor of the layer dtype")
        if tuple(t.shape) != self.shape:
            raise ValueError(f"{name} must have shape {self.shape}")
        return t

    @property
    def handle(self):
        if self._h is None:
            raise RuntimeError("layer is closed")
        return self._h

    # -- C ABI calls ----------------------------------------------------
    def forward(self, q, k, v, alpha=None, beta=None, clean_pass: bool = False, out=None,
                stream=None):
        """One denoising pass; returns out [B, L, H, d].  alpha [B, H] ([B, H, d]
        with elementwise gating) and beta [B, H, L] (fp32 CUDA) are needed on
        the clean pass only."""
        self._tok(q, "q"), self._tok(k, "k"), self._tok(v, "v")
        if out is None:
            out = torch.empty_like(q)
        self._tok(out, "out")
        B, L, H, _ = self.shape
        gates = clean_pass or self.token_level  # token-level access reads the gates on every pass
        if gates:
            if alpha is None or beta is None:
                raise ValueError("this pass needs alpha and beta")
            if not (alpha.is_cuda and alpha.dtype == torch.float32 and alpha.is_contiguous()
                    and tuple(alpha.shape) == self.alpha_shape(B, H)):
                raise ValueError(f"alpha must be a contiguous fp32 CUDA tensor {list(self.alpha_shape(B, H))}")
            if not (beta.is_cuda and beta.dtype == torch.float32 and beta.is_contiguous()
                    and tuple(beta.shape) == (B, H, L)):
                raise ValueError("beta must be a contiguous fp32 CUDA tensor [B, H, L]")
        _check(_lib.arl2_frame_forward(self.handle, _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(alpha) if gates else None,
                                       _ptr(beta) if gates else None,
                                       1 if clean_pass else 0, _ptr(out), _stream(stream)),
               "arl2_frame_forward")
        return out

    def forward_host(self, q, k, v, alpha, beta, clean_pass: bool, out, stream=None):
        """arl2_frame_forward_host: q, k, v, alpha, beta, out are host (pinned) tensors."""
        for t in (q, k, v, out):
            if t.is_cuda or not t.is_contiguous() or tuple(t.shape) != self.shape or t.dtype != self.dtype:
                raise ValueError("host token tensors must be contiguous CPU tensors of the layer shape")
        gates = clean_pass or self.token_level
        if gates and (alpha is None or beta is None or alpha.is_cuda or beta.is_cuda):
            raise ValueError("this pass needs host alpha and beta")
        _check(_lib.arl2_frame_forward_host(self.handle, _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(alpha) if gates else None,
                                            _ptr(beta) if gates else None,
                                            1 if clean_pass else 0, _ptr(out), _stream(stream)),
               "arl2_frame_forward_host")
        return out

    def _hidden(self, x):
        B, L, _, _ = self.shape
        if not (x.is_cuda and x.is_contiguous() and x.dtype == self.dtype
                and tuple(x.shape) == (B, L, self.hidden_dim)):
            raise ValueError(f"x must be a contiguous CUDA tensor [B, L, D] = {[B, L, self.hidden_dim]}")
        return x

    def gates_apply(self, x, stream=None):
        """arl2_gates_apply: (alpha [B, H], beta [B, H, L]) projected from the
        hidden states x [B, L, D]."""
        B, L, H, _ = self.shape
        self._hidden(x)
        alpha = torch.empty(B, H, dtype=torch.float32, device=self.device)
        beta = torch.empty(B, H, L, dtype=torch.float32, device=self.device)
        _check(_lib.arl2_gates_apply(self.handle, _ptr(x), _ptr(alpha), _ptr(beta), _stream(stream)),
               "arl2_gates_apply")
        return alpha, beta

    def forward_hidden(self, q, k, v, x=None, clean_pass: bool = False, out=None, stream=None):
        """One pass with the gates projected from x [B, L, D] (needed on the
        clean pass, and on every pass with token-level access)."""
        self._tok(q, "q"), self._tok(k, "k"), self._tok(v, "v")
        if out is None:
            out = torch.empty_like(q)
        self._tok(out, "out")
        if x is not None:
            self._hidden(x)
        elif clean_pass or self.token_level:
            raise ValueError("this pass needs the hidden states x")
        _check(_lib.arl2_frame_forward_hidden(self.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(x),
                                              1 if clean_pass else 0, _ptr(out), _stream(stream)),
               "arl2_frame_forward_hidden")
        return out

    def forward_hidden_host(self, q, k, v, x, clean_pass: bool, out, stream=None):
        """arl2_frame_forward_hidden_host: q, k, v, x, out are host (pinned) tensors."""
        B, L, _, _ = self.shape
        for t in (q, k, v, out):
            if t.is_cuda or not t.is_contiguous() or tuple(t.shape) != self.shape or t.dtype != self.dtype:
                raise ValueError("host token tensors must be contiguous CPU tensors of the layer shape")
        if x is not None and (x.is_cuda or not x.is_contiguous() or x.dtype != self.dtype
                              or tuple(x.shape) != (B, L, self.hidden_dim)):
            raise ValueError("x must be a contiguous CPU tensor [B, L, D] of the layer dtype")
        _check(_lib.arl2_frame_forward_hidden_host(self.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(x),
                                                   1 if clean_pass else 0, _ptr(out), _stream(stream)),
               "arl2_frame_forward_hidden_host")
        return out

    def state_reset(self, stream=None) -> None:
        _check(_lib.arl2_state_reset(self.handle, _stream(stream)), "arl2_state_reset")

    def state_get(self, out=None, stream=None):
        B, _, H, d = self.shape
        if out is None:
            out = torch.empty(B, H, d, d, dtype=torch.float32, device=self.device)
        _check(_lib.arl2_state_get(self.handle, _ptr(out), _stream(stream)), "arl2_state_get")
        return out

    def state_set(self, src, stream=None) -> None:
        B, _, H, d = self.shape
        if not (src.is_cuda and src.dtype == torch.float32 and src.is_contiguous()
                and tuple(src.shape) == (B, H, d, d)):
            raise ValueError("state must be a contiguous fp32 CUDA tensor [B, H, d, d]")
        _check(_lib.arl2_state_set(self.handle, _ptr(src), _stream(stream)), "arl2_state_set")

    def phi_apply(self, which: str, x, out=None, stream=None):
        """which in {"q", "k", "v"}: x W_q, rownorm(x W_k) or x W_v."""
        self._tok(x, "x")
        if out is None:
            out = torch.empty_like(x)
        self._tok(out, "out")
        _check(_lib.arl2_phi_apply(self.handle, {"q": 0, "k": 1, "v": 2}[which], _ptr(x), _ptr(out),
                                   _stream(stream)), "arl2_phi_apply")
        return out

    def selftest_wait_timeout(self, limit_us: int, stream=None) -> None:
        """arl2_selftest_wait_timeout: a bounded wait on a word nothing sets,
        which gives up after limit_us and sets the error word."""
        _check(_lib.arl2_selftest_wait_timeout(self.handle, int(limit_us), _stream(stream)),
               "arl2_selftest_wait_timeout")

    def device_status(self, stream=None) -> int:
        """Synchronise and return the device status code (0, or ARL2_ERR_TIMEOUT)."""
        return _lib.arl2_device_status(self.handle, _stream(stream))

    def device_bytes(self) -> int:
        return int(_lib.arl2_device_bytes(self.handle))

    def kernel_launches(self) -> int:
        """Kernels this layer has enqueued (or recorded into a graph) so far."""
        return int(_lib.arl2_kernel_launches(self.handle))

    def close(self) -> None:
        if getattr(self, "_h", None) is not None:
            _lib.arl2_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()


class TeacherLayer:
    """The softmax teacher layer with a KV cache (arl2_kv_* in the C ABI).

    One pass of frame N: out = softmax([Q Kc^T, Q K^T] scale) [Vc; V], where
    (Kc, Vc) are the clean keys/values of frames 0..N-1 (the cache) and
    (K, V) the pass's own; a clean pass appends its k, v.  The cache holds up
    to max_frames frames, allocated at creation.
    """

    def __init__(self, batch: int, heads: int, head_dim: int, tokens: int, max_frames: int, *,
                 dtype: torch.dtype = torch.bfloat16, softmax_scale: float = 0.0,
                 host_staging: bool = False, impl: str = "auto", max_ctas: int = 0,
                 device=None, stream=None):
        if dtype not in (torch.bfloat16, torch.float32):
            raise ValueError("dtype must be torch.bfloat16 or torch.float32")
        self.shape = (batch, tokens, heads, head_dim)
        self.dtype = dtype
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        cfg = Arl2KvConfig(batch, heads, head_dim, tokens, max_frames,
                           ARL2_BF16 if dtype == torch.bfloat16 else ARL2_FP32, float(softmax_scale),
                           1 if host_staging else 0,
                           {"auto": ARL2_IMPL_AUTO, "simt": ARL2_IMPL_SIMT}[impl], int(max_ctas))
        h = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            _check(_lib.arl2_kv_create(ctypes.byref(cfg), _stream(stream), ctypes.byref(h)), "arl2_kv_create")
        self._h = h

    def _tok(self, t, name):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == self.dtype):
            raise ValueError(f"{name} must be a contiguous CUDA tensor of the layer dtype")
        if tuple(t.shape) != self.shape:
            raise ValueError(f"{name} must have shape {self.shape}")
        return t

    @property
    def handle(self):
        if self._h is None:
            raise RuntimeError("layer is closed")
        return self._h

    def forward(self, q, k, v, clean_pass: bool = False, out=None, stream=None):
        """One pass of the current frame; returns out [B, L, H, d]."""
        self._tok(q, "q"), self._tok(k, "k"), self._tok(v, "v")
        if out is None:
            out = torch.empty_like(q)
        self._tok(out, "out")
        _check(_lib.arl2_kv_frame_forward(self.handle, _ptr(q), _ptr(k), _ptr(v), 1 if clean_pass else 0,
                                          _ptr(out), _stream(stream)), "arl2_kv_frame_forward")
        return out

    def forward_host(self, q, k, v, clean_pass: bool, out, stream=None):
        """arl2_kv_frame_forward_host: q, k, v, out are host (pinned) tensors."""
        for t in (q, k, v, out):
            if t.is_cuda or not t.is_contiguous() or tuple(t.shape) != self.shape or t.dtype != self.dtype:
                raise ValueError("host token tensors must be contiguous CPU tensors of the layer shape")
        _check(_lib.arl2_kv_frame_forward_host(self.handle, _ptr(q), _ptr(k), _ptr(v), 1 if clean_pass else 0,
                                               _ptr(out), _stream(stream)), "arl2_kv_frame_forward_host")
        return out

    def reset(self) -> None:
        _check(_lib.arl2_kv_reset(self.handle), "arl2_kv_reset")

    def frames(self) -> int:
        return int(_lib.arl2_kv_frames(self.handle))

    def cache_get(self, stream=None):
        """(k, v) in the cache: [B, frames * L, H, d] each."""
        B, L, H, d = self.shape
        n = self.frames() * L
        kc = torch.empty(B, n, H, d, dtype=self.dtype, device=self.device)
        vc = torch.empty_like(kc)
        _check(_lib.arl2_kv_cache_get(self.handle, _ptr(kc), _ptr(vc), _stream(stream)), "arl2_kv_cache_get")
        return kc, vc

    def cache_set(self, k, v, stream=None) -> None:
        """Load the cache from (k, v), [B, n * L, H, d] each (n whole frames)."""
        B, L, H, d = self.shape
        for t in (k, v):
            if not (t.is_cuda and t.is_contiguous() and t.dtype == self.dtype and t.dim() == 4
                    and t.shape[0] == B and t.shape[2:] == (H, d) and t.shape[1] % L == 0):
                raise ValueError("cache tensors must be contiguous CUDA tensors [B, n * L, H, d]")
        if k.shape != v.shape:
            raise ValueError("k and v must have the same shape")
        _check(_lib.arl2_kv_cache_set(self.handle, _ptr(k), _ptr(v), k.shape[1] // L, _stream(stream)),
               "arl2_kv_cache_set")

    def device_status(self, stream=None) -> int:
        return _lib.arl2_kv_device_status(self.handle, _stream(stream))

    def device_bytes(self) -> int:
        return int(_lib.arl2_kv_device_bytes(self.handle))

    def cache_bytes(self) -> int:
        return int(_lib.arl2_kv_cache_bytes(self.handle))

    def kernel_launches(self) -> int:
        return int(_lib.arl2_kv_kernel_launches(self.handle))

    def close(self) -> None:
        if getattr(self, "_h", None) is not None:
            _lib.arl2_kv_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()
