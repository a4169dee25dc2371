"""CPU oracle of the ARL2 hybrid attention layer (fp64), for tests only.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never calls it, and it never calls the CUDA library.

The arithmetic lives in ``arl2_oracle.c`` (plain C, fp64, one loop nest per
step of the method).  This module compiles it with gcc on first use and
marshals numpy arrays in and out.  Inputs are upcast to float64 from exactly
the values given to the GPU (bf16- or fp32-rounded).

Method source: "Attend Locally, Remember Linearly" technical summary,
section 2.1 (hybrid decomposition, phi maps, state update, inter read) and
section 2.2 (frame-level access, clean-pass updates).  The softmax teacher
layer with a KV cache (teacher_pass) follows section 1 ("KV Cache Growth")
and section 4 ("Efficiency"): the attention the hybrid layer replaces.  The
gate projections (gate_projection) follow section 2.1 ("State Update").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "arl2_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile arl2_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", _SRC, "-o", _LIB + ".tmp", "-lm"]
    subprocess.check_call(cmd)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            D = ctypes.c_double
            lib.arl2_oracle_pass.argtypes = [I, I, I, I, D, P, P, P, P, P, P, P, P, I, P, P]
            lib.arl2_oracle_rows.argtypes = [I, I, I, I, D, P, P, P, P, P, I, P, P, P]
            lib.arl2_oracle_state_update.argtypes = [I, I, I, I, P, P, P, P, P, P, P]
            lib.arl2_oracle_state_update_gated.argtypes = [I, I, I, I, P, P, P, P, P, I, P, P]
            lib.arl2_oracle_phi.argtypes = [I, I, I, I, P, P, I, P]
            lib.arl2_oracle_pass_token_level.argtypes = [I, I, I, I, D, P, P, P, P, P, P, P, I, P, I,
                                                         P, P]
            lib.arl2_oracle_teacher_pass.argtypes = [I, I, I, I, I, D, P, P, P, P, P, P]
            lib.arl2_oracle_teacher_rows.argtypes = [I, I, I, I, I, D, P, P, P, P, P, I, P, P, P]
            lib.arl2_oracle_gate_projection.argtypes = [I, I, I, I, P, P, P, P, P]
            for f in (lib.arl2_oracle_pass, lib.arl2_oracle_rows,
                      lib.arl2_oracle_state_update, lib.arl2_oracle_state_update_gated,
                      lib.arl2_oracle_phi, lib.arl2_oracle_pass_token_level,
                      lib.arl2_oracle_teacher_pass, lib.arl2_oracle_teacher_rows,
                      lib.arl2_oracle_gate_projection):
                f.restype = I
            _lib = lib
    return _lib


def f64(x) -> np.ndarray:
    """Exact upcast of a torch tensor or array to a contiguous float64 array."""
    if hasattr(x, "detach"):
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dims(q):
    B, L, H, d = q.shape
    return B, H, d, L


def default_scale(d: int) -> float:
    """Softmax scale 1/sqrt(d) (the tiny workload's 'sqrt(16)')."""
    return 1.0 / float(np.sqrt(d))


def frame_pass(q, k, v, w_q, w_k, w_v, alpha, beta, S, clean: bool, scale=None):
    """One pass.  Returns (out [B,L,H,d], S_after [B,H,d,d]); S is not modified."""
    q, k, v = f64(q), f64(k), f64(v)
    w_q, w_k, w_v = f64(w_q), f64(w_k), f64(w_v)
    B, H, d, L = _dims(q)
    alpha = f64(alpha) if alpha is not None else np.ones((B, H))
    beta = f64(beta) if beta is not None else np.zeros((B, H, L))
    S2 = f64(S).copy()
    out = np.zeros_like(q)
    sc = default_scale(d) if scale is None else float(scale)
    per_key = alpha.ndim == 3  # elementwise gating: the update runs separately
    rc = _load().arl2_oracle_pass(B, H, d, L, sc, _p(q), _p(k), _p(v), _p(w_q), _p(w_k),
                                  _p(w_v), _p(alpha), _p(beta), int(bool(clean) and not per_key),
                                  _p(S2), _p(out))
    if rc != 0:
        raise RuntimeError("arl2_oracle_pass failed")
    if clean and per_key:
        S2 = state_update(k, v, w_k, w_v, alpha, beta, S2)
    return out, S2


def frame_pass_token_level(q, k, v, w_q, w_k, w_v, alpha, beta, S, clean: bool, scale=None):
    """One pass with token-level (sequential) state access, the ablation the
    pages compare with frame-level access: token i reads the state left by
    tokens 0..i-1, then updates it (delta rule); the forget gate acts once,
    with token 0's update.  alpha [B, H] (or [B, H, d] per key feature) and
    beta [B, H, L] are used on every pass; only a clean pass keeps the final
    state.  Returns (out, S_after); S is not modified."""
    q, k, v = f64(q), f64(k), f64(v)
    w_q, w_k, w_v = f64(w_q), f64(w_k), f64(w_v)
    B, H, d, L = _dims(q)
    alpha, beta = f64(alpha), f64(beta)
    per_key = alpha.ndim == 3
    if alpha.shape != ((B, H, d) if per_key else (B, H)) or beta.shape != (B, H, L):
        raise ValueError("alpha/beta shape")
    S2 = f64(S).copy()
    out = np.zeros_like(q)
    sc = default_scale(d) if scale is None else float(scale)
    rc = _load().arl2_oracle_pass_token_level(B, H, d, L, sc, _p(q), _p(k), _p(v), _p(w_q), _p(w_k),
                                              _p(w_v), _p(alpha), int(per_key), _p(beta),
                                              int(bool(clean)), _p(S2), _p(out))
    if rc != 0:
        raise RuntimeError("arl2_oracle_pass_token_level failed")
    return out, S2


def rows(q, k, v, w_q, S, rows_b, rows_t, scale=None):
    """Outputs of selected token rows: returns [nrows, H, d]."""
    q, k, v, w_q, S = f64(q), f64(k), f64(v), f64(w_q), f64(S)
    B, H, d, L = _dims(q)
    rb = np.ascontiguousarray(np.asarray(rows_b, dtype=np.int32))
    rt = np.ascontiguousarray(np.asarray(rows_t, dtype=np.int32))
    n = int(rb.shape[0])
    out = np.zeros((n, H, d))
    sc = default_scale(d) if scale is None else float(scale)
    rc = _load().arl2_oracle_rows(B, H, d, L, sc, _p(q), _p(k), _p(v), _p(w_q), _p(S), n,
                                  _p(rb), _p(rt), _p(out))
    if rc != 0:
        raise RuntimeError("arl2_oracle_rows failed")
    return out


def state_update(k, v, w_k, w_v, alpha, beta, S):
    """Clean-pass update; returns the new state (input S untouched).

    alpha [B, H] is the headwise forget gate (S_N = alpha S + ...); alpha
    [B, H, d] gates each key feature (elementwise gating, S_N = diag(alpha) S
    + ...), the variant the atlas summary's "Surprising findings" compares.
    """
    k, v, w_k, w_v = f64(k), f64(v), f64(w_k), f64(w_v)
    alpha, beta = f64(alpha), f64(beta)
    B, H, d, L = _dims(k)
    per_key = alpha.ndim == 3
    if alpha.shape != ((B, H, d) if per_key else (B, H)):
        raise ValueError(f"alpha shape {alpha.shape}")
    S2 = f64(S).copy()
    rc = _load().arl2_oracle_state_update_gated(B, H, d, L, _p(k), _p(v), _p(w_k), _p(w_v),
                                                _p(alpha), int(per_key), _p(beta), _p(S2))
    if rc != 0:
        raise RuntimeError("arl2_oracle_state_update_gated failed")
    return S2


def phi(x, w, l2norm: bool):
    """x' = x W[h] per head, optionally with L2-normalised rows."""
    x, w = f64(x), f64(w)
    B, H, d, L = _dims(x)
    out = np.zeros_like(x)
    rc = _load().arl2_oracle_phi(B, H, d, L, _p(x), _p(w), int(bool(l2norm)), _p(out))
    if rc != 0:
        raise RuntimeError("arl2_oracle_phi failed")
    return out


def _cache(cache_k, cache_v, B, H, d):
    if cache_k is None:
        return np.zeros((B, 0, H, d)), np.zeros((B, 0, H, d))
    kc, vc = f64(cache_k), f64(cache_v)
    if kc.shape != vc.shape or kc.shape[0] != B or kc.shape[2:] != (H, d):
        raise ValueError(f"cache shape {kc.shape} / {vc.shape}")
    return kc, vc


def teacher_pass(q, k, v, cache_k=None, cache_v=None, scale=None):
    """Softmax teacher layer with a KV cache, one pass of one frame:
    O = softmax([Q Kc^T, Q K^T] scale) [Vc; V], the frame's queries attending
    to the clean keys/values of every earlier frame (cache_k, cache_v
    [B, Lc, H, d], frames in order; None for the first frame) and,
    bidirectionally, to their own.  Returns out [B, L, H, d].  The caller
    appends a clean pass's k, v to the cache (teacher_append)."""
    q, k, v = f64(q), f64(k), f64(v)
    B, H, d, L = _dims(q)
    kc, vc = _cache(cache_k, cache_v, B, H, d)
    Lc = int(kc.shape[1])
    out = np.zeros_like(q)
    sc = default_scale(d) if scale is None else float(scale)
    rc = _load().arl2_oracle_teacher_pass(B, H, d, L, Lc, sc, _p(q), _p(k), _p(v), _p(kc), _p(vc),
                                          _p(out))
    if rc != 0:
        raise RuntimeError("arl2_oracle_teacher_pass failed")
    return out


def teacher_rows(q, k, v, cache_k, cache_v, rows_b, rows_t, scale=None):
    """teacher_pass for selected token rows only: returns [nrows, H, d]."""
    q, k, v = f64(q), f64(k), f64(v)
    B, H, d, L = _dims(q)
    kc, vc = _cache(cache_k, cache_v, B, H, d)
    Lc = int(kc.shape[1])
    rb = np.ascontiguousarray(np.asarray(rows_b, dtype=np.int32))
    rt = np.ascontiguousarray(np.asarray(rows_t, dtype=np.int32))
    n = int(rb.shape[0])
    out = np.zeros((n, H, d))
    sc = default_scale(d) if scale is None else float(scale)
    rc = _load().arl2_oracle_teacher_rows(B, H, d, L, Lc, sc, _p(q), _p(k), _p(v), _p(kc), _p(vc),
                                          n, _p(rb), _p(rt), _p(out))
    if rc != 0:
        raise RuntimeError("arl2_oracle_teacher_rows failed")
    return out


def teacher_append(cache_k, cache_v, k, v):
    """The cache after a clean pass: (cache_k; k), (cache_v; v) along tokens."""
    k, v = f64(k), f64(v)
    if cache_k is None:
        return k.copy(), v.copy()
    return np.concatenate([f64(cache_k), k], axis=1), np.concatenate([f64(cache_v), v], axis=1)


def gate_projection(x, w, bias):
    """Gates from the layer's hidden states (the reading of "learned per-token
    projections", technical summary section 2.1): per token and head the
    logits a = x w[:, h] + bias[h] and g = x w[:, H + h] + bias[H + h];
    beta = sigmoid(g) per token, alpha = sigmoid(mean over the frame's tokens
    of a).  x [B, L, D], w [D, 2H], bias [2H].  Returns (alpha [B, H],
    beta [B, H, L])."""
    x, w, bias = f64(x), f64(w), f64(bias)
    B, L, D = x.shape
    if w.ndim != 2 or w.shape[0] != D or w.shape[1] % 2 or bias.shape != (w.shape[1],):
        raise ValueError(f"gate weights {w.shape} / bias {bias.shape} for hidden size {D}")
    H = w.shape[1] // 2
    alpha = np.zeros((B, H))
    beta = np.zeros((B, H, L))
    rc = _load().arl2_oracle_gate_projection(B, L, D, H, _p(x), _p(w), _p(bias), _p(alpha), _p(beta))
    if rc != 0:
        raise RuntimeError("arl2_oracle_gate_projection failed")
    return alpha, beta


def zero_state(B: int, H: int, d: int) -> np.ndarray:
    return np.zeros((B, H, d, d))


def max_abs_rel(x, ref) -> float:
    """max_i |x_i - ref_i| / max(max_i |ref_i|, 1e-30), per tensor."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = max(float(np.max(np.abs(ref))) if ref.size else 0.0, 1e-30)
    return float(np.max(np.abs(x - ref))) / den if ref.size else 0.0
