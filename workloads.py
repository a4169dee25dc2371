"""Seeded synthetic inputs for the ARL2 hybrid attention layer.

This module only draws random numbers and rounds them to the run's dtype.
It holds none of the layer's arithmetic, so both the CUDA path and the CPU
oracle can take their inputs from it.

Workload shapes follow the video-DiT layer the ARL2 pages describe
("Attend Locally, Remember Linearly", P1 Technical Summary section 2.1 and
2.2): per latent frame, B independent streams, H heads of width d, and L
tokens per frame (the latent patch grid of one frame).

Value recipe (identical for every workload, per stream b and layer l):
  q, k, v       ~ N(0, 1), shape [B, L, H, d], one draw per (frame, pass)
  W_q, W_k, W_v = I + N(0, 0.02) per head, shape [H, d, d], one per layer
  alpha         = sigmoid(N(2, 0.5)), shape [B, H], one per frame
                  (elementwise gating: shape [B, H, d], same distribution)
  beta          = sigmoid(N(0, 1)) / L, shape [B, H, L], one per frame
  (gate projections: hidden states x ~ N(0, 1) [B, L, H d] per frame,
   w_gate ~ N(0, 1/(H d)) [H d, 2H], bias 2 (alpha) and -ln L (beta))
Every tensor is rounded to the run's dtype (q, k, v and W) or kept fp32
(alpha, beta); the same rounded values go to the GPU and to the oracle.

Seeds: stream b of layer l uses base = 20260519 + 1000 * l + b.  Each draw
gets its own generator, seeded by mixing (base, tag, frame, pass) with
splitmix64, so any frame can be regenerated without replaying the ones
before it.
"""
from __future__ import annotations

import dataclasses

import torch

SEED_BASE = 20260519
_MASK64 = (1 << 64) - 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one synthetic ARL2 workload."""

    name: str
    batch: int          # B: independent streams
    heads: int          # H
    head_dim: int       # d
    tokens: int         # L: tokens per latent frame
    frames: int         # latent frames per stream
    passes: int         # denoising passes per frame; the last one is clean
    dtype: str          # "bf16" or "fp32"
    layers: int = 1     # independent layers (own weights, gates and state)
    patches: tuple = () # (rows, cols) patch grid of one latent frame, if any

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 1, 16, 16, 4, 1, "fp32"),
    "480p_bf16": Workload("480p_bf16", 1, 12, 128, 1560, 21, 4, "bf16", patches=(30, 52)),
    "long_stream_bf16": Workload("long_stream_bf16", 1, 12, 128, 1560, 240, 4, "bf16", patches=(30, 52)),
    "720p_bf16": Workload("720p_bf16", 1, 12, 128, 3600, 30, 4, "bf16", patches=(45, 80)),
    "stack30_bf16": Workload("stack30_bf16", 4, 12, 128, 1560, 60, 4, "bf16", layers=30, patches=(30, 52)),
}


def _splitmix64(x: int) -> int:
    x = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = x
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def subseed(*parts: int) -> int:
    """Deterministic 63-bit seed from a tuple of integers."""
    h = 0x243F6A8885A308D3
    for p in parts:
        h = _splitmix64(h ^ (int(p) & _MASK64))
    return h & ((1 << 63) - 1)


def stream_base(layer: int, stream: int) -> int:
    return SEED_BASE + 1000 * layer + stream


_TAG_QKV, _TAG_GATES, _TAG_W, _TAG_GATES_ELEM, _TAG_HIDDEN, _TAG_W_GATE = 1, 2, 3, 4, 5, 6


def _gen(*parts: int, device: str = "cpu") -> torch.Generator:
    return torch.Generator(device=device).manual_seed(subseed(*parts))


def phi_weights(w: Workload, layer: int = 0):
    """W_q, W_k, W_v: [H, d, d] each, identity plus N(0, 0.02), in w's dtype.

    Row index = input feature, column index = output feature, so that the
    map is x' = x @ W[h] for a row vector x.
    """
    H, d = w.heads, w.head_dim
    g = _gen(stream_base(layer, 0), _TAG_W)
    eye = torch.eye(d, dtype=torch.float32)
    out = []
    for _ in range(3):
        m = eye + 0.02 * torch.randn(H, d, d, generator=g, dtype=torch.float32)
        out.append(m.to(w.torch_dtype).contiguous())
    return tuple(out)


def pass_inputs(w: Workload, layer: int, frame: int, pass_idx: int, device: str = "cpu"):
    """q, k, v for one (frame, pass): [B, L, H, d] each, in w's dtype.

    device="cuda" draws with the device generator (same seeds and
    distribution, different random stream; much faster for long streams).
    """
    B, L, H, d = w.batch, w.tokens, w.heads, w.head_dim
    q = torch.empty(B, L, H, d, dtype=torch.float32, device=device)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    for b in range(B):
        g = _gen(stream_base(layer, b), _TAG_QKV, frame, pass_idx, device=device)
        q[b] = torch.randn(L, H, d, generator=g, device=device)
        k[b] = torch.randn(L, H, d, generator=g, device=device)
        v[b] = torch.randn(L, H, d, generator=g, device=device)
    t = w.torch_dtype
    return q.to(t).contiguous(), k.to(t).contiguous(), v.to(t).contiguous()


def frame_gates(w: Workload, layer: int, frame: int):
    """alpha [B, H] and beta [B, H, L], fp32, for one frame."""
    B, L, H = w.batch, w.tokens, w.heads
    alpha = torch.empty(B, H, dtype=torch.float32)
    beta = torch.empty(B, H, L, dtype=torch.float32)
    for b in range(B):
        g = _gen(stream_base(layer, b), _TAG_GATES, frame)
        alpha[b] = torch.sigmoid(2.0 + 0.5 * torch.randn(H, generator=g))
        beta[b] = torch.sigmoid(torch.randn(H, L, generator=g)) / L
    return alpha.contiguous(), beta.contiguous()


def frame_gates_elementwise(w: Workload, layer: int, frame: int):
    """alpha [B, H, d] (one forget gate per key feature) and beta [B, H, L],
    fp32, for one frame: alpha = sigmoid(N(2, 0.5)) per entry, beta as in
    frame_gates (the same draw, so the two gatings share their beta)."""
    B, L, H, d = w.batch, w.tokens, w.heads, w.head_dim
    _, beta = frame_gates(w, layer, frame)
    alpha = torch.empty(B, H, d, dtype=torch.float32)
    for b in range(B):
        g = _gen(stream_base(layer, b), _TAG_GATES_ELEM, frame)
        alpha[b] = torch.sigmoid(2.0 + 0.5 * torch.randn(H, d, generator=g))
    return alpha.contiguous(), beta


def hidden_dim(w: Workload) -> int:
    """Width D of the hidden states the gate projections read: H d (the DiT's
    model width, 1536 for 12 heads of 128)."""
    return w.heads * w.head_dim


def hidden_states(w: Workload, layer: int, frame: int, device: str = "cpu"):
    """x [B, L, D] ~ N(0, 1) in w's dtype: the layer input the gate
    projections read (one draw per frame: the clean pass's)."""
    B, L, D = w.batch, w.tokens, hidden_dim(w)
    x = torch.empty(B, L, D, dtype=torch.float32, device=device)
    for b in range(B):
        g = _gen(stream_base(layer, b), _TAG_HIDDEN, frame, device=device)
        x[b] = torch.randn(L, D, generator=g, device=device)
    return x.to(w.torch_dtype).contiguous()


def gate_projection_weights(w: Workload, layer: int = 0):
    """w_gate [D, 2H] ~ N(0, 1/D) in w's dtype (logits of unit variance for
    x ~ N(0, 1)) and bias [2H] fp32: 2 for the alpha columns (alpha near
    sigmoid(2), as in frame_gates) and -ln(L) for the beta columns (beta
    near e^{N(0,1)} / L, the scale of frame_gates' sigmoid(N(0,1)) / L)."""
    import math
    H, D, L = w.heads, hidden_dim(w), w.tokens
    g = _gen(stream_base(layer, 0), _TAG_W_GATE)
    wg = (torch.randn(D, 2 * H, generator=g) / math.sqrt(D)).to(w.torch_dtype).contiguous()
    bias = torch.tensor([2.0] * H + [-math.log(L)] * H, dtype=torch.float32)
    return wg, bias


def is_clean(w: Workload, pass_idx: int) -> bool:
    """The last denoising pass of a frame is the clean pass."""
    return pass_idx == w.passes - 1


def describe(w: Workload) -> dict:
    return dataclasses.asdict(w)
