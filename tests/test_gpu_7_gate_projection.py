"""GPU parity of the gate projections: alpha and beta computed from the
layer's hidden states (technical summary §2.1 "State Update": learned
per-token projections; read as per-token linear logits, beta = sigmoid of
the token's logit, alpha = sigmoid of the frame's mean logit), alone
(arl2_gates_apply) and inside the layer's pass (arl2_frame_forward_hidden),
against the oracle.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_harness import TOL, err
from hybrid_softmax_gated_b200 import Arl2Layer

pytestmark = pytest.mark.gpu

BASE = workloads.WORKLOADS["480p_bf16"]
GATE_TOL = 1e-4  # fp32 accumulation over D features against fp64


def small(L, B=2, H=2, frames=3, passes=2):
    return dataclasses.replace(BASE, name=f"bf16_L{L}", batch=B, heads=H, tokens=L, frames=frames,
                               passes=passes)


def make(w, **kw):
    wq, wk, wv = workloads.phi_weights(w, 0)
    wg, bg = workloads.gate_projection_weights(w, 0)
    lay = Arl2Layer(w.batch, w.heads, w.head_dim, w.tokens, wq.cuda(), wk.cuda(), wv.cuda(),
                    dtype=w.torch_dtype, gate_weights=(wg.cuda(), bg.cuda()), **kw)
    return lay, (wq, wk, wv), (wg, bg)


@pytest.mark.parametrize("w,impl", [
    (BASE, "auto"), (small(17), "auto"), (small(100, B=3, H=5), "auto"), (small(300, B=2, H=20), "auto"),
    (small(260, B=2, H=40), "auto"), (BASE, "simt"), (small(100, B=3, H=5), "simt"),
    (workloads.WORKLOADS["tiny_fp32"], "simt"),
    (dataclasses.replace(workloads.WORKLOADS["tiny_fp32"], heads=40, head_dim=24, tokens=33, batch=2), "simt")],
    ids=["480p_tc", "L17_tc", "L100_B3_H5_tc", "L300_H20_tc", "L260_H40_tc", "480p_simt", "L100_simt",
         "tiny_fp32", "fp32_H40"])
def test_gates_apply_matches_oracle(w, impl):
    # bf16 layers on the default path use the tensor-core kernel (2H padded
    # to 32, 64 or 96 outputs; the hidden features split over a cluster),
    # impl="simt" and fp32 layers the SIMT kernel
    lay, _, (wg, bg) = make(w, impl=impl)
    try:
        for f in range(2):
            x = workloads.hidden_states(w, 0, f)
            a, b = lay.gates_apply(x.cuda())
            a_ref, b_ref = oracle.gate_projection(x, wg, bg)
            assert err(a.cpu().numpy(), a_ref) <= GATE_TOL
            assert err(b.cpu().numpy(), b_ref) <= GATE_TOL
            a2, b2 = lay.gates_apply(x.cuda())  # deterministic, and the count re-arms
            assert torch.equal(a, a2) and torch.equal(b, b2)
    finally:
        lay.close()


def run_hidden(w, frames=None, access="frame", full_rows=True):
    tol = TOL[w.dtype]
    lay, (wq, wk, wv), (wg, bg) = make(w, access=access)
    S_ref = oracle.zero_state(w.batch, w.heads, w.head_dim)
    pass_fn = oracle.frame_pass_token_level if access == "token" else oracle.frame_pass
    try:
        for f in range(w.frames if frames is None else frames):
            x = workloads.hidden_states(w, 0, f)
            alpha, beta = oracle.gate_projection(x, wg, bg)
            xd = x.cuda()
            for p in range(w.passes):
                q, k, v = workloads.pass_inputs(w, 0, f, p)
                clean = workloads.is_clean(w, p)
                needs_x = clean or access == "token"
                out = lay.forward_hidden(q.cuda(), k.cuda(), v.cuda(), xd if needs_x else None, clean_pass=clean)
                ref, S_next = pass_fn(q, k, v, wq, wk, wv, alpha, beta, S_ref, clean)
                e = err(out.float().cpu().numpy(), ref)
                assert e <= tol, f"output frame {f} pass {p}: {e:.3e}"
                if clean:
                    S_ref = S_next
                    e = err(lay.state_get().cpu().numpy(), S_ref)
                    assert e <= tol, f"state after frame {f}: {e:.3e}"
        assert lay.device_status() == 0
    finally:
        lay.close()


@pytest.mark.parametrize("L", [17, 300])
def test_forward_hidden_matches_oracle(L):
    run_hidden(small(L))


def test_forward_hidden_480p_frames():
    run_hidden(dataclasses.replace(BASE, passes=2), frames=2)


def test_forward_hidden_token_level_access():
    run_hidden(small(70, frames=2), access="token")


def test_forward_hidden_equals_forward_with_applied_gates():
    w = small(260)
    lay_h, _, _ = make(w)
    lay_g, _, _ = make(w)
    try:
        for f in range(3):
            x = workloads.hidden_states(w, 0, f).cuda()
            q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, f, 1))
            a, b = lay_g.gates_apply(x)
            oh = lay_h.forward_hidden(q, k, v, x, clean_pass=True)
            og = lay_g.forward(q, k, v, a, b, clean_pass=True)
            assert torch.equal(oh, og)
            assert torch.equal(lay_h.state_get(), lay_g.state_get())
            # a read-only pass needs no hidden states
            assert torch.equal(lay_h.forward_hidden(q, k, v), lay_g.forward(q, k, v))
    finally:
        lay_h.close()
        lay_g.close()


def test_gate_projection_launch_count():
    w = small(64)
    lay, _, _ = make(w)
    try:
        x = workloads.hidden_states(w, 0, 0).cuda()
        q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, 0, 0))
        n0 = lay.kernel_launches()
        lay.forward_hidden(q, k, v)
        n1 = lay.kernel_launches()
        lay.forward_hidden(q, k, v, x, clean_pass=True)
        n2 = lay.kernel_launches()
        assert n1 - n0 == 1           # attention only
        assert n2 - n1 == 1 + 1 + 2   # gates, attention, update
    finally:
        lay.close()


@pytest.mark.parametrize("staging", [1, 2])
def test_forward_hidden_host_entry_matches_device_entry(staging):
    """Host-buffer passes with projected gates, staging on the caller's stream
    (1) or double-buffered on the handle's copy streams (2), with no
    synchronisation between calls: every output and the state equal the
    device entry's bit for bit."""
    w = small(150, B=1)
    lay_h, _, _ = make(w, host_staging=staging)
    lay_d, _, _ = make(w)
    try:
        keep, outs, refs = [], [], []
        for f in range(2):
            x = workloads.hidden_states(w, 0, f)
            xh = x.pin_memory()
            for p in range(w.passes):
                q, k, v = workloads.pass_inputs(w, 0, f, p)
                clean = workloads.is_clean(w, p)
                qh, kh, vh = (t.pin_memory() for t in (q, k, v))
                out_h = torch.empty_like(q).pin_memory()
                lay_h.forward_hidden_host(qh, kh, vh, xh if clean else None, clean, out_h)
                keep.append((qh, kh, vh, xh))
                outs.append(out_h)
                refs.append(lay_d.forward_hidden(q.cuda(), k.cuda(), v.cuda(), x.cuda() if clean else None,
                                                 clean_pass=clean))
        torch.cuda.synchronize()
        for i, (o, r) in enumerate(zip(outs, refs)):
            assert torch.equal(o, r.cpu()), i
        assert torch.equal(lay_h.state_get(), lay_d.state_get())
    finally:
        lay_h.close()
        lay_d.close()
