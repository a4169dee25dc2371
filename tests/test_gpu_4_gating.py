"""GPU parity of elementwise gating: one forget gate per key feature,
S_N = diag(alpha) S_{N-1} + K'^T diag(beta)(V' - K' S_{N-1}) (atlas summary,
"Surprising findings": elementwise vs headwise gating), through the C ABI,
against the oracle; tensor-core and SIMT kernels.
"""
import dataclasses

import pytest
import torch

import workloads
from gpu_harness import make_layer, run_and_check

pytestmark = pytest.mark.gpu

BASE = workloads.WORKLOADS["480p_bf16"]


def small(L, B=2, H=2, frames=3, passes=2):
    return dataclasses.replace(BASE, name=f"bf16_L{L}", batch=B, heads=H, tokens=L, frames=frames,
                               passes=passes)


@pytest.mark.parametrize("L", [17, 300])
def test_tc_elementwise_gating_matches_oracle(L):
    run_and_check(small(L), gating="elementwise")


def test_tc_elementwise_gating_on_480p_frames():
    run_and_check(BASE, frames=2, gating="elementwise",
                  full_rows=lambda f, p: p == BASE.passes - 1, sample_rows=256)


def test_simt_elementwise_gating_matches_oracle():
    run_and_check(workloads.WORKLOADS["tiny_fp32"], impl="simt", gating="elementwise")
    run_and_check(small(40, frames=2), impl="simt", gating="elementwise")


def test_uniform_elementwise_gate_equals_headwise_gate_bit_exact():
    w = small(260, B=2, H=2)
    lay_h, _ = make_layer(w)
    lay_e, _ = make_layer(w, gating="elementwise")
    try:
        for f in range(3):
            a, b = workloads.frame_gates(w, 0, f)
            ae = a[:, :, None].expand(w.batch, w.heads, w.head_dim).contiguous()
            q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, f, 1))
            oh = lay_h.forward(q, k, v, a.cuda(), b.cuda(), clean_pass=True)
            oe = lay_e.forward(q, k, v, ae.cuda(), b.cuda(), clean_pass=True)
            assert torch.equal(oh, oe)
            assert torch.equal(lay_h.state_get(), lay_e.state_get())
        assert lay_h.device_status() == 0 and lay_e.device_status() == 0
    finally:
        lay_h.close()
        lay_e.close()


def test_host_entry_carries_the_elementwise_gates():
    w = small(200, B=1)
    lay_h, _ = make_layer(w, host_staging=True, gating="elementwise")
    lay_d, _ = make_layer(w, gating="elementwise")
    try:
        for f in range(2):
            q, k, v = workloads.pass_inputs(w, 0, f, 1)
            a, b = workloads.frame_gates_elementwise(w, 0, f)
            out_h = torch.empty_like(q).pin_memory()
            lay_h.forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), a.pin_memory(),
                               b.pin_memory(), True, out_h)
            torch.cuda.synchronize()
            od = lay_d.forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), clean_pass=True)
            assert torch.equal(out_h, od.cpu())
        assert torch.equal(lay_h.state_get(), lay_d.state_get())
    finally:
        lay_h.close()
        lay_d.close()


def test_alpha_shape_follows_the_gating():
    w = small(64, B=1)
    lay, _ = make_layer(w, gating="elementwise")
    try:
        q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, 0, 1))
        a, b = workloads.frame_gates(w, 0, 0)  # headwise shape: rejected
        with pytest.raises(ValueError):
            lay.forward(q, k, v, a.cuda(), b.cuda(), clean_pass=True)
    finally:
        lay.close()
