"""GPU parity of token-level (sequential) state access, the ablation of the
technical summary's §2.2 "Frame-Level Access": token i reads the state left
by tokens 0..i-1 and then updates it (delta rule), the forget gate acting
once with token 0; every pass reads through its own sequential states and
only the clean pass keeps the final one.  Compared through the C ABI with the
oracle's plain token-by-token loop, on the tensor-core (intra) + fp32 chunked
scan path and on the all-SIMT path.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_harness import TOL, err, make_layer

pytestmark = pytest.mark.gpu

BASE = workloads.WORKLOADS["480p_bf16"]


def small(L, B=2, H=2, frames=3, passes=2):
    return dataclasses.replace(BASE, name=f"bf16_L{L}", batch=B, heads=H, tokens=L, frames=frames,
                               passes=passes)


def run_token_level(w, impl="auto", gating="headwise", frames=None):
    tol = TOL[w.dtype]
    lay, (wq, wk, wv) = make_layer(w, impl=impl, gating=gating, access="token")
    gates = workloads.frame_gates_elementwise if gating == "elementwise" else workloads.frame_gates
    S_ref = oracle.zero_state(w.batch, w.heads, w.head_dim)
    worst = 0.0
    try:
        for f in range(w.frames if frames is None else frames):
            alpha, beta = gates(w, 0, f)
            a_d, b_d = alpha.cuda(), beta.cuda()
            for p in range(w.passes):
                q, k, v = workloads.pass_inputs(w, 0, f, p)
                clean = workloads.is_clean(w, p)
                out = lay.forward(q.cuda(), k.cuda(), v.cuda(), a_d, b_d, clean_pass=clean)
                ref, S_next = oracle.frame_pass_token_level(q, k, v, wq, wk, wv, alpha, beta, S_ref, clean)
                e = err(out.float().cpu().numpy(), ref)
                worst = max(worst, e)
                assert e <= tol, f"output frame {f} pass {p}: {e:.3e}"
                if clean:
                    S_ref = S_next
                    e = err(lay.state_get().cpu().numpy(), S_ref)
                    assert e <= tol, f"state after frame {f}: {e:.3e}"
                else:
                    assert np.array_equal(S_next, S_ref)
        assert lay.device_status() == 0
    finally:
        lay.close()
    return worst


@pytest.mark.parametrize("L", [1, 17, 64, 65, 300])
def test_token_level_tc_matches_oracle(L):
    run_token_level(small(L))


def test_token_level_elementwise_gating_matches_oracle():
    run_token_level(small(130), gating="elementwise")


def test_token_level_simt_matches_oracle():
    run_token_level(workloads.WORKLOADS["tiny_fp32"], impl="simt")
    run_token_level(dataclasses.replace(workloads.WORKLOADS["tiny_fp32"], tokens=100, head_dim=24,
                                        heads=3, batch=2, frames=2, passes=2), impl="simt")


def test_token_level_480p_frame():
    run_token_level(dataclasses.replace(BASE, passes=2), frames=1)


def test_token_level_with_one_token_equals_frame_level():
    w = small(1, frames=3)
    lay_t, _ = make_layer(w, access="token")
    lay_f, _ = make_layer(w)
    try:
        for f in range(3):
            a, b = workloads.frame_gates(w, 0, f)
            q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, f, 1))
            ot = lay_t.forward(q, k, v, a.cuda(), b.cuda(), clean_pass=True).float()
            of = lay_f.forward(q, k, v, a.cuda(), b.cuda(), clean_pass=True).float()
            assert float((ot - of).abs().max() / of.abs().max()) <= TOL["bf16"]
            st, sf = lay_t.state_get(), lay_f.state_get()
            assert float((st - sf).abs().max() / sf.abs().max()) <= TOL["bf16"]
    finally:
        lay_t.close()
        lay_f.close()
