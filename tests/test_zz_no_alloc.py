"""arl2_state_update_noalloc against the handle's clean-pass update and the oracle.

The no-allocation entry point serves callers that cannot call cudaMalloc
where they run the state update (a plugin that only receives fixed buffers
from its host framework, or a process whose caching allocator already holds
the device memory).  It updates a state buffer the caller owns, with its
scratch in a static device array inside the library.  Here it must give the
same state as arl2_frame_forward's clean pass on the same inputs, and as the
CPU oracle's state update carried from the zero state (technical summary
section 2.1 "State Update"), within the tolerance used everywhere else (1e-4
for fp32 data, 2e-2 for bf16), on two calls in a row, through the C ABI.

This file is collected last on purpose, so that a run stopping at its first
failure has already run every other test.  It needs nothing from the other
tests and also passes when run alone in a fresh process.
"""
import ctypes
import dataclasses

import pytest
import torch

import oracle
import workloads
import hybrid_softmax_gated_b200 as arl2

pytestmark = pytest.mark.gpu

CASES = {
    "fp32": (dataclasses.replace(workloads.WORKLOADS["tiny_fp32"], name="na_fp32", batch=2,
                                 heads=3, tokens=77, head_dim=32), 1e-4),
    "bf16": (dataclasses.replace(workloads.WORKLOADS["480p_bf16"], name="na_bf16", batch=1,
                                 heads=12, tokens=1560), 2e-2),
}


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_update_matches_handle_update_and_oracle_twice(case):
    w, tol = CASES[case]
    wq_h, wk_h, wv_h = workloads.phi_weights(w, 0)
    wq, wk, wv = (x.cuda() for x in (wq_h, wk_h, wv_h))
    S_ref = oracle.zero_state(w.batch, w.heads, w.head_dim)
    lay = arl2.Arl2Layer(w.batch, w.heads, w.head_dim, w.tokens, wq, wk, wv, dtype=w.torch_dtype)
    state = torch.zeros(w.batch, w.heads, w.head_dim, w.head_dim, dtype=torch.float32,
                        device="cuda")
    lib = ctypes.CDLL(arl2.library_path())
    lib.arl2_state_update_noalloc.restype = ctypes.c_int
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    dt = arl2.ARL2_BF16 if w.dtype == "bf16" else arl2.ARL2_FP32
    try:
        for frame in range(2):
            q_h, k_h, v_h = workloads.pass_inputs(w, 0, frame, 0)
            a_h, b_h = workloads.frame_gates(w, 0, frame)
            q, k, v = (x.cuda() for x in (q_h, k_h, v_h))
            a, b = a_h.cuda(), b_h.cuda()
            lay.forward(q, k, v, a, b, clean_pass=True)
            rc = lib.arl2_state_update_noalloc(
                w.batch, w.heads, w.head_dim, w.tokens, dt, _p(k), _p(v), _p(wk), _p(wv), _p(a),
                _p(b), _p(state), stream)
            assert rc == 0, arl2._lib.arl2_status_string(rc)
            torch.cuda.synchronize()
            ref = lay.state_get()
            e = float((state - ref).abs().max() / ref.abs().max())
            assert e <= tol, f"call {frame + 1}: max-abs-rel {e:.3e} > {tol} against the handle"
            S_ref = oracle.state_update(k_h, v_h, wk_h, wv_h, a_h, b_h, S_ref)
            e = oracle.max_abs_rel(state.cpu().double().numpy(), S_ref)
            assert e <= tol, f"call {frame + 1}: max-abs-rel {e:.3e} > {tol} against the oracle"
        assert lay.device_status() == 0
    finally:
        lay.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = ctypes.CDLL(arl2.library_path())
    lib.arl2_state_update_noalloc.restype = ctypes.c_int
    x = torch.zeros(16, dtype=torch.float32, device="cuda")
    p = _p(x)
    tokens = arl2.NOALLOC_MAX_ELEMENTS // (12 * 128) + 1  # one token too many for B=1, H=12
    rc = lib.arl2_state_update_noalloc(1, 12, 128, tokens, arl2.ARL2_FP32, p, p, p, p, p, p, p, None)
    assert rc == -2  # ARL2_ERR_SHAPE, nothing enqueued
    # heads and batch are grid dimensions: beyond the caps they are shape errors too
    assert lib.arl2_state_update_noalloc(1, 70000, 1, 1, arl2.ARL2_FP32, p, p, p, p, p, p, p, None) == -2
    assert lib.arl2_state_update_noalloc(70000, 1, 1, 1, arl2.ARL2_FP32, p, p, p, p, p, p, p, None) == -2
    rc = lib.arl2_state_update_noalloc(1, 1, 16, 16, arl2.ARL2_FP32, p, p, p, p, p, p, None, None)
    assert rc == -1
