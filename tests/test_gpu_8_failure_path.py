"""Failure detection without a GPU fault: a bounded device wait on a word
that nothing sets gives up after its limit, sets the handle's error word,
and the host reads ARL2_ERR_TIMEOUT; the context stays usable and later
passes still match the oracle."""
import dataclasses
import time

import pytest
import torch

import oracle
import workloads
from gpu_harness import TOL, err, make_layer
from hybrid_softmax_gated_b200 import ARL2_ERR_TIMEOUT

pytestmark = pytest.mark.gpu

BASE = workloads.WORKLOADS["480p_bf16"]


@pytest.mark.parametrize("w,impl", [
    (dataclasses.replace(BASE, batch=1, heads=2, tokens=300, frames=2, passes=2), "auto"),
    (workloads.WORKLOADS["tiny_fp32"], "simt")], ids=["tensor_core", "simt"])
def test_bounded_wait_gives_up_and_the_context_stays_usable(w, impl):
    lay, (wq, wk, wv) = make_layer(w, impl=impl)
    S_ref = oracle.zero_state(w.batch, w.heads, w.head_dim)
    try:
        def frame(f):
            nonlocal S_ref
            alpha, beta = workloads.frame_gates(w, 0, f)
            for p in range(w.passes):
                q, k, v = workloads.pass_inputs(w, 0, f, p)
                clean = workloads.is_clean(w, p)
                out = lay.forward(q.cuda(), k.cuda(), v.cuda(), alpha.cuda(), beta.cuda(), clean_pass=clean)
                ref, S_next = oracle.frame_pass(q, k, v, wq, wk, wv, alpha, beta, S_ref, clean)
                assert err(out.float().cpu().numpy(), ref) <= TOL[w.dtype]
                if clean:
                    S_ref = S_next

        frame(0)
        assert lay.device_status() == 0
        t0 = time.time()
        lay.selftest_wait_timeout(20000)  # 20 ms on a word nothing sets
        assert lay.device_status() == ARL2_ERR_TIMEOUT
        assert time.time() - t0 < 5.0     # it gave up; nothing hung
        assert lay.device_status() == 0   # read and cleared
        frame(1)                          # the context and the state are intact
        assert lay.device_status() == 0
        assert err(lay.state_get().cpu().numpy(), S_ref) <= TOL[w.dtype]
    finally:
        lay.close()
