"""GPU parity of the SIMT kernels (the fp32 path) against the CPU oracle."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_harness import TOL, err, make_layer, run_and_check

pytestmark = pytest.mark.gpu


def test_tiny_fp32_stream_matches_oracle_everywhere():
    w = workloads.WORKLOADS["tiny_fp32"]
    eo, es = run_and_check(w)
    assert eo <= 1e-4 and es <= 1e-4


@pytest.mark.parametrize("L,d", [(1, 16), (33, 16), (77, 32), (130, 128)])
def test_fp32_ragged_multi_tile_shapes(L, d):
    w = dataclasses.replace(workloads.WORKLOADS["tiny_fp32"], name="fp32_shape", batch=2, heads=3,
                            head_dim=d, tokens=L, frames=3, passes=2)
    run_and_check(w)


def test_bf16_simt_small_stream():
    w = dataclasses.replace(workloads.WORKLOADS["480p_bf16"], name="bf16_small", batch=2, heads=2,
                            tokens=200, frames=3, passes=2)
    run_and_check(w, impl="simt")


@pytest.mark.parametrize("which", ["q", "k", "v"])
@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_phi_apply_matches_oracle(which, dtype):
    base = workloads.WORKLOADS["tiny_fp32"] if dtype == "fp32" else workloads.WORKLOADS["480p_bf16"]
    w = dataclasses.replace(base, name="phi", batch=2, heads=3, tokens=45)
    lay, ws = make_layer(w, impl="simt")
    try:
        x = workloads.pass_inputs(w, 0, 0, 0)[0]
        out = lay.phi_apply(which, x.cuda()).float().cpu().numpy()
        i = "qkv".index(which)
        ref = oracle.phi(x, ws[i], which == "k")
        assert err(out, ref) <= TOL[dtype]
    finally:
        lay.close()
