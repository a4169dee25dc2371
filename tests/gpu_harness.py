"""Shared GPU-test helpers: run a workload through the C ABI and check it
against the CPU oracle pass by pass.

Tolerances (max-abs-relative per tensor, max|x - ref| / max|ref|): 2e-2 for
bf16 workloads and 1e-4 for fp32 ones.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads
from hybrid_softmax_gated_b200 import Arl2Layer

TOL = {"bf16": 2e-2, "fp32": 1e-4}


def make_layer(w: workloads.Workload, layer: int = 0, impl: str = "auto", **kw):
    wq, wk, wv = workloads.phi_weights(w, layer)
    lay = Arl2Layer(w.batch, w.heads, w.head_dim, w.tokens, wq.cuda(), wk.cuda(), wv.cuda(),
                    dtype=w.torch_dtype, impl=impl, **kw)
    return lay, (wq, wk, wv)


def err(x, ref) -> float:
    return oracle.max_abs_rel(np.asarray(x, dtype=np.float64), ref)


def run_and_check(w: workloads.Workload, *, impl: str = "auto", layer: int = 0, frames=None,
                  full_rows=lambda f, p: True, sample_rows: int = 64, seed: int = 0,
                  device_inputs: bool = False, layer_kw=None, gating: str = "headwise"):
    """Run frames of workload w on the GPU and on the oracle.

    full_rows(frame, pass) selects passes whose every output row is
    compared; other passes compare `sample_rows` random (stream, token)
    rows.  The state is compared in full after every clean pass.  Returns
    the worst output and state errors.  gating="elementwise" draws one forget
    gate per key feature.
    """
    tol = TOL[w.dtype]
    lay, (wq, wk, wv) = make_layer(w, layer, impl, gating=gating, **(layer_kw or {}))
    gates = workloads.frame_gates_elementwise if gating == "elementwise" else workloads.frame_gates
    rng = np.random.default_rng(seed)
    S_ref = oracle.zero_state(w.batch, w.heads, w.head_dim)
    worst_o = worst_s = 0.0
    dev = "cuda" if device_inputs else "cpu"
    try:
        for f in range(w.frames if frames is None else frames):
            alpha, beta = gates(w, layer, f)
            a_d, b_d = alpha.cuda(), beta.cuda()
            for p in range(w.passes):
                q, k, v = workloads.pass_inputs(w, layer, f, p, device=dev)
                qd, kd, vd = (t.cuda() for t in (q, k, v))
                clean = workloads.is_clean(w, p)
                out = lay.forward(qd, kd, vd, a_d, b_d, clean_pass=clean)
                out_h = out.float().cpu().numpy()
                if full_rows(f, p):
                    rb = np.repeat(np.arange(w.batch), w.tokens)
                    rt = np.tile(np.arange(w.tokens), w.batch)
                else:
                    n = min(sample_rows, w.batch * w.tokens)
                    pick = rng.choice(w.batch * w.tokens, size=n, replace=False)
                    rb, rt = pick // w.tokens, pick % w.tokens
                ref = oracle.rows(q, k, v, wq, S_ref, rb, rt)
                e = err(out_h[rb, rt], ref)
                worst_o = max(worst_o, e)
                assert e <= tol, f"output frame {f} pass {p}: max-abs-rel {e:.3e} > {tol}"
                if clean:
                    S_ref = oracle.state_update(k, v, wk, wv, alpha, beta, S_ref)
                    S_gpu = lay.state_get().cpu().numpy()
                    e = err(S_gpu, S_ref)
                    worst_s = max(worst_s, e)
                    assert e <= tol, f"state after frame {f}: max-abs-rel {e:.3e} > {tol}"
        assert lay.device_status() == 0
    finally:
        lay.close()
    return worst_o, worst_s
