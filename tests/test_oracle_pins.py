"""Pins of the CPU oracle against what the ARL2 pages and mathematics fix.

None of these tests compares the oracle with a retyped copy of itself.  Each
pin is one of: a case worked out by hand (tests/golden), a special case that
reduces to a library routine (torch's scaled_dot_product_attention), a
closed form of the update (orthonormal keys), or an invariant the method
implies (frame-level sharing, clean-pass-only updates, independence of
streams and heads, scale invariance of the k' normalisation).

Method text: "Attend Locally, Remember Linearly", technical summary
section 2.1 (branches, phi maps, state update, read) and section 2.2
(frame-level access, clean-pass updates); the softmax teacher layer with a
KV cache from section 1 (KV Cache Growth) and section 4 (Efficiency); the
gate projections from section 2.1 (State Update).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_cases.json")


def rnd(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def eye_w(H, d):
    return np.broadcast_to(np.eye(d), (H, d, d)).copy()


def make(rng, B=2, L=7, H=3, d=8, wscale=0.3):
    q, k, v = (rnd(rng, B, L, H, d) for _ in range(3))
    wq, wk, wv = (np.eye(d)[None] + rnd(rng, H, d, d, scale=wscale) for _ in range(3))
    alpha = 1.0 / (1.0 + np.exp(-(2.0 + 0.5 * rnd(rng, B, H))))
    beta = 1.0 / (1.0 + np.exp(-rnd(rng, B, H, L))) / L
    S = rnd(rng, B, H, d, d, scale=0.1)
    return dict(q=q, k=k, v=v, wq=wq, wk=wk, wv=wv, alpha=alpha, beta=beta, S=S)


def run(x, clean, S=None, **over):
    a = dict(x)
    a.update(over)
    return oracle.frame_pass(a["q"], a["k"], a["v"], a["wq"], a["wk"], a["wv"], a["alpha"],
                             a["beta"], a["S"] if S is None else S, clean)


def as_blhd(m):
    """[L][d] (one stream, one head) -> [1][L][1][d]."""
    m = np.asarray(m, dtype=np.float64)
    return m[None, :, None, :]


def w_from(spec, d):
    if spec == "identity":
        return np.eye(d)[None]
    return np.asarray(spec, dtype=np.float64)[None]


def s_from(spec, d):
    if spec == "zero":
        return np.zeros((1, 1, d, d))
    return np.asarray(spec, dtype=np.float64)[None, None]


# --------------------------------------------------------------------------
# Hand-worked cases (tests/golden)
# --------------------------------------------------------------------------

def golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", golden_cases(), ids=lambda c: c["name"])
def test_hand_worked_case(case):
    if case.get("layer") == "gates":
        alpha, beta = oracle.gate_projection(np.asarray(case["x"], dtype=np.float64)[None],
                                             np.asarray(case["w"], dtype=np.float64),
                                             np.asarray(case["bias"], dtype=np.float64))
        np.testing.assert_allclose(alpha[0, 0], case["expected_alpha"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(beta[0, 0], case["expected_beta"], rtol=0, atol=1e-12)
        return
    d, L = case["d"], case["L"]
    zeros = np.zeros((L, d))
    q = as_blhd(case.get("q", zeros))
    k = as_blhd(case["k"])
    v = as_blhd(case["v"])
    if case.get("layer") == "teacher":
        out = oracle.teacher_pass(q, k, v, as_blhd(case["cache_k"]), as_blhd(case["cache_v"]),
                                  scale=case.get("scale"))
        np.testing.assert_allclose(out[0, :, 0, :], case["expected_out"], rtol=0, atol=1e-12)
        return
    wq = w_from(case.get("w_q", "identity"), d)
    wk = w_from(case.get("w_k", "identity"), d)
    wv = w_from(case.get("w_v", "identity"), d)
    S = s_from(case.get("S_prev", "zero"), d)
    a = case.get("alpha", 1.0)
    # a list: one gate per key feature (elementwise gating), else headwise
    alpha = np.asarray(a, dtype=np.float64)[None, None] if isinstance(a, list) else np.array([[a]])
    beta = np.asarray(case.get("beta", [0.0] * L), dtype=np.float64)[None, None]
    clean = "expected_S" in case
    run_pass = oracle.frame_pass_token_level if case.get("access") == "token" else oracle.frame_pass
    out, S_new = run_pass(q, k, v, wq, wk, wv, alpha, beta, S, clean)
    if "expected_out" in case:
        np.testing.assert_allclose(out[0, :, 0, :], case["expected_out"], rtol=0, atol=1e-12)
    if clean:
        np.testing.assert_allclose(S_new[0, 0], case["expected_S"], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Intra branch: textbook softmax attention
# --------------------------------------------------------------------------

def test_intra_equals_library_sdpa_when_state_is_zero():
    rng = np.random.default_rng(1)
    x = make(rng, B=2, L=13, H=3, d=8)
    S0 = np.zeros_like(x["S"])
    out, _ = run(x, clean=False, S=S0)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a.transpose(0, 2, 1, 3)))  # [B,H,L,d]
    ref = torch.nn.functional.scaled_dot_product_attention(t(x["q"]), t(x["k"]), t(x["v"]))
    np.testing.assert_allclose(out, ref.numpy().transpose(0, 2, 1, 3), rtol=0, atol=1e-12)


def test_single_token_frame_returns_its_value():
    rng = np.random.default_rng(2)
    x = make(rng, B=1, L=1, H=2, d=5)
    out, _ = run(x, clean=False, S=np.zeros_like(x["S"]))
    np.testing.assert_allclose(out, x["v"], rtol=0, atol=1e-14)


def test_identical_keys_average_the_values():
    rng = np.random.default_rng(3)
    x = make(rng, B=1, L=9, H=2, d=6)
    k = np.broadcast_to(x["k"][:, :1], x["k"].shape).copy()
    out, _ = run(x, clean=False, S=np.zeros_like(x["S"]), k=k)
    mean_v = np.broadcast_to(x["v"].mean(axis=1, keepdims=True), x["v"].shape)
    np.testing.assert_allclose(out, mean_v, rtol=0, atol=1e-13)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(4)
    B, L, H, d = 1, 6, 1, 4
    q = np.zeros((B, L, H, d)); q[..., 0] = 1.0
    k = np.zeros((B, L, H, d)); k[0, 3, 0, 0] = 200.0   # score 100 vs 0 after the 1/2 scale
    v = rnd(rng, B, L, H, d)
    out, _ = oracle.frame_pass(q, k, v, eye_w(H, d), eye_w(H, d), eye_w(H, d), None, None,
                               np.zeros((B, H, d, d)), False)
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(v[0, 3, 0], (L, d)), atol=1e-30)


# --------------------------------------------------------------------------
# Inter read
# --------------------------------------------------------------------------

def test_zero_state_adds_nothing_and_read_is_linear_in_state():
    rng = np.random.default_rng(5)
    x = make(rng)
    o0, _ = run(x, clean=False, S=np.zeros_like(x["S"]))
    o1, _ = run(x, clean=False, S=x["S"])
    o2, _ = run(x, clean=False, S=2.0 * x["S"])
    # O(S) - O(0) is linear in S: O(2S) - O(0) = 2 (O(S) - O(0))
    np.testing.assert_allclose(o2 - o0, 2.0 * (o1 - o0), rtol=0, atol=1e-12)
    assert np.max(np.abs(o1 - o0)) > 1e-3


def test_read_with_shift_map_and_identity_state():
    # W_q[a][a+1] = 1 shifts features right by one; with S = I and v = 0
    # the output is the shifted query: o[:, c] = q[:, c-1], o[:, 0] = 0.
    rng = np.random.default_rng(6)
    B, L, H, d = 1, 5, 2, 6
    q = rnd(rng, B, L, H, d)
    k = rnd(rng, B, L, H, d)
    v = np.zeros((B, L, H, d))
    shift = np.zeros((d, d))
    for a in range(d - 1):
        shift[a, a + 1] = 1.0
    wq = np.broadcast_to(shift, (H, d, d)).copy()
    S = np.broadcast_to(np.eye(d), (B, H, d, d)).copy()
    out, _ = oracle.frame_pass(q, k, v, wq, eye_w(H, d), eye_w(H, d), None, None, S, False)
    np.testing.assert_allclose(out[..., 1:], q[..., :-1], rtol=0, atol=1e-14)
    np.testing.assert_allclose(out[..., 0], 0.0, atol=1e-14)


# --------------------------------------------------------------------------
# State update: closed forms
# --------------------------------------------------------------------------

def test_alpha_one_beta_zero_leaves_state_unchanged():
    rng = np.random.default_rng(7)
    x = make(rng)
    _, S1 = run(x, clean=True, alpha=np.ones_like(x["alpha"]), beta=np.zeros_like(x["beta"]))
    assert np.array_equal(S1, x["S"])


def test_one_token_unit_key_alpha_beta_one_stores_value():
    # k' S_N = v' for ||k'|| = 1 and alpha = beta = 1, whatever S_{N-1}.
    rng = np.random.default_rng(8)
    B, L, H, d = 2, 1, 3, 8
    x = make(rng, B=B, L=L, H=H, d=d)
    # identity maps, so k' = k / ||k|| and v' = v independently of phi
    _, S1 = run(x, clean=True, wk=eye_w(H, d), wv=eye_w(H, d), alpha=np.ones((B, H)),
                beta=np.ones((B, H, L)))
    for b in range(B):
        for h in range(H):
            kp = x["k"][b, 0, h] / np.linalg.norm(x["k"][b, 0, h])
            np.testing.assert_allclose(kp @ S1[b, h], x["v"][b, 0, h], rtol=0, atol=1e-12)


@pytest.mark.parametrize("L", [1, 4, 8])
def test_orthonormal_keys_closed_form(L):
    # With orthonormal k' rows (L <= d): k'_i S_N = alpha k'_i S + beta_i (v'_i - k'_i S).
    # Rows of K are orthonormal rows scaled by positive factors, W_k = I, so
    # the L2 normalisation must undo the scaling.
    rng = np.random.default_rng(10 + L)
    B, H, d = 1, 2, 8
    x = make(rng, B=B, L=L, H=H, d=d)
    k = np.zeros((B, L, H, d))
    for h in range(H):
        qmat, _ = np.linalg.qr(rng.standard_normal((d, d)))
        k[0, :, h, :] = qmat[:L] * rng.uniform(0.5, 3.0, size=(L, 1))
    beta = rng.uniform(0.1, 0.9, size=(B, H, L))
    alpha = rng.uniform(0.3, 0.95, size=(B, H))
    _, S1 = run(x, clean=True, k=k, wk=eye_w(H, d), wv=eye_w(H, d), beta=beta, alpha=alpha)
    vp = x["v"]
    for h in range(H):
        kp = k[0, :, h, :] / np.linalg.norm(k[0, :, h, :], axis=1, keepdims=True)
        S0 = x["S"][0, h]
        lhs = kp @ S1[0, h]
        rhs = alpha[0, h] * (kp @ S0) + beta[0, h][:, None] * (vp[0, :, h] - kp @ S0)
        np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12)


def test_update_from_zero_state_is_rank_L_outer_product_sum():
    # S_{N-1} = 0: S_N = sum_i beta_i k'_i^T v'_i, so S_N lies in span(k'_i)
    # on the row side and span(v'_i) on the column side.
    rng = np.random.default_rng(11)
    B, L, H, d = 1, 3, 1, 8
    x = make(rng, B=B, L=L, H=H, d=d)
    _, S1 = run(x, clean=True, S=np.zeros((B, H, d, d)))
    kp = oracle.phi(x["k"], x["wk"], True)[0, :, 0]
    vp = oracle.phi(x["v"], x["wv"], False)[0, :, 0]
    assert np.linalg.matrix_rank(S1[0, 0], tol=1e-10) == L
    # project out span(k') from the rows: nothing is left
    Qk, _ = np.linalg.qr(kp.T)
    np.testing.assert_allclose(S1[0, 0] - Qk @ (Qk.T @ S1[0, 0]), 0.0, atol=1e-12)
    Qv, _ = np.linalg.qr(vp.T)
    np.testing.assert_allclose(S1[0, 0] - (S1[0, 0] @ Qv) @ Qv.T, 0.0, atol=1e-12)


def test_key_normalisation_is_scale_invariant():
    rng = np.random.default_rng(12)
    x = make(rng)
    _, S1 = run(x, clean=True)
    c = rng.uniform(0.25, 4.0, size=x["k"].shape[:3] + (1,))
    _, S2 = run(x, clean=True, k=x["k"] * c)
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-13)
    _, S3 = run(x, clean=True, wk=3.0 * x["wk"])
    np.testing.assert_allclose(S3, S1, rtol=0, atol=1e-13)


def test_phi_k_rows_have_unit_norm_and_phi_v_is_unnormalised():
    rng = np.random.default_rng(13)
    x = make(rng)
    kp = oracle.phi(x["k"], x["wk"], True)
    np.testing.assert_allclose(np.linalg.norm(kp, axis=-1), 1.0, atol=1e-13)
    vp = oracle.phi(x["v"], x["wv"], False)
    np.testing.assert_allclose(oracle.phi(2.0 * x["v"], x["wv"], False), 2.0 * vp, atol=1e-13)


# --------------------------------------------------------------------------
# Clean-pass updates and frame-level access (section 2.2)
# --------------------------------------------------------------------------

def test_non_clean_pass_keeps_state_bit_identical():
    rng = np.random.default_rng(14)
    x = make(rng)
    _, S1 = run(x, clean=False)
    assert np.array_equal(S1, x["S"])


def test_clean_pass_output_reads_pre_update_state():
    rng = np.random.default_rng(15)
    x = make(rng)
    o_read, _ = run(x, clean=False)
    o_clean, S1 = run(x, clean=True)
    assert np.array_equal(o_read, o_clean)
    assert not np.array_equal(S1, x["S"])


def test_token_permutation_permutes_output_and_keeps_state():
    rng = np.random.default_rng(16)
    x = make(rng, L=11)
    perm = rng.permutation(11)
    o1, S1 = run(x, clean=True)
    o2, S2 = run(x, clean=True, q=x["q"][:, perm], k=x["k"][:, perm], v=x["v"][:, perm],
                 beta=x["beta"][:, :, perm])
    np.testing.assert_allclose(o2, o1[:, perm], rtol=0, atol=1e-13)
    np.testing.assert_allclose(S2, S1, rtol=0, atol=1e-14)


def test_streams_and_heads_are_independent():
    rng = np.random.default_rng(17)
    x = make(rng, B=3, H=2)
    o, S = run(x, clean=True)
    for b in range(3):
        for h in range(2):
            sl = dict(q=x["q"][b:b + 1, :, h:h + 1], k=x["k"][b:b + 1, :, h:h + 1],
                      v=x["v"][b:b + 1, :, h:h + 1], wq=x["wq"][h:h + 1], wk=x["wk"][h:h + 1],
                      wv=x["wv"][h:h + 1], alpha=x["alpha"][b:b + 1, h:h + 1],
                      beta=x["beta"][b:b + 1, h:h + 1], S=x["S"][b:b + 1, h:h + 1])
            ob, Sb = run(sl, clean=True)
            np.testing.assert_array_equal(ob[0, :, 0], o[b, :, h])
            np.testing.assert_array_equal(Sb[0, 0], S[b, h])


def test_rows_entry_matches_full_pass_rows():
    rng = np.random.default_rng(18)
    x = make(rng, B=2, L=9)
    o, _ = run(x, clean=False)
    rb, rt = [0, 1, 1, 0], [0, 8, 3, 5]
    r = oracle.rows(x["q"], x["k"], x["v"], x["wq"], x["S"], rb, rt)
    for i, (b, t) in enumerate(zip(rb, rt)):
        np.testing.assert_array_equal(r[i], o[b, t])


def test_state_stays_bounded_over_a_long_stream():
    # alpha < 1 and beta ~ 1/L keep the state bounded: a 200-frame stream of
    # the tiny workload's distributions must not grow without limit.
    rng = np.random.default_rng(19)
    B, L, H, d = 1, 16, 1, 16
    S = np.zeros((B, H, d, d))
    wq, wk, wv = (np.eye(d)[None] + rnd(rng, H, d, d, scale=0.02) for _ in range(3))
    norms = []
    for f in range(200):
        k, v = rnd(rng, B, L, H, d), rnd(rng, B, L, H, d)
        alpha = 1 / (1 + np.exp(-(2 + 0.5 * rnd(rng, B, H))))
        beta = 1 / (1 + np.exp(-rnd(rng, B, H, L))) / L
        S = oracle.state_update(k, v, wk, wv, alpha, beta, S)
        norms.append(np.linalg.norm(S))
    assert max(norms[100:]) < 3.0 * max(norms[:100]) + 1e-9
    assert all(math.isfinite(n) for n in norms)


def test_oracle_rejects_bad_arguments():
    with pytest.raises(RuntimeError):
        oracle.rows(np.zeros((1, 2, 1, 4)), np.zeros((1, 2, 1, 4)), np.zeros((1, 2, 1, 4)),
                    np.zeros((1, 4, 4)), np.zeros((1, 1, 4, 4)), [0], [2])


# --------------------------------------------------------------------------
# Elementwise gating (atlas summary, "Surprising findings": one forget gate
# per key feature instead of one per head; S_N = diag(alpha) S_{N-1} + ...)
# --------------------------------------------------------------------------

def _update_inputs(seed, B=2, H=2, d=6, L=7):
    rng = np.random.default_rng(seed)
    k = rng.normal(size=(B, L, H, d))
    v = rng.normal(size=(B, L, H, d))
    wk = rng.normal(size=(H, d, d))
    wv = rng.normal(size=(H, d, d))
    beta = rng.random((B, H, L))
    S = rng.normal(size=(B, H, d, d))
    return rng, k, v, wk, wv, beta, S


def test_uniform_elementwise_gate_equals_headwise_gate():
    rng, k, v, wk, wv, beta, S = _update_inputs(41)
    a = rng.random((2, 2))
    s_head = oracle.state_update(k, v, wk, wv, a, beta, S)
    s_elem = oracle.state_update(k, v, wk, wv, np.repeat(a[:, :, None], 6, axis=2), beta, S)
    assert np.array_equal(s_head, s_elem)


def test_elementwise_gate_zero_clears_and_one_keeps_a_key_row():
    _, k, v, wk, wv, beta, S = _update_inputs(42)
    a = np.tile(np.array([0.0, 1.0, 0.0, 1.0, 1.0, 0.0]), (2, 2, 1))
    S_new = oracle.state_update(k, v, wk, wv, a, np.zeros_like(beta), S)
    for c in range(6):
        if a[0, 0, c] == 0.0:
            assert not S_new[:, :, c, :].any()
        else:
            assert np.array_equal(S_new[:, :, c, :], S[:, :, c, :])


def test_elementwise_gate_enters_as_a_row_scaling_of_the_previous_state():
    rng, k, v, wk, wv, beta, S = _update_inputs(43)
    a = rng.random((2, 2, 6))
    with_gate = oracle.state_update(k, v, wk, wv, a, beta, S)
    no_gate = oracle.state_update(k, v, wk, wv, np.zeros_like(a), beta, S)
    np.testing.assert_allclose(with_gate - no_gate, a[:, :, :, None] * S, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Token-level (sequential) access: the ablation of technical summary §2.2
# "Frame-Level Access" (atlas summary, "Surprising findings")
# --------------------------------------------------------------------------

def _pass_inputs(seed, B=2, H=2, d=6, L=9):
    rng = np.random.default_rng(seed)
    x = {n: rng.normal(size=(B, L, H, d)) for n in ("q", "k", "v")}
    x.update({n: np.eye(d) + 0.3 * rng.normal(size=(H, d, d)) for n in ("wq", "wk", "wv")})
    x["alpha"] = rng.random((B, H))
    x["beta"] = rng.random((B, H, L))
    x["S"] = rng.normal(size=(B, H, d, d))
    return rng, x


def _tl(x, clean=True, **kw):
    y = dict(x, **kw)
    return oracle.frame_pass_token_level(y["q"], y["k"], y["v"], y["wq"], y["wk"], y["wv"],
                                         y["alpha"], y["beta"], y["S"], clean)


def _fl(x, clean=True, **kw):
    y = dict(x, **kw)
    return oracle.frame_pass(y["q"], y["k"], y["v"], y["wq"], y["wk"], y["wv"], y["alpha"], y["beta"],
                             y["S"], clean)


def test_token_level_with_one_token_is_the_frame_level_rule():
    _, x = _pass_inputs(51, L=1)
    o_t, s_t = _tl(x)
    o_f, s_f = _fl(x)
    assert np.array_equal(o_t, o_f) and np.array_equal(s_t, s_f)


def test_token_level_without_writes_reads_the_frame_state():
    # beta = 0 and alpha = 1: no token changes the state, so every token
    # reads S_{N-1} exactly as under frame-level access
    _, x = _pass_inputs(52)
    kw = dict(beta=np.zeros_like(x["beta"]), alpha=np.ones_like(x["alpha"]))
    o_t, s_t = _tl(x, **kw)
    o_f, s_f = _fl(x, **kw)
    np.testing.assert_allclose(o_t, o_f, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s_t, x["S"], rtol=0, atol=0)


def test_token_level_orthonormal_keys_end_in_the_frame_level_state():
    # with orthonormal k' (L <= d) and alpha = 1 each token's residual is the
    # same against S^(i) as against S_{N-1}: the final states agree, and
    # token i's read differs by q'_i sum_{j<i} beta_j k'_j^T u_j
    rng, x = _pass_inputs(53, B=1, H=1, d=8, L=5)
    Qm, _ = np.linalg.qr(rng.normal(size=(8, 8)))
    k = Qm[:5][None, :, None, :]
    kw = dict(k=k, wk=np.eye(8)[None], alpha=np.ones((1, 1)))
    o_t, s_t = _tl(x, **kw)
    o_f, s_f = _fl(x, **kw)
    np.testing.assert_allclose(s_t, s_f, rtol=0, atol=1e-12)
    qp = x["q"][0, :, 0, :] @ x["wq"][0]
    vp = x["v"][0, :, 0, :] @ x["wv"][0]
    u = vp - k[0, :, 0, :] @ x["S"][0, 0]
    b = x["beta"][0, 0]
    for i in range(5):
        extra = sum(b[j] * (qp[i] @ k[0, j, 0]) * u[j] for j in range(i)) if i else 0.0
        np.testing.assert_allclose(o_t[0, i, 0] - o_f[0, i, 0], extra, rtol=0, atol=1e-12)


def test_token_level_reads_ignore_later_tokens():
    # the inter-frame part of token i (token-level minus frame-level output,
    # whose intra parts agree) depends on no token after i
    _, x = _pass_inputs(54)
    base = _tl(x)[0] - _fl(x)[0]
    v2 = x["v"].copy()
    v2[:, -1] += 5.0
    pert = _tl(x, v=v2)[0] - _fl(x, v=v2)[0]
    np.testing.assert_allclose(pert[:, :-1], base[:, :-1], rtol=0, atol=1e-12)
    assert np.abs(pert[:, -1] - base[:, -1]).max() < 1e-12  # its own read precedes its write


def test_token_level_noisy_pass_keeps_the_state():
    _, x = _pass_inputs(55)
    o_noisy, s_noisy = _tl(x, clean=False)
    o_clean, _ = _tl(x, clean=True)
    assert np.array_equal(s_noisy, x["S"])
    assert np.array_equal(o_noisy, o_clean)


def test_token_level_gate_acts_once_per_frame():
    # beta = 0: the only change is the gate with token 0's update, so tokens
    # after the first read alpha S_{N-1} and the frame ends in alpha S_{N-1}
    # (not alpha^L S_{N-1})
    _, x = _pass_inputs(56)
    kw = dict(beta=np.zeros_like(x["beta"]))
    o_t, s_t = _tl(x, **kw)
    np.testing.assert_allclose(s_t, x["alpha"][:, :, None, None] * x["S"], rtol=0, atol=1e-12)
    o_f, _ = _fl(x, **kw)
    o_g, _ = _fl(x, S=x["alpha"][:, :, None, None] * x["S"], **kw)
    np.testing.assert_allclose(o_t[:, 0], o_f[:, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(o_t[:, 1:], o_g[:, 1:], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# Softmax teacher layer with a KV cache (technical summary section 1 "KV
# Cache Growth", section 4 "Efficiency"): frame N attends to the clean keys
# and values of frames 0..N-1 and, bidirectionally, to its own
# --------------------------------------------------------------------------

def _teacher_inputs(seed, B=2, H=3, d=8, L=5, frames=3):
    rng = np.random.default_rng(seed)
    q, k, v = (rnd(rng, B, L, H, d) for _ in range(3))
    kc, vc = (rnd(rng, B, frames * L, H, d) for _ in range(2))
    return q, k, v, kc, vc


def _sdpa(q, k, v, scale=None):
    """torch's scaled_dot_product_attention in float64, [B, L, H, d] layout."""
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).permute(0, 2, 1, 3)
    o = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


@pytest.mark.parametrize("frames", [0, 1, 3])
def test_teacher_equals_library_sdpa_over_cache_then_frame(frames):
    q, k, v, kc, vc = _teacher_inputs(21 + frames, frames=frames)
    out = oracle.teacher_pass(q, k, v, kc if frames else None, vc if frames else None)
    ref = _sdpa(q, np.concatenate([kc, k], axis=1), np.concatenate([vc, v], axis=1))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_teacher_scale_is_used():
    q, k, v, kc, vc = _teacher_inputs(30, frames=2)
    out = oracle.teacher_pass(q, k, v, kc, vc, scale=0.9)
    ref = _sdpa(q, np.concatenate([kc, k], axis=1), np.concatenate([vc, v], axis=1), scale=0.9)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_teacher_with_empty_cache_is_the_hybrid_intra_branch():
    # the first frame has no cache: the teacher is then the hybrid layer's
    # intra-frame softmax (with a zero state the inter read adds nothing)
    q, k, v, _, _ = _teacher_inputs(31)
    B, L, H, d = q.shape
    eye = eye_w(H, d)
    hybrid, _ = oracle.frame_pass(q, k, v, eye, eye, eye, None, None, oracle.zero_state(B, H, d), False)
    np.testing.assert_allclose(oracle.teacher_pass(q, k, v), hybrid, rtol=0, atol=1e-13)


def test_teacher_frame_duplicated_in_cache_changes_nothing():
    # each key appearing twice doubles numerator and denominator alike
    q, k, v, _, _ = _teacher_inputs(32)
    alone = oracle.teacher_pass(q, k, v)
    np.testing.assert_allclose(oracle.teacher_pass(q, k, v, k, v), alone, rtol=0, atol=1e-12)
    kk, vv = np.concatenate([k, k], axis=1), np.concatenate([v, v], axis=1)
    np.testing.assert_allclose(oracle.teacher_pass(q, k, v, kk, vv), alone, rtol=0, atol=1e-12)


def test_teacher_cache_token_order_is_irrelevant():
    q, k, v, kc, vc = _teacher_inputs(33, frames=4)
    perm = np.random.default_rng(3).permutation(kc.shape[1])
    a = oracle.teacher_pass(q, k, v, kc, vc)
    b = oracle.teacher_pass(q, k, v, kc[:, perm], vc[:, perm])
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_teacher_dominant_cached_key_selects_its_value():
    # one cached key aligned with every query at a large scale takes all the weight
    q, k, v, kc, vc = _teacher_inputs(34, B=1, H=1, d=4, L=3, frames=2)
    q = np.abs(q) + 0.5
    kc[0, 4, 0] = 60.0 * np.ones(4)
    out = oracle.teacher_pass(q, k, v, kc, vc)
    for i in range(3):
        np.testing.assert_allclose(out[0, i, 0], vc[0, 4, 0], rtol=0, atol=1e-9)


def test_teacher_streams_and_heads_read_their_own_cache():
    q, k, v, kc, vc = _teacher_inputs(35, frames=2)
    base = oracle.teacher_pass(q, k, v, kc, vc)
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[1] += 1.0
    vc2[1] -= 2.0
    kc2[:, :, 2] *= 3.0
    out = oracle.teacher_pass(q, k, v, kc2, vc2)
    np.testing.assert_array_equal(out[0, :, :2], base[0, :, :2])  # stream 0, heads 0-1 untouched
    assert np.abs(out[1] - base[1]).max() > 1e-3
    assert np.abs(out[0, :, 2] - base[0, :, 2]).max() > 1e-3


def test_teacher_rows_match_the_full_pass():
    q, k, v, kc, vc = _teacher_inputs(36, frames=2)
    full = oracle.teacher_pass(q, k, v, kc, vc)
    rb, rt = [1, 0, 1, 0], [4, 0, 2, 3]
    np.testing.assert_array_equal(oracle.teacher_rows(q, k, v, kc, vc, rb, rt), full[rb, rt])


def test_teacher_append_is_concatenation_in_frame_order():
    q, k, v, kc, vc = _teacher_inputs(37, frames=1)
    k2, v2 = oracle.teacher_append(kc, vc, k, v)
    np.testing.assert_array_equal(k2[:, :kc.shape[1]], kc)
    np.testing.assert_array_equal(v2[:, kc.shape[1]:], v)
    k0, v0 = oracle.teacher_append(None, None, k, v)
    np.testing.assert_array_equal(k0, k)


def test_teacher_rejects_bad_arguments():
    q, k, v, kc, vc = _teacher_inputs(38, frames=1)
    with pytest.raises(ValueError):
        oracle.teacher_pass(q, k, v, kc[:, :, :2], vc[:, :, :2])
    with pytest.raises(ValueError):
        oracle.teacher_pass(q, k, v, kc, vc[:, :3])
    with pytest.raises(RuntimeError):
        oracle.teacher_rows(q, k, v, kc, vc, [2], [0])


# --------------------------------------------------------------------------
# Gate projections (technical summary section 2.1 "State Update": alpha and
# beta are learned per-token projections; reading: linear logits per token,
# beta = sigmoid(g_i), alpha = sigmoid(mean_i a_i))
# --------------------------------------------------------------------------

def _gate_inputs(seed, B=2, L=9, D=12, H=3):
    rng = np.random.default_rng(seed)
    x = rnd(rng, B, L, D)
    w = rnd(rng, D, 2 * H, scale=1.0 / np.sqrt(D))
    bias = rnd(rng, 2 * H)
    return x, w, bias


def _logit(p):
    return np.log(p) - np.log1p(-p)


def test_gates_of_zero_hidden_states_are_the_bias_sigmoids():
    x, w, bias = _gate_inputs(40)
    a, b = oracle.gate_projection(np.zeros_like(x), w, bias)
    H = w.shape[1] // 2
    np.testing.assert_allclose(a, np.broadcast_to(1 / (1 + np.exp(-bias[:H])), a.shape), rtol=0, atol=1e-15)
    np.testing.assert_allclose(b, np.broadcast_to((1 / (1 + np.exp(-bias[H:])))[None, :, None], b.shape),
                               rtol=0, atol=1e-15)


def test_gate_logits_are_affine_in_the_hidden_state():
    # logit(beta(x + y)) = logit(beta(x)) + logit(beta(y)) - bias, and the
    # frame gate's logit (a mean of affine logits) obeys the same identity
    x, w, bias = _gate_inputs(41)
    y, _, _ = _gate_inputs(42)
    H = w.shape[1] // 2
    ax, bx = oracle.gate_projection(x, w, bias)
    ay, by = oracle.gate_projection(y, w, bias)
    axy, bxy = oracle.gate_projection(x + y, w, bias)
    np.testing.assert_allclose(_logit(bxy), _logit(bx) + _logit(by) - bias[H:][None, :, None], rtol=0, atol=1e-9)
    np.testing.assert_allclose(_logit(axy), _logit(ax) + _logit(ay) - bias[:H][None], rtol=0, atol=1e-9)


def test_frame_gate_of_repeated_tokens_is_the_token_gate():
    # L copies of one token: the mean logit is that token's logit
    x, w, bias = _gate_inputs(43, L=1)
    a1, _ = oracle.gate_projection(x, w, bias)
    aL, bL = oracle.gate_projection(np.repeat(x, 7, axis=1), w, bias)
    np.testing.assert_allclose(aL, a1, rtol=0, atol=1e-14)
    np.testing.assert_allclose(bL, np.repeat(bL[:, :, :1], 7, axis=2), rtol=0, atol=0)


def test_frame_gate_is_the_sigmoid_of_the_mean_logit_not_the_mean_sigmoid():
    # two single-token frames and their union: the union's logit is the mean
    x, w, bias = _gate_inputs(44, L=2)
    a0, b0 = oracle.gate_projection(x[:, :1], w, bias)
    a1, b1 = oracle.gate_projection(x[:, 1:], w, bias)
    a, b = oracle.gate_projection(x, w, bias)
    np.testing.assert_allclose(_logit(a), (_logit(a0) + _logit(a1)) / 2, rtol=0, atol=1e-9)
    np.testing.assert_allclose(b, np.concatenate([b0, b1], axis=2), rtol=0, atol=0)
    assert np.abs(a - (a0 + a1) / 2).max() > 1e-4


def test_gate_token_permutation():
    x, w, bias = _gate_inputs(45)
    perm = np.random.default_rng(4).permutation(x.shape[1])
    a, b = oracle.gate_projection(x, w, bias)
    ap, bp = oracle.gate_projection(x[:, perm], w, bias)
    np.testing.assert_allclose(ap, a, rtol=0, atol=1e-14)
    np.testing.assert_array_equal(bp, b[:, :, perm])


def test_gate_heads_read_their_own_columns():
    x, w, bias = _gate_inputs(46)
    H = w.shape[1] // 2
    a, b = oracle.gate_projection(x, w, bias)
    w2, bias2 = w.copy(), bias.copy()
    w2[:, 1] += 1.0          # head 1's alpha column
    bias2[H + 2] -= 3.0      # head 2's beta bias
    a2, b2 = oracle.gate_projection(x, w2, bias2)
    np.testing.assert_array_equal(a2[:, [0, 2]], a[:, [0, 2]])
    np.testing.assert_array_equal(b2[:, :2], b[:, :2])
    assert np.abs(a2[:, 1] - a[:, 1]).max() > 1e-3 and np.abs(b2[:, 2] - b[:, 2]).max() > 1e-3
    # and streams only their own hidden states
    x2 = x.copy()
    x2[1] += 1.0
    a3, b3 = oracle.gate_projection(x2, w, bias)
    np.testing.assert_array_equal(a3[0], a[0])
    np.testing.assert_array_equal(b3[0], b[0])


def test_gate_projection_rejects_bad_shapes():
    x, w, bias = _gate_inputs(47)
    with pytest.raises(ValueError):
        oracle.gate_projection(x, w[:-1], bias)
    with pytest.raises(ValueError):
        oracle.gate_projection(x, w, bias[:-1])
    with pytest.raises(ValueError):
        oracle.gate_projection(x, w[:, :-1], bias[:-1])
