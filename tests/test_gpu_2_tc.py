"""GPU parity of the tensor-core (tcgen05) path, bf16 with head_dim 128.

Covers ragged token counts (one token, a partial tile, exact tiles, a
tile plus one, a last block of 64 and of 65 keys), several streams and heads, and the method's invariants on
the GPU: read-only passes leave the state bit-identical, streams are
independent, token permutation permutes the output, checkpoint/resume is
exact.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_harness import TOL, err, make_layer, run_and_check

pytestmark = pytest.mark.gpu

BASE = workloads.WORKLOADS["480p_bf16"]


def small(L, B=2, H=2, frames=3, passes=2):
    return dataclasses.replace(BASE, name=f"bf16_L{L}", batch=B, heads=H, tokens=L, frames=frames,
                               passes=passes)


@pytest.mark.parametrize("L", [1, 17, 128, 129, 192, 193, 300, 515])
def test_tc_stream_matches_oracle_everywhere(L):
    # 192 and 193: a last key block of exactly 64 keys (its softmax skips the
    # second half of P) and of 65 (it does not)
    run_and_check(small(L))


@pytest.mark.parametrize("L,max_ctas", [(129, 3), (129, 7), (515, 3), (515, 7), (515, 19), (700, 5)])
def test_split_tile_schedule_matches_oracle(L, max_ctas):
    # More tiles than CTAs: the persistent schedule cuts tiles into a head
    # and a tail piece on different CTAs and merges them.
    run_and_check(small(L, B=2, H=2, frames=2), layer_kw={"max_ctas": max_ctas})


def test_split_schedule_repeats_bit_exactly():
    w = small(515, B=2, H=2)
    lay, _ = make_layer(w, max_ctas=7)
    try:
        q, k, v, a, b = _inputs(w)
        o1 = lay.forward(q, k, v).clone()
        for _ in range(3):
            assert torch.equal(lay.forward(q, k, v), o1)
        assert lay.device_status() == 0
    finally:
        lay.close()


def _inputs(w, f=0, p=0):
    q, k, v = workloads.pass_inputs(w, 0, f, p)
    a, b = workloads.frame_gates(w, 0, f)
    return q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda()


def test_read_only_pass_keeps_state_bit_identical():
    w = small(260)
    lay, _ = make_layer(w)
    try:
        q, k, v, a, b = _inputs(w)
        lay.forward(q, k, v, a, b, clean_pass=True)
        s0 = lay.state_get().clone()
        q, k, v, a, b = _inputs(w, 1, 0)
        o1 = lay.forward(q, k, v)
        assert torch.equal(lay.state_get(), s0)
        # the clean pass's own output reads the pre-update state
        o2 = lay.forward(q, k, v, a, b, clean_pass=True)
        assert torch.equal(o1, o2)
        assert not torch.equal(lay.state_get(), s0)
    finally:
        lay.close()


def test_streams_are_independent_bit_exact():
    w3 = small(200, B=3, H=2)
    lay3, ws = make_layer(w3)
    w1 = dataclasses.replace(w3, batch=1)
    lays = [make_layer(w1)[0] for _ in range(3)]
    try:
        for f in range(2):
            q, k, v, a, b = _inputs(w3, f, 1)
            o3 = lay3.forward(q, k, v, a, b, clean_pass=True)
            for i, l1 in enumerate(lays):
                o1 = l1.forward(q[i:i + 1].contiguous(), k[i:i + 1].contiguous(),
                                v[i:i + 1].contiguous(), a[i:i + 1].contiguous(),
                                b[i:i + 1].contiguous(), clean_pass=True)
                assert torch.equal(o1[0], o3[i])
                assert torch.equal(l1.state_get()[0], lay3.state_get()[i])
    finally:
        lay3.close()
        for l1 in lays:
            l1.close()


def test_token_permutation_permutes_output():
    w = small(300, B=1, H=2)
    lay, _ = make_layer(w)
    try:
        q, k, v, a, b = _inputs(w)
        lay.forward(q, k, v, a, b, clean_pass=True)  # non-zero state
        s = lay.state_get().clone()
        q, k, v, a, b = _inputs(w, 1, 0)
        o = lay.forward(q, k, v).float()
        perm = torch.randperm(w.tokens, generator=torch.Generator().manual_seed(3)).cuda()
        op = lay.forward(q[:, perm].contiguous(), k[:, perm].contiguous(), v[:, perm].contiguous()).float()
        assert err(op.cpu().numpy(), o[:, perm].cpu().numpy()) <= 1e-2
        assert torch.equal(lay.state_get(), s)
    finally:
        lay.close()


def test_checkpoint_resume_is_exact():
    w = small(200, frames=4)
    lay_a, _ = make_layer(w)
    lay_b, _ = make_layer(w)
    try:
        outs_a = []
        for f in range(4):
            q, k, v, a, b = _inputs(w, f, 1)
            outs_a.append(lay_a.forward(q, k, v, a, b, clean_pass=True).clone())
            if f == 1:
                ckpt = lay_a.state_get().clone()
        lay_b.state_set(ckpt)
        for f in range(2, 4):
            q, k, v, a, b = _inputs(w, f, 1)
            ob = lay_b.forward(q, k, v, a, b, clean_pass=True)
            assert torch.equal(ob, outs_a[f])
        assert torch.equal(lay_b.state_get(), lay_a.state_get())
        lay_b.state_reset()
        assert int(torch.count_nonzero(lay_b.state_get())) == 0
    finally:
        lay_a.close()
        lay_b.close()


def test_tc_matches_simt_on_a_full_480p_frame():
    w = BASE
    lay_t, _ = make_layer(w, impl="auto")
    lay_s, _ = make_layer(w, impl="simt")
    try:
        for f in range(2):
            a, b = workloads.frame_gates(w, 0, f)
            a, b = a.cuda(), b.cuda()
            for p in range(w.passes):
                q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, f, p))
                clean = workloads.is_clean(w, p)
                ot = lay_t.forward(q, k, v, a, b, clean_pass=clean).float()
                os_ = lay_s.forward(q, k, v, a, b, clean_pass=clean).float()
                e = float((ot - os_).abs().max() / os_.abs().max())
                assert e <= TOL["bf16"], (f, p, e)
            st, ss = lay_t.state_get(), lay_s.state_get()
            assert float((st - ss).abs().max() / ss.abs().max()) <= TOL["bf16"]
        assert lay_t.device_status() == 0
    finally:
        lay_t.close()
        lay_s.close()


def test_host_buffer_entry_matches_device_entry():
    w = small(200, B=1)
    lay_h, _ = make_layer(w, host_staging=True)
    lay_d, _ = make_layer(w)
    try:
        for f in range(2):
            q, k, v = workloads.pass_inputs(w, 0, f, 1)
            a, b = workloads.frame_gates(w, 0, f)
            out_h = torch.empty_like(q).pin_memory()
            qh, kh, vh, ah, bh = (t.pin_memory() for t in (q, k, v, a, b))
            lay_h.forward_host(qh, kh, vh, ah, bh, True, out_h)
            torch.cuda.synchronize()
            od = lay_d.forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), clean_pass=True)
            assert torch.equal(out_h, od.cpu())
    finally:
        lay_h.close()
        lay_d.close()


@pytest.mark.parametrize("L", [200, 1560])
def test_pipelined_host_staging_matches_device_entry(L):
    """host_staging = 2: consecutive host calls alternate staging sets, the
    input copies overlap the previous call's pass and output copy, and no
    synchronisation between calls; every output and the state must equal the
    device entry's bit for bit."""
    w = small(L, B=1, frames=3, passes=3)
    lay_h, _ = make_layer(w, host_staging=2)
    lay_d, _ = make_layer(w)
    try:
        keep, outs, refs = [], [], []
        for f in range(w.frames):
            a, b = workloads.frame_gates(w, 0, f)
            ah, bh = a.pin_memory(), b.pin_memory()
            for p in range(w.passes):
                q, k, v = workloads.pass_inputs(w, 0, f, p)
                clean = workloads.is_clean(w, p)
                qh, kh, vh = (t.pin_memory() for t in (q, k, v))
                out_h = torch.empty_like(q).pin_memory()
                lay_h.forward_host(qh, kh, vh, ah, bh, clean, out_h)
                keep.append((qh, kh, vh, ah, bh))
                outs.append(out_h)
                refs.append(lay_d.forward(q.cuda(), k.cuda(), v.cuda(), a.cuda(), b.cuda(), clean_pass=clean))
        torch.cuda.synchronize()
        for i, (o, r) in enumerate(zip(outs, refs)):
            assert torch.equal(o, r.cpu()), i
        assert torch.equal(lay_h.state_get(), lay_d.state_get())
        # one output buffer for every call: it holds the last pass's output
        shared = torch.empty_like(outs[0]).pin_memory()
        lay_h.state_reset()
        lay_d.state_reset()
        for f in range(w.frames):
            a, b = workloads.frame_gates(w, 0, f)
            for p in range(w.passes):
                qh, kh, vh, ah, bh = keep[f * w.passes + p]
                lay_h.forward_host(qh, kh, vh, ah, bh, workloads.is_clean(w, p), shared)
        torch.cuda.synchronize()
        assert torch.equal(shared, outs[-1])
        assert lay_h.device_status() == 0
    finally:
        lay_h.close()
        lay_d.close()
