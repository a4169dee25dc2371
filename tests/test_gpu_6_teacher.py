"""GPU parity of the softmax teacher layer with a KV cache (technical summary
§1 "KV Cache Growth", §4 "Efficiency"): frame N's queries attend to the
clean keys/values of frames 0..N-1 and, bidirectionally, to their own; a
clean pass appends its keys and values.  Through the C ABI (TeacherLayer),
against the oracle's teacher_pass / teacher_rows, on the tensor-core kernel
(bf16, d = 128) and the SIMT kernel.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_harness import TOL, err, make_layer
from hybrid_softmax_gated_b200 import Arl2Error, TeacherLayer

pytestmark = pytest.mark.gpu

BASE = workloads.WORKLOADS["480p_bf16"]


def small(L, B=2, H=2, frames=4, passes=2):
    return dataclasses.replace(BASE, name=f"bf16_L{L}", batch=B, heads=H, tokens=L, frames=frames,
                               passes=passes)


def make_teacher(w, max_frames=None, **kw):
    return TeacherLayer(w.batch, w.heads, w.head_dim, w.tokens, max_frames or w.frames,
                        dtype=w.torch_dtype, **kw)


def run_teacher(w, *, frames=None, impl="auto", max_ctas=0, sample_rows=None, seed=0):
    """Frames of workload w through the teacher layer and the oracle.  With
    sample_rows, only that many random (stream, token) rows of each pass are
    compared (long caches); else every row.  Returns the worst error."""
    tol = TOL[w.dtype]
    n_frames = w.frames if frames is None else frames
    lay = make_teacher(w, max_frames=n_frames, impl=impl, max_ctas=max_ctas)
    rng = np.random.default_rng(seed)
    kc = vc = None
    worst = 0.0
    try:
        for f in range(n_frames):
            for p in range(w.passes):
                q, k, v = workloads.pass_inputs(w, 0, f, p)
                clean = workloads.is_clean(w, p)
                out = lay.forward(q.cuda(), k.cuda(), v.cuda(), clean_pass=clean).float().cpu().numpy()
                if sample_rows:
                    rb = rng.integers(0, w.batch, sample_rows)
                    rt = rng.integers(0, w.tokens, sample_rows)
                    ref = oracle.teacher_rows(q, k, v, kc, vc, rb, rt)
                    e = err(out[rb, rt], ref)
                else:
                    e = err(out, oracle.teacher_pass(q, k, v, kc, vc))
                worst = max(worst, e)
                assert e <= tol, f"frame {f} pass {p}: {e:.3e}"
                if clean:
                    kc, vc = oracle.teacher_append(kc, vc, k, v)
            assert lay.frames() == f + 1
        # the cache holds exactly the clean passes' keys and values
        k_dev, v_dev = lay.cache_get()
        assert np.array_equal(k_dev.double().cpu().numpy(), kc)
        assert np.array_equal(v_dev.double().cpu().numpy(), vc)
        assert lay.cache_bytes() == 2 * kc.size * (2 if w.dtype == "bf16" else 4)
        assert lay.device_status() == 0
    finally:
        lay.close()
    return worst


@pytest.mark.parametrize("L", [1, 17, 100, 128, 300])
def test_teacher_tc_matches_oracle(L):
    run_teacher(small(L))


def test_teacher_tc_split_schedule_with_cache():
    # more tiles than CTAs: split tiles whose key runs cross from cache to frame
    run_teacher(small(300, B=2, H=3, frames=5), max_ctas=5)
    run_teacher(small(200, B=1, H=2, frames=6), max_ctas=3)


def test_teacher_simt_matches_oracle():
    run_teacher(dataclasses.replace(workloads.WORKLOADS["tiny_fp32"], passes=2), impl="simt")
    run_teacher(dataclasses.replace(workloads.WORKLOADS["tiny_fp32"], tokens=37, head_dim=24, heads=3,
                                    batch=2, frames=3, passes=2), impl="simt")
    run_teacher(small(70, frames=3), impl="simt")


def test_teacher_480p_frames_sampled_rows():
    run_teacher(dataclasses.replace(BASE, passes=2), frames=4, sample_rows=96)


def test_teacher_long_cache_sampled_rows():
    # 24 cached 480p frames (37,440 keys) for two heads
    w = dataclasses.replace(BASE, heads=2, passes=1)
    run_teacher(w, frames=25, sample_rows=48)


def test_teacher_first_frame_equals_hybrid_layer_with_zero_state():
    # no cache yet and a zero state: the two layers compute the same softmax
    w = small(260, B=2, H=2)
    hyb, _ = make_layer(w)
    tea = make_teacher(w)
    try:
        q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, 0, 0))
        oh = hyb.forward(q, k, v)
        ot = tea.forward(q, k, v)
        assert torch.equal(oh, ot)
    finally:
        hyb.close()
        tea.close()


def test_teacher_noisy_passes_leave_the_cache_alone():
    w = small(90, frames=3)
    lay = make_teacher(w)
    try:
        q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, 0, 1))
        lay.forward(q, k, v, clean_pass=True)
        k0, v0 = lay.cache_get()
        q2, k2, v2 = (t.cuda() for t in workloads.pass_inputs(w, 0, 1, 0))
        a = lay.forward(q2, k2, v2).clone()
        b = lay.forward(q2, k2, v2)
        assert torch.equal(a, b) and lay.frames() == 1
        k1, v1 = lay.cache_get()
        assert torch.equal(k0, k1) and torch.equal(v0, v1)
    finally:
        lay.close()


def test_teacher_full_cache_and_reset():
    w = small(64, frames=2)
    lay = make_teacher(w, max_frames=2)
    try:
        q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, 0, 1))
        first = lay.forward(q, k, v, clean_pass=True).clone()
        lay.forward(q, k, v, clean_pass=True)
        with pytest.raises(Arl2Error):
            lay.forward(q, k, v, clean_pass=True)  # a third frame does not fit
        lay.forward(q, k, v)  # a read-only pass still runs
        assert lay.frames() == 2
        lay.reset()
        assert lay.frames() == 0 and lay.cache_bytes() == 0
        assert torch.equal(lay.forward(q, k, v, clean_pass=True), first)
        assert lay.device_status() == 0
    finally:
        lay.close()


def test_teacher_host_entry_matches_device_entry():
    w = small(150, B=1, frames=3)
    lay_h = make_teacher(w, host_staging=True)
    lay_d = make_teacher(w)
    try:
        for f in range(3):
            q, k, v = workloads.pass_inputs(w, 0, f, 1)
            out_h = torch.empty_like(q).pin_memory()
            lay_h.forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), True, out_h)
            torch.cuda.synchronize()
            od = lay_d.forward(q.cuda(), k.cuda(), v.cuda(), clean_pass=True)
            assert torch.equal(out_h, od.cpu())
    finally:
        lay_h.close()
        lay_d.close()


def test_teacher_kernel_launch_count():
    w = small(64, frames=2)
    lay = make_teacher(w)
    try:
        q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, 0, 0))
        lay.forward(q, k, v)
        assert lay.kernel_launches() == 1
        lay.forward(q, k, v, clean_pass=True)
        assert lay.kernel_launches() == 3  # attention, then the append
    finally:
        lay.close()


def test_teacher_cache_checkpoint_and_resume():
    # a layer resumed from another's cache continues exactly as the original
    w = small(130, frames=4)
    a = make_teacher(w)
    b = make_teacher(w)
    try:
        for f in range(2):
            q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, f, 1))
            a.forward(q, k, v, clean_pass=True)
        kc, vc = a.cache_get()
        b.cache_set(kc, vc)
        assert b.frames() == 2
        for f in range(2, 4):
            q, k, v = (t.cuda() for t in workloads.pass_inputs(w, 0, f, 1))
            assert torch.equal(a.forward(q, k, v, clean_pass=True), b.forward(q, k, v, clean_pass=True))
        with pytest.raises(Arl2Error):
            b.cache_set(torch.cat([kc] * 3, 1), torch.cat([vc] * 3, 1))  # 6 frames > capacity 4
        b.cache_set(kc[:, :0], vc[:, :0])
        assert b.frames() == 0
    finally:
        a.close()
        b.close()
