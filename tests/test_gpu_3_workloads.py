"""Full-size workloads on the GPU, in the launch configuration the benchmark
times, against the CPU oracle on sampled output rows and the full state.

- 480p: 21 frames x 4 passes; every row of the first and the last clean
  pass, 64 random rows of every other pass, the full state after each
  frame.
- 720p: 30 frames x 4 passes; every row of the first pass, 16 random rows
  elsewhere, the full state after each frame.
- long stream (240 frames): device memory and per-frame time stay flat;
  the oracle carries its own state through all 240 clean passes and the
  GPU state matches it every 20 frames and at the end; sampled rows of
  frames 0, 1, 120 and 239 match the oracle's outputs.
- 30-layer stack with 4 streams: layer 0 over all 60 frames, layers 0, 7,
  15, 22 and 29 over 4 frames, against the oracle (sampled rows, full
  state); every layer's streams independent of each other.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads
from gpu_harness import TOL, err, make_layer, run_and_check

pytestmark = pytest.mark.gpu

W = workloads.WORKLOADS


def test_480p_stream_sampled_parity():
    w = W["480p_bf16"]
    last = w.frames - 1
    eo, es = run_and_check(
        w, full_rows=lambda f, p: (f == 0 and p == 0) or (f == last and p == w.passes - 1),
        sample_rows=64)
    print(f"480p worst output err {eo:.3e}, worst state err {es:.3e}")


def test_720p_stream_sampled_parity():
    w = W["720p_bf16"]
    eo, es = run_and_check(w, full_rows=lambda f, p: f == 0 and p == 0, sample_rows=16)
    print(f"720p worst output err {eo:.3e}, worst state err {es:.3e}")


def test_long_stream_memory_and_time_flat_and_state_trajectory_parity():
    """240 frames x 4 passes.  The oracle carries its own state from S_0
    through all 240 clean passes (technical summary section 2.1 "State
    Update", section 2.2 "Clean-Pass Updates"); the GPU state is compared
    with it in full every 20 frames and after the last frame, and 64 random
    output rows of every pass of frames 0, 1, 120 and 239 with the oracle's
    outputs from the oracle's state.  Device memory and per-frame time must
    not grow with the frame index (section 4, "Efficiency": constant memory)."""
    w = W["long_stream_bf16"]
    lay, (wq, wk, wv) = make_layer(w)
    S_ref = oracle.zero_state(w.batch, w.heads, w.head_dim)
    check_rows = {0, 1, 120, w.frames - 1}
    check_state = set(range(19, w.frames, 20)) | {w.frames - 1}
    rng = np.random.default_rng(11)
    worst_o = worst_s = 0.0
    try:
        alloc0 = torch.cuda.memory_allocated()
        times, frees = [], []
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for f in range(w.frames):
            a, b = workloads.frame_gates(w, 0, f)
            ins = [workloads.pass_inputs(w, 0, f, p, device="cuda") for p in range(w.passes)]
            start.record()
            outs = []
            for p in range(w.passes):
                q, k, v = ins[p]
                outs.append(lay.forward(q, k, v, a.cuda(), b.cuda(), clean_pass=workloads.is_clean(w, p)))
            stop.record()
            stop.synchronize()
            times.append(start.elapsed_time(stop))
            frees.append(torch.cuda.mem_get_info()[0])
            if f in check_rows:
                for p in range(w.passes):
                    q, k, v = (x.cpu() for x in ins[p])
                    rt = rng.choice(w.tokens, size=64, replace=False)
                    rb = np.zeros_like(rt)
                    ref = oracle.rows(q, k, v, wq, S_ref, rb, rt)
                    e = err(outs[p].float().cpu().numpy()[rb, rt], ref)
                    worst_o = max(worst_o, e)
                    assert e <= TOL["bf16"], f"frame {f} pass {p}: output max-abs-rel {e:.3e}"
            # the oracle's own trajectory: its update from its own state
            k, v = ins[w.passes - 1][1].cpu(), ins[w.passes - 1][2].cpu()
            S_ref = oracle.state_update(k, v, wk, wv, a, b, S_ref)
            if f in check_state:
                e = err(lay.state_get().cpu().numpy(), S_ref)
                worst_s = max(worst_s, e)
                assert e <= TOL["bf16"], f"state after frame {f}: max-abs-rel {e:.3e}"
            del outs, ins
        assert lay.device_status() == 0
        # memory: nothing grows with the frame index
        assert max(frees) - min(frees) <= 64 << 20
        assert torch.cuda.memory_allocated() - alloc0 <= 64 << 20
        # time: the second half is not slower than the first
        t = np.array(times[5:])
        assert np.median(t[len(t) // 2:]) <= 1.25 * np.median(t[: len(t) // 2])
        print(f"long stream: worst output err {worst_o:.3e}, worst state err {worst_s:.3e}, "
              f"median frame {np.median(t):.3f} ms, free-mem spread {(max(frees) - min(frees)) / 2**20:.1f} MiB")
    finally:
        lay.close()


def test_stack30_layer0_whole_trajectory_against_oracle():
    """Layer 0 of the 30-layer stack, 4 streams, all 60 frames: 16 random
    rows of every pass and the full state after every clean pass."""
    w = W["stack30_bf16"]
    eo, es = run_and_check(w, layer=0, full_rows=lambda f, p: False, sample_rows=16, device_inputs=True)
    print(f"stack30 layer 0, 60 frames: worst output err {eo:.3e}, worst state err {es:.3e}")


@pytest.mark.parametrize("layer", [0, 7, 15, 22, 29])
def test_stack30_layers_against_oracle(layer):
    """Five layers spread over the stack (own weights, gates and states), 4
    streams, the first 4 frames: 32 random rows of every pass and the full
    state after every clean pass."""
    w = W["stack30_bf16"]
    run_and_check(w, layer=layer, frames=4, full_rows=lambda f, p: False, sample_rows=32, device_inputs=True)


def test_stack30_streams_independent():
    w = W["stack30_bf16"]
    # all 30 layers: 4-stream runs equal single-stream runs of the same inputs
    # (states bit-exact; outputs up to the summation order of tiles that the
    # persistent schedule splits differently for 4 and for 1 stream)
    import dataclasses
    w1 = dataclasses.replace(w, batch=1)
    for layer in range(w.layers):
        lay4, _ = make_layer(w, layer)
        lay1, _ = make_layer(w1, layer)
        try:
            for f in range(2):
                a, b = (t.cuda() for t in workloads.frame_gates(w, layer, f))
                q, k, v = (t.cuda() for t in workloads.pass_inputs(w, layer, f, w.passes - 1))
                o4 = lay4.forward(q, k, v, a, b, clean_pass=True)
                s = 3
                o1 = lay1.forward(q[s:s + 1].contiguous(), k[s:s + 1].contiguous(),
                                  v[s:s + 1].contiguous(), a[s:s + 1].contiguous(),
                                  b[s:s + 1].contiguous(), clean_pass=True)
                e = float((o1[0].float() - o4[s].float()).abs().max() / o4[s].float().abs().max())
                assert e <= 1e-2, (layer, f, e)
            assert torch.equal(lay1.state_get()[0], lay4.state_get()[s])
        finally:
            lay4.close()
            lay1.close()
