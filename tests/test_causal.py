"""Causal attention on the GPU against the fp64 oracle (FA_FLAG_CAUSAL).

The causal mask (LLM explainer page, section 7.1) hides every future position
from a query: row i sees keys j <= i.  Forward and backward are compared with
the oracle's causal definition element by element on small and ragged shapes
(every head size, both 16-bit types, both forward kernels and both backward
kernels, tails around the 128-row tiles), on sampled rows and whole heads at
full size, and against the unmasked GPU result on the last row, which sees
every key.
"""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from tests.gpu_helpers import (err_stats, grad_ok, guard_intact, guarded, o_ok, sample_rows, to64,
                               GRAD_MAX, LSE_MAX, O_MAX, O_MEAN)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_attention_144_b200 as fa
    fa.fa_get_device_status(clear=True)
    yield fa
    assert fa.fa_get_device_status() == 0, "a kernel gave up a bounded wait"


def fwd(fa, q, k, v, scale):
    B, N, H, d = q.shape
    o, o_flat = guarded((B, N, H, d), q.dtype)
    lse, l_flat = guarded((B, H, N), torch.float32)
    fa.forward(q, k, v, scale=scale, o=o, lse=lse, causal=True)
    torch.cuda.synchronize()
    assert guard_intact(o_flat) and guard_intact(l_flat), "write past the end of an output"
    return o, lse


def check_fwd(fa, B, N, H, d, dtype, seed, scale=None):
    q, k, v = attn_inputs.draw(B, N, H, d, dtype, seed, 3, device="cuda")
    scale = float(np.float32(1.0 / math.sqrt(d))) if scale is None else scale
    o, lse = fwd(fa, q, k, v, scale)
    o_ref, lse_ref = oracle.attn_fwd(to64(q), to64(k), to64(v), scale, causal=True)
    eo, el = err_stats(to64(o), o_ref), err_stats(lse.cpu().double().numpy(), lse_ref)
    assert o_ok(eo), eo
    assert el["max"] <= LSE_MAX, el
    return q, k, v, o, lse


@pytest.mark.parametrize("N", [1, 2, 63, 127, 128, 129, 255, 256, 257, 400, 1000])
def test_causal_forward_ragged_d64(fa, N):
    check_fwd(fa, 2, N, 2, 64, "bf16", 1100 + N)


@pytest.mark.parametrize("d", [64, 96, 128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("N", [100, 300])
def test_causal_forward_head_sizes_and_types(fa, d, dtype, N):
    check_fwd(fa, 1, N, 2, d, dtype, 1200 + N + d)


@pytest.mark.parametrize("B,N,H,d", [(1, 2048, 8, 64), (1, 2000, 4, 128), (2, 1500, 1, 256)])
def test_causal_forward_many_tiles(fa, B, N, H, d):
    # several waves of units of different lengths on the alternating schedule
    check_fwd(fa, B, N, H, d, "bf16", 1300 + N)


def test_causal_forward_long_sequence_sampled_rows(fa):
    w = attn_inputs.WORKLOADS["c4"]
    q, k, v = attn_inputs.draw_workload(w, count=3, device="cuda")
    o, lse = fwd(fa, q, k, v, w.scale)
    rows = sample_rows(w.B, w.H, w.N, 96)
    o_ref, lse_ref = oracle.attn_fwd_rows(to64(q), to64(k), to64(v), w.scale, rows, causal=True)
    idx = np.array(rows)
    eo = err_stats(to64(o)[idx[:, 0], idx[:, 2], idx[:, 1]], o_ref)
    el = err_stats(lse.cpu().double().numpy()[idx[:, 0], idx[:, 1], idx[:, 2]], lse_ref)
    assert o_ok(eo), eo
    assert el["max"] <= LSE_MAX, el
    # the last row sees every key: it equals the unmasked forward's last row
    o_full, lse_full = fa.forward(q, k, v, scale=w.scale)
    torch.cuda.synchronize()
    assert (o[:, -1].float() - o_full[:, -1].float()).abs().max().item() <= 2e-2
    assert (lse[:, :, -1] - lse_full[:, :, -1]).abs().max().item() <= 1e-3
    # the first row sees only key 0: O = V_0 exactly (one probability of 1)
    assert torch.equal(o[:, 0], v[:, 0])


def bwd(fa, q, k, v, dout, scale):
    o, lse = fa.forward(q, k, v, scale=scale, causal=True)
    bufs = [guarded(tuple(q.shape), q.dtype) for _ in range(3)]
    dq, dk, dv = (x[0] for x in bufs)
    fa.backward(q, k, v, o, dout, lse, scale=scale, dq=dq, dk=dk, dv=dv, causal=True)
    torch.cuda.synchronize()
    for _, flat in bufs:
        assert guard_intact(flat), "write past the end of a gradient"
    return dq, dk, dv


def check_bwd(fa, B, N, H, d, dtype, seed):
    q, k, v, dout = attn_inputs.draw(B, N, H, d, dtype, seed, 4, device="cuda")
    scale = float(np.float32(1.0 / math.sqrt(d)))
    got = bwd(fa, q, k, v, dout, scale)
    ref = oracle.attn_bwd(to64(q), to64(k), to64(v), to64(dout), scale, causal=True)
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        s = err_stats(to64(g), r)
        assert grad_ok(s, name), (name, s)


@pytest.mark.parametrize("d", [64, 96, 128, 256])
@pytest.mark.parametrize("N", [1, 17, 64, 127, 128, 129, 300, 640])
def test_causal_backward_ragged(fa, d, N):
    check_bwd(fa, 2, N, 2, d, "bf16", 1400 + N + d)


@pytest.mark.parametrize("d", [64, 128])
def test_causal_backward_fp16_and_many_tiles(fa, d):
    check_bwd(fa, 1, 257, 3, d, "fp16", 1500 + d)
    check_bwd(fa, 1, 2048, 2, d, "bf16", 1510 + d)


def test_causal_backward_training_shape_sampled_heads(fa):
    w = attn_inputs.WORKLOADS["c5"]
    q, k, v, dout = attn_inputs.draw_workload(w, device="cuda")
    dq, dk, dv = bwd(fa, q, k, v, dout, w.scale)
    for (b, h) in [(0, 0), (w.B - 1, w.H - 1)]:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1), slice(None))
        ref = oracle.attn_bwd(to64(q[sl]), to64(k[sl]), to64(v[sl]), to64(dout[sl]), w.scale,
                              causal=True)
        for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            s = err_stats(to64(g[sl]), r)
            assert grad_ok(s, name), (b, h, name, s)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()


def test_causal_deterministic(fa):
    q, k, v, dout = attn_inputs.draw(1, 700, 2, 64, "bf16", 1600, 4, device="cuda")
    a = bwd(fa, q, k, v, dout, 0.125)
    b = bwd(fa, q, k, v, dout, 0.125)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    o1, l1 = fa.forward(q, k, v, scale=0.125, causal=True)
    o2, l2 = fa.forward(q, k, v, scale=0.125, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
