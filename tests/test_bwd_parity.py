"""Backward pass on the GPU against the fp64 oracle, element by element.

The GPU backward consumes the GPU forward's O and LSE (as a training step
does); the oracle differentiates the definition from Q, K, V and dO alone.
Small shapes compare every gradient; the full-size training workload compares
whole sampled heads.
"""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from tests.gpu_helpers import err_stats, grad_ok, guard_intact, guarded, to64, GRAD_MAX

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_attention_144_b200 as fa
    fa.fa_get_device_status(clear=True)
    yield fa
    assert fa.fa_get_device_status() == 0, "a kernel gave up a bounded wait"


def run_bwd(fa, q, k, v, dout, scale):
    o, lse = fa.forward(q, k, v, scale=scale)
    shape = tuple(q.shape)
    bufs = [guarded(shape, q.dtype) for _ in range(3)]
    dq, dk, dv = (b[0] for b in bufs)
    fa.backward(q, k, v, o, dout, lse, scale=scale, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    for _, flat in bufs:
        assert guard_intact(flat), "write past the end of a gradient"
    return dq, dk, dv


def check_grads(fa, B, N, H, d, dtype, seed, std=1.0):
    q, k, v, dout = attn_inputs.draw(B, N, H, d, dtype, seed, 4, std=std, device="cuda")
    scale = float(np.float32(1.0 / math.sqrt(d)))
    dq, dk, dv = run_bwd(fa, q, k, v, dout, scale)
    ref = oracle.attn_bwd(to64(q), to64(k), to64(v), to64(dout), scale)
    stats = {}
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        g = to64(got)
        assert np.all(np.isfinite(g)), name
        stats[name] = err_stats(g, r)
        assert grad_ok(stats[name], name), (name, stats[name])
    return stats


@pytest.mark.parametrize("N", [1, 2, 17, 64, 65, 127, 128, 129, 300, 640])
def test_ragged_lengths_bf16(fa, N):
    check_grads(fa, 2, N, 2, 64, "bf16", 500 + N)


@pytest.mark.parametrize("N", [1, 100, 257])
def test_fp16(fa, N):
    check_grads(fa, 1, N, 3, 64, "fp16", 600 + N)


@pytest.mark.parametrize("N", [1, 17, 63, 64, 65, 127, 128, 129, 300, 640])
def test_head_dim_128_bf16(fa, N):
    # d = 128 runs the transposed-dQ kernel (64-query inner tiles)
    check_grads(fa, 2, N, 2, 128, "bf16", 800 + N)


@pytest.mark.parametrize("N", [1, 100, 257])
def test_head_dim_128_fp16(fa, N):
    check_grads(fa, 1, N, 3, 128, "fp16", 900 + N)


@pytest.mark.parametrize("N", [1, 17, 64, 65, 127, 128, 129, 300, 640])
def test_head_dim_96_bf16(fa, N):
    # d = 96 runs the transposed-dQ kernel on the d = 128 tile layout with
    # the last 32 columns of every row zero filled
    check_grads(fa, 2, N, 2, 96, "bf16", 1100 + N)


@pytest.mark.parametrize("B,N,H", [(1, 100, 3), (1, 257, 3), (1, 2048, 2)])
def test_head_dim_96_fp16(fa, B, N, H):
    check_grads(fa, B, N, H, 96, "fp16", 1150 + N)


@pytest.mark.parametrize("N", [1, 17, 64, 65, 127, 128, 129, 300, 640])
def test_head_dim_256_bf16(fa, N):
    # d = 256: two blocks per key tile, each producing one 128-wide half of
    # dK, dV and dQ^T while S^T and dP^T contract all 256 columns
    check_grads(fa, 2, N, 2, 256, "bf16", 1300 + N)


@pytest.mark.parametrize("N", [1, 100, 257, 1500])
def test_head_dim_256_fp16(fa, N):
    check_grads(fa, 1, N, 2, 256, "fp16", 1350 + N, std=0.5)


def test_detector_neck_backward_full_size(fa):
    # the detector neck workload (one head, d = 256, N = 6400, fp16, x0.5)
    # at full size: with dO zero outside a set R of query rows, every
    # gradient is exactly R's contribution (dS vanishes elsewhere), which the
    # row-restricted oracle returns for all keys
    w = attn_inputs.WORKLOADS["c3"]
    q, k, v, dout = attn_inputs.draw_workload(w, count=4, device="cuda")
    blocks = [(0, 64), (3200, 3264), (w.N - 40, w.N)]
    keep = torch.zeros(w.N, dtype=torch.bool, device="cuda")
    for a, b in blocks:
        keep[a:b] = True
    dout_r = torch.where(keep.view(1, w.N, 1, 1), dout, torch.zeros_like(dout))
    dq, dk, dv = run_bwd(fa, q, k, v, dout_r, w.scale)
    q64, k64, v64, d64 = (to64(t) for t in (q, k, v, dout_r))
    ref = None
    for a, b in blocks:
        part = oracle.attn_bwd_rows(q64, k64, v64, d64, w.scale, a, b)
        ref = part if ref is None else tuple(x + y for x, y in zip(ref, part))
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        s = err_stats(to64(got), r)
        assert grad_ok(s, name), (name, s)
    assert bool((dq[:, ~keep] == 0).all())


@pytest.mark.parametrize("d", [64, 128])
def test_batch_beyond_grid_dimension_limit(fa, d):
    # 66,000 short sequences: more (batch, head) pairs than a grid's y or z
    # dimension holds (65,535); the backward grid is 1-D, so every pair runs
    B, N, H = 66000, 20, 1
    q, k, v, dout = attn_inputs.draw(B, N, H, d, "bf16", 1400 + d, 4, device="cuda")
    scale = float(np.float32(1.0 / math.sqrt(d)))
    dq, dk, dv = run_bwd(fa, q, k, v, dout, scale)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    for b in (0, 1, 65534, 65535, 65536, B - 1):
        sl = slice(b, b + 1)
        ref = oracle.attn_bwd(to64(q[sl]), to64(k[sl]), to64(v[sl]), to64(dout[sl]), scale)
        for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            s = err_stats(to64(got[sl]), r)
            assert grad_ok(s, name), (b, name, s)


def test_head_dim_128_many_tiles(fa):
    # 16 key tiles per head, 32 query tiles each: both dQ^T buffers and every
    # Q/dO stage are reused many times over
    check_grads(fa, 1, 2048, 4, 128, "bf16", 950)


def test_several_heads_and_batches(fa):
    check_grads(fa, 3, 200, 5, 64, "bf16", 701)


def test_long_sequence_d128_backward_sampled_head(fa):
    # the long-sequence shape (N = 8192, d = 128) through the transposed-dQ
    # kernel: one whole head against the oracle, the rest checked for finiteness
    w = attn_inputs.WORKLOADS["c4train"]
    q, k, v, dout = attn_inputs.draw_workload(w, device="cuda")
    dq, dk, dv = run_bwd(fa, q, k, v, dout, w.scale)
    for (b, h) in [(0, 3)]:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1), slice(None))
        ref = oracle.attn_bwd(to64(q[sl]), to64(k[sl]), to64(v[sl]), to64(dout[sl]), w.scale)
        for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            s = err_stats(to64(got[sl]), r)
            assert grad_ok(s, name), (b, h, name, s)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()


def test_training_workload_sampled_heads(fa):
    w = attn_inputs.WORKLOADS["c5"]
    q, k, v, dout = attn_inputs.draw_workload(w, device="cuda")
    dq, dk, dv = run_bwd(fa, q, k, v, dout, w.scale)
    for (b, h) in [(0, 0), (w.B - 1, w.H - 1), (2, 5)]:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1), slice(None))
        ref = oracle.attn_bwd(to64(q[sl]), to64(k[sl]), to64(v[sl]), to64(dout[sl]), w.scale)
        for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
            s = err_stats(to64(got[sl]), r)
            assert grad_ok(s, name), (b, h, name, s)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()


@pytest.mark.parametrize("d,dtype", [(64, "bf16"), (96, "fp16"), (128, "bf16")])
def test_split_query_ranges(fa, d, dtype):
    # few key tiles: each key tile's query range is split over several
    # blocks (2 at d = 64, 4 at d = 96, 128), whose fp32 dK, dV partials a
    # separate kernel sums
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert fa.fa_bwd_plan(1, 2, 2048, d, sms)["n_split"] >= 2
    check_grads(fa, 1, 2048, 2, d, dtype, 1200 + d)
    # and the split partials are summed in a fixed order: bitwise repeatable
    q, k, v, dout = attn_inputs.draw(1, 2048, 2, d, dtype, 1210 + d, 4, device="cuda")
    a = run_bwd(fa, q, k, v, dout, 0.125)
    b = run_bwd(fa, q, k, v, dout, 0.125)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


@pytest.mark.parametrize("d", [64, 96, 128, 256])
def test_deterministic_dk_dv(fa, d):
    # dK and dV are owned by one block each (no atomics): bitwise repeatable.
    q, k, v, dout = attn_inputs.draw(1, 700, 2, d, "bf16", 702, 4, device="cuda")
    a = run_bwd(fa, q, k, v, dout, 0.125)
    b = run_bwd(fa, q, k, v, dout, 0.125)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert (a[0].float() - b[0].float()).abs().max().item() <= 1e-2
