"""Forward pass on the GPU against the fp64 oracle, element by element.

Small shapes compare every output; the full-size workloads compare sampled
rows that the oracle computes one by one, in the same launch configuration
the bench times.  Edge cases: N = 1 and ragged tails around the 128-row tiles,
every head size, both 16-bit types, the split-K/V path, guard bands after
every output, closed forms, and bitwise determinism.
"""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from tests.gpu_helpers import (err_stats, guard_intact, guarded, o_ok, sample_rows, to64, LSE_MAX,
                               O_MAX, O_MEAN)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_attention_144_b200 as fa
    fa.fa_get_device_status(clear=True)
    yield fa
    assert fa.fa_get_device_status() == 0, "a kernel gave up a bounded wait"


def run(fa, q, k, v, scale):
    B, N, H, d = q.shape
    o, o_flat = guarded((B, N, H, d), q.dtype)
    lse, l_flat = guarded((B, H, N), torch.float32)
    fa.forward(q, k, v, scale=scale, o=o, lse=lse)
    torch.cuda.synchronize()
    assert guard_intact(o_flat) and guard_intact(l_flat), "write past the end of an output"
    return o, lse


def check_full(fa, B, N, H, d, dtype, seed, std=1.0, scale=None):
    q, k, v = attn_inputs.draw(B, N, H, d, dtype, seed, 3, std=std, device="cuda")
    scale = float(np.float32(1.0 / math.sqrt(d))) if scale is None else scale
    o, lse = run(fa, q, k, v, scale)
    o_ref, lse_ref = oracle.attn_fwd(to64(q), to64(k), to64(v), scale)
    eo, el = err_stats(to64(o), o_ref), err_stats(lse.cpu().double().numpy(), lse_ref)
    assert np.all(np.isfinite(to64(o))) and np.all(np.isfinite(lse.cpu().numpy()))
    assert o_ok(eo), eo
    assert el["max"] <= LSE_MAX, el
    return eo, el


@pytest.mark.parametrize("N", [1, 2, 17, 63, 64, 65, 127, 128, 129, 255, 256, 400, 1000])
def test_ragged_lengths_d64_bf16(fa, N):
    check_full(fa, 2, N, 3, 64, "bf16", 100 + N)


@pytest.mark.parametrize("B,N,H,dtype", [(1, 3000, 1, "fp16"), (1, 2500, 1, "bf16"),
                                         (1, 2000, 3, "bf16"), (1, 1537, 2, "fp16")])
def test_d256_key_splits_with_ragged_last_tile(fa, B, N, H, dtype):
    # d = 256 walks 128-key tiles with one K and one V stage.  These shapes cut
    # the K/V range into 3, 2, 2 and 1 shares whose last tile is ragged (56,
    # 68, 80 and 1 keys); split shares leave as fp32 partial rows through the
    # per-warp staging tiles and are merged afterwards
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = fa.fa_fwd_plan(B, H, N, 256, sms)
    assert plan["kernel"] == 0 and plan["kv_tile_rows"] == 128, plan
    check_full(fa, B, N, H, 256, dtype, 3300 + N, std=0.5)


@pytest.mark.parametrize("d", [64, 96, 128, 256])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("N", [1, 65, 129, 300])
def test_head_sizes_and_types(fa, d, dtype, N):
    check_full(fa, 1, N, 2, d, dtype, 200 + N + d)


def test_split_kv_path(fa):
    # one (b, h) with 24 Q tiles leaves most SMs idle, so the K/V range is
    # split and the partial results are merged
    check_full(fa, 1, 3000, 1, 64, "bf16", 301)
    check_full(fa, 1, 2500, 1, 128, "fp16", 302)
    check_full(fa, 1, 1900, 1, 256, "bf16", 303)
    check_full(fa, 1, 3000, 1, 96, "fp16", 304)


@pytest.mark.parametrize("B,N,H,d,dtype", [(1, 2000, 20, 64, "bf16"), (1, 2000, 20, 128, "fp16"),
                                             (1, 4096, 10, 64, "bf16"), (1, 2000, 20, 96, "bf16")])
def test_balanced_schedule(fa, B, N, H, d, dtype):
    # 160 units of 256 query rows on 148 SMs: every block takes an equal range
    # of (unit, K/V tile) steps, so units are cut in pieces on neighbouring
    # blocks and merged in the kernel by their log-sum-exps
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert fa.fa_fwd_plan(B, H, N, d, sms)["balanced"] == 1
    check_full(fa, B, N, H, d, dtype, 310 + d + N)


def test_workload_c1_tiny(fa):
    w = attn_inputs.WORKLOADS["c1"]
    check_full(fa, w.B, w.N, w.H, w.d, w.dtype, w.seed)


def test_workload_c2_detector_deep(fa):
    w = attn_inputs.WORKLOADS["c2"]
    check_full(fa, w.B, w.N, w.H, w.d, w.dtype, w.seed)


@pytest.mark.parametrize("name", ["c3", "c4", "sweep1024", "sweep2048", "sweep4096", "sweep8192",
                                  "c5"])
def test_full_size_workloads_sampled_rows(fa, name):
    w = attn_inputs.WORKLOADS[name]
    q, k, v = attn_inputs.draw_workload(w, count=3, device="cuda")
    o, lse = run(fa, q, k, v, w.scale)
    rows = sample_rows(w.B, w.H, w.N, 96)
    o_ref, lse_ref = oracle.attn_fwd_rows(to64(q), to64(k), to64(v), w.scale, rows)
    idx = np.array(rows)
    o_got = to64(o)[idx[:, 0], idx[:, 2], idx[:, 1]]
    lse_got = lse.cpu().double().numpy()[idx[:, 0], idx[:, 1], idx[:, 2]]
    eo, el = err_stats(o_got, o_ref), err_stats(lse_got, lse_ref)
    assert o_ok(eo), eo
    assert el["max"] <= LSE_MAX, el
    # properties that hold at any size, over every row: finite outputs, and
    # each output row inside the convex hull's bounding box of the V rows
    o32 = o.float()
    assert torch.isfinite(o32).all() and torch.isfinite(lse).all()
    vmax = v.float().amax(dim=1, keepdim=True)
    vmin = v.float().amin(dim=1, keepdim=True)
    tol = 1e-2 * (vmax - vmin + 1)
    assert bool(((o32 <= vmax + tol) & (o32 >= vmin - tol)).all())
    # LSE is at least the largest scaled score (sampled rows) and at most that plus ln N
    assert np.all(lse_got >= lse_ref - LSE_MAX)


def test_zero_queries_give_mean_of_values(fa):
    B, N, H, d = 2, 333, 2, 64
    _, k, v = attn_inputs.draw(B, N, H, d, "bf16", 401, 3, device="cuda")
    q = torch.zeros_like(k)
    o, lse = run(fa, q, k, v, 0.125)
    mean_v = v.double().mean(dim=1, keepdim=True)
    assert (o.double() - mean_v).abs().max().item() <= 1e-2
    assert (lse.double() - math.log(N)).abs().max().item() <= 1e-4


def test_constant_values(fa):
    B, N, H, d = 1, 517, 2, 128
    q, k, _ = attn_inputs.draw(B, N, H, d, "bf16", 402, 3, device="cuda")
    c = torch.linspace(-2, 2, d, device="cuda").to(torch.bfloat16)
    v = c.view(1, 1, 1, d).expand(B, N, H, d).contiguous()
    o, _ = run(fa, q, k, v, 1.0 / math.sqrt(d))
    # every P row sums to one, so O = c up to the rounding of P and of O
    assert (o.float() - c.float()).abs().max().item() <= 2e-2


def test_large_scale_is_stable(fa):
    # scale 64 on unit-norm rows: scores up to 64, one key dominates; without
    # the running max this overflows fp32 exponentials
    N, d = 256, 64
    k = torch.eye(N, d, device="cuda")[torch.randperm(N, generator=torch.Generator().manual_seed(5))]
    k = torch.nn.functional.normalize(k + 0.01, dim=-1).view(1, N, 1, d).to(torch.bfloat16)
    q = k.clone()
    _, _, v = attn_inputs.draw(1, N, 1, d, "bf16", 403, 3, device="cuda")
    o, lse = run(fa, q, k, v, 64.0)
    o_ref, lse_ref = oracle.attn_fwd(to64(q), to64(k), to64(v), 64.0)
    assert np.all(np.isfinite(to64(o)))
    assert err_stats(to64(o), o_ref)["max"] <= O_MAX
    assert err_stats(lse.cpu().double().numpy(), lse_ref)["max"] <= 1e-3 * 64


@pytest.mark.parametrize("N,d,sign", [(128, 64, 1), (256, 64, 1), (256, 64, -1), (256, 128, 1),
                                      (128, 256, 1), (256, 256, -1)])
def test_row_max_in_last_column_group(fa, N, d, sign):
    # Every row's dominant key sits in the last 8 columns of a 128-key tile,
    # 200 above the other scores (2^288 in base 2): a row max that left those
    # columns out would overflow the exponentials.  Rows of tile t's group use
    # the directions 8 t .. 8 t + 7, so no two dominant keys tie.  N = 128 runs
    # the single-tile kernel, N = 256 (d <= 128) the pair kernel; sign -1 takes
    # the min branch (negative scale).
    g = torch.Generator().manual_seed(77 + N + d)
    n_t = N // 128
    k = 0.01 * torch.randn(N, d, generator=g)
    q = torch.zeros(N, d)
    for t in range(n_t):
        for j in range(8):
            k[t * 128 + 120 + j] = 0.0
            k[t * 128 + 120 + j, 8 * t + j] = 1.0
    for i in range(N):
        c = i % (8 * n_t)
        q[i, c] = float(sign)
    to_dev = lambda x: x.view(1, N, 1, d).to(torch.bfloat16).cuda()  # noqa: E731
    q, k = to_dev(q), to_dev(k)
    _, _, v = attn_inputs.draw(1, N, 1, d, "bf16", 406 + N + d, 3, device="cuda")
    scale = 200.0 * sign
    o, lse = run(fa, q, k, v, scale)
    o_ref, lse_ref = oracle.attn_fwd(to64(q), to64(k), to64(v), scale)
    assert np.all(np.isfinite(to64(o))) and np.all(np.isfinite(lse.cpu().numpy()))
    assert err_stats(to64(o), o_ref)["max"] <= O_MAX
    assert err_stats(lse.cpu().double().numpy(), lse_ref)["max"] <= LSE_MAX


def test_deterministic(fa):
    w = attn_inputs.WORKLOADS["c3"]
    q, k, v = attn_inputs.draw_workload(w, count=3, device="cuda")
    o1, l1 = fa.forward(q, k, v, scale=w.scale)
    o2, l2 = fa.forward(q, k, v, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_negative_and_zero_scale(fa):
    check_full(fa, 1, 200, 2, 64, "bf16", 404, scale=-0.125)
    check_full(fa, 1, 200, 2, 64, "bf16", 405, scale=0.0)
