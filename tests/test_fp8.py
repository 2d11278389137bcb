"""Forward pass on 8-bit (E4M3) Q, K, V against the fp64 oracle.

The oracle computes the plain definition on the decoded inputs times their
descale factors.  The GPU rounds P to E4M3 before the P.V product (the row
sums use the unrounded values), so its O differs from the exact one by up to
the rounding of every P_ij.  Each O element is compared against its own
bound, derived from that arithmetic:
  * P is stored relative to a reference max that is at most the true row max,
    so a stored value is p = 2^k exp(s_ij - m_i) <= 2^8 with k >= 0 and the
    row sum l_i >= sum_j exp(s_ij - m_i) >= 1;
  * rounding to E4M3 changes p by at most 2^-4 p (normal range, 3 mantissa
    bits) and by at most 2^-10 below 2^-6 (subnormal spacing 2^-9), so the
    normalised weight P_ij moves by at most max(2^-4 P_ij, 2^-10 / l_i);
  * the exponentials (MUFU or the FMA polynomial, relative error < 1e-4),
    the fp32 scores and the fp32 accumulation over N keys add at most
    (2^-8 + N 2^-24) of sum_j P_ij |V_jx|, and O is rounded to bf16 (2^-8).
  |O_gpu - O_ref|_ix <= sum_j max(2^-4 P_ij, 2^-10/l_i) |V_jx| (1 + 2^-8)
                        + N 2^-24 sum_j P_ij |V_jx| + 2^-8 |O_ref,ix| + 1e-6.
The LSE does not see the rounding of P and keeps the 16-bit bar (1e-3).
P, l and m for the bound are recomputed in fp64 from the same decoded inputs
(the expected O and LSE come from the oracle alone).
"""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from tests.gpu_helpers import LSE_MAX, err_stats, guard_intact, guarded, sample_rows, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_attention_144_b200 as fa
    fa.fa_get_device_status(clear=True)
    yield fa
    assert fa.fa_get_device_status() == 0, "a kernel gave up a bounded wait"


def weights_rows(q, k, scale, rows, causal):
    """fp64 P rows and l for the (b, h, i) in rows: P [R, N], l [R]."""
    N = k.shape[1]
    P, L = [], []
    for (b, h, i) in rows:
        s = scale * (k[b, :, h, :] @ q[b, i, h, :])
        if causal:
            s[i + 1:] = -np.inf
        m = s.max()
        p = np.exp(s - m)
        L.append(p.sum())
        P.append(p / L[-1])
    return np.array(P), np.array(L)


def bound_rows(q, k, v, scale, rows, o_ref_rows, causal):
    N = k.shape[1]
    P, L = weights_rows(q, k, scale, rows, causal)
    dP = np.where(P > 0, np.maximum(2.0 ** -4 * P, 2.0 ** -10 / L[:, None]), 0.0)
    av = np.stack([np.abs(v[b, :, h, :]) for (b, h, _) in rows])  # [R, N, d]
    wsum = np.einsum("rn,rnd->rd", dP, av)
    psum = np.einsum("rn,rnd->rd", P, av)
    return (wsum * (1 + 2.0 ** -8) + N * 2.0 ** -24 * psum + 2.0 ** -8 * np.abs(o_ref_rows)
            + 1e-6)


def run(fa, q8, k8, v8, scale, dq, dk, dv, causal):
    B, N, H, d = q8.shape
    o, o_flat = guarded((B, N, H, d), torch.bfloat16)
    lse, l_flat = guarded((B, H, N), torch.float32)
    fa.fa_fwd_fp8(q8, k8, v8, dq, dk, dv, o=o, lse=lse, scale=scale,
                  flags=fa.FA_FLAG_CAUSAL if causal else 0)
    torch.cuda.synchronize()
    assert guard_intact(o_flat) and guard_intact(l_flat), "write past the end of an output"
    return o, lse


def check(fa, B, N, H, seed, dq=1.0, dk=1.0, dv=1.0, causal=False, std=1.0, rows=None,
          scale=None):
    d = 128
    q8, k8, v8 = attn_inputs.draw(B, N, H, d, "fp8", seed, 3, std=std, device="cuda")
    scale = float(np.float32(1.0 / math.sqrt(d))) if scale is None else scale
    o, lse = run(fa, q8, k8, v8, scale, dq, dk, dv, causal)
    q, k, v = to64(q8) * dq, to64(k8) * dk, to64(v8) * dv
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(N)]
        o_ref, lse_ref = oracle.attn_fwd(q, k, v, scale, causal=causal)
        o_ref_rows = np.stack([o_ref[b, i, h] for (b, h, i) in rows])
        lse_ref_rows = np.array([lse_ref[b, h, i] for (b, h, i) in rows])
    else:
        o_ref_rows, lse_ref_rows = oracle.attn_fwd_rows(q, k, v, scale, rows, causal=causal)
    idx = np.array(rows)
    o_got = to64(o)[idx[:, 0], idx[:, 2], idx[:, 1]]
    lse_got = lse.cpu().double().numpy()[idx[:, 0], idx[:, 1], idx[:, 2]]
    assert np.all(np.isfinite(o_got)) and np.all(np.isfinite(lse_got))
    bnd = bound_rows(q, k, v, scale, rows, o_ref_rows, causal)
    err = np.abs(o_got - o_ref_rows)
    worst = np.unravel_index(np.argmax(err / bnd), err.shape)
    assert np.all(err <= bnd), (float((err / bnd).max()), rows[worst[0]], worst[1],
                                float(err[worst]), float(bnd[worst]))
    el = err_stats(lse_got, lse_ref_rows)
    assert el["max"] <= LSE_MAX, el
    return err_stats(o_got, o_ref_rows), el


@pytest.mark.parametrize("N", [1, 2, 65, 127, 128, 129, 256, 300, 1000])
def test_fp8_ragged_lengths(fa, N):
    check(fa, 2, N, 2, 2100 + N)


@pytest.mark.parametrize("N", [1, 100, 129, 513])
def test_fp8_causal(fa, N):
    check(fa, 2, N, 2, 2200 + N, causal=True)


def test_fp8_descale_factors(fa):
    # the problem is attention on (descale_q Q, descale_k K, descale_v V);
    # std 4 draws use more of E4M3's range
    check(fa, 1, 700, 3, 2301, dq=0.5, dk=0.125, dv=3.0, std=4.0)
    check(fa, 1, 300, 2, 2302, dq=2.0, dk=1.5, dv=0.25, causal=True)


def test_fp8_split_kv_and_balanced_schedules(fa):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # one head of 24 Q tiles: split K/V ranges merged by fa_combine_kernel
    assert fa.fa_fwd_plan(1, 1, 3000, 128, sms)["n_split"] > 1
    check(fa, 1, 3000, 1, 2401)
    # 160 units on 148 SMs: units cut across blocks and merged in the kernel
    assert fa.fa_fwd_plan(1, 20, 2000, 128, sms)["balanced"] == 1
    check(fa, 1, 2000, 20, 2402, rows=sample_rows(1, 20, 2000, 160))


def test_fp8_long_sequence_sampled_rows(fa):
    w = attn_inputs.WORKLOADS["c4fp8"]
    o_stats, _ = check(fa, w.B, w.N, w.H, w.seed, rows=sample_rows(w.B, w.H, w.N, 96))
    assert o_stats["rms_rel"] <= 0.05, o_stats


def test_fp8_deterministic(fa):
    q8, k8, v8 = attn_inputs.draw(1, 1500, 4, 128, "fp8", 2501, 3, device="cuda")
    a = fa.fa_fwd_fp8(q8, k8, v8, 0.5, 0.5, 2.0)
    b = fa.fa_fwd_fp8(q8, k8, v8, 0.5, 0.5, 2.0)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
