"""Pins for the fp64 oracle against what the pages and the mathematics fix.

None of these compares the oracle with a retyped copy of itself.  Each test
pins a property that a plausible mistake in the oracle would break:
closed forms (Q = 0, N = 1, constant V, a hand-worked one-dimensional case),
invariances (shifting every key by the same vector, permuting keys with their
values, permuting queries), one-hot dominance at large scale (also catches a
missing max subtraction, which overflows), head/batch independence (catches a
wrong stride in the [B, N, H, d] layout), the exactness of the online
recurrence against two-pass softmax (the pages' "not an approximation"), and
central finite differences for the backward pass.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

ORC = oracle.default()

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, std=1.0):
    return np.random.Generator(np.random.PCG64(seed)).standard_normal(shape) * std


# ----------------------------------------------------------------- forward

def check_probability_rows_sum_to_one(orc):
    q, k = rnd((2, 37, 3, 8), 1), rnd((2, 37, 3, 8), 2)
    p = orc.attn_probs(q, k, 0.7)
    assert p.shape == (2, 3, 37, 37)
    assert np.all(p >= 0.0)
    assert np.max(np.abs(p.sum(-1) - 1.0)) <= 1e-12


def check_zero_queries_give_mean_of_values(orc):
    B, N, H, d = 2, 29, 2, 5
    q = np.zeros((B, N, H, d))
    k, v = rnd((B, N, H, d), 3), rnd((B, N, H, d), 4)
    o, lse = orc.attn_fwd(q, k, v, 0.4)
    mean_v = v.mean(axis=1, keepdims=True)
    assert np.max(np.abs(o - mean_v)) <= 1e-13
    assert np.max(np.abs(lse - math.log(N))) <= 1e-13


def check_single_key_gives_its_value(orc):
    B, N, H, d = 3, 1, 2, 7
    q, k, v = rnd((B, N, H, d), 5), rnd((B, N, H, d), 6), rnd((B, N, H, d), 7)
    scale = 0.3
    o, lse = orc.attn_fwd(q, k, v, scale)
    assert np.array_equal(o, v)
    expect = scale * np.einsum("bnhx,bnhx->bhn", q, k)
    assert np.max(np.abs(lse - expect)) <= 1e-14


def check_constant_values_give_that_value(orc):
    B, N, H, d = 1, 41, 3, 6
    q, k = rnd((B, N, H, d), 8), rnd((B, N, H, d), 9)
    c = rnd((d,), 10)
    v = np.broadcast_to(c, (B, N, H, d)).copy()
    o, _ = orc.attn_fwd(q, k, v, 0.5)
    assert np.max(np.abs(o - c)) <= 1e-14


def check_hand_worked_one_dimensional_case(orc):
    # d = 1, scale = 1, q = 1: scores are the keys themselves.
    # keys (0, ln 3) give weights 1/4 and 3/4; values (0, 4) give O = 3; LSE = ln 4.
    q = np.ones((1, 2, 1, 1))
    k = np.array([0.0, math.log(3.0)]).reshape(1, 2, 1, 1)
    v = np.array([0.0, 4.0]).reshape(1, 2, 1, 1)
    o, lse = orc.attn_fwd(q, k, v, 1.0)
    assert abs(o[0, 0, 0, 0] - 3.0) <= 1e-15 and abs(o[0, 1, 0, 0] - 3.0) <= 1e-15
    assert abs(lse[0, 0, 0] - math.log(4.0)) <= 1e-15
    # three keys (ln 1, ln 2, ln 5), values (1, 2, 3), scale 1:
    # O = (1*1 + 2*2 + 5*3) / 8 = 2.5, LSE = ln 8.
    q = np.ones((1, 3, 1, 1))
    k = np.log(np.array([1.0, 2.0, 5.0])).reshape(1, 3, 1, 1)
    v = np.array([1.0, 2.0, 3.0]).reshape(1, 3, 1, 1)
    o, lse = orc.attn_fwd(q, k, v, 1.0)
    assert np.max(np.abs(o - 2.5)) <= 1e-15
    assert np.max(np.abs(lse - math.log(8.0))) <= 1e-15


def check_shift_of_every_key_leaves_output_and_shifts_lse(orc):
    B, N, H, d = 2, 33, 2, 8
    q, k, v = rnd((B, N, H, d), 11), rnd((B, N, H, d), 12), rnd((B, N, H, d), 13)
    u = rnd((d,), 14)
    scale = 0.35
    o1, lse1 = orc.attn_fwd(q, k, v, scale)
    o2, lse2 = orc.attn_fwd(q, k + u, v, scale)
    assert np.max(np.abs(o1 - o2)) <= 1e-13
    shift = scale * np.einsum("bnhx,x->bhn", q, u)
    assert np.max(np.abs(lse2 - lse1 - shift)) <= 1e-12


def check_permutations(orc):
    B, N, H, d = 1, 27, 2, 4
    q, k, v = rnd((B, N, H, d), 15), rnd((B, N, H, d), 16), rnd((B, N, H, d), 17)
    perm = np.random.Generator(np.random.PCG64(18)).permutation(N)
    o, lse = orc.attn_fwd(q, k, v, 0.6)
    o_kv, lse_kv = orc.attn_fwd(q, k[:, perm], v[:, perm], 0.6)
    assert np.max(np.abs(o - o_kv)) <= 1e-13 and np.max(np.abs(lse - lse_kv)) <= 1e-13
    o_q, lse_q = orc.attn_fwd(q[:, perm], k, v, 0.6)
    assert np.max(np.abs(o[:, perm] - o_q)) <= 1e-15
    assert np.max(np.abs(lse[:, :, perm] - lse_q)) <= 1e-15


def check_one_hot_dominance_at_large_scale(orc):
    # q_i equal to k_{pi(i)} with unit-norm keys: at scale 1000 every other key
    # is exp(-1000 * gap) smaller, so O_i = V_{pi(i)} to rounding.  Without the
    # max subtraction exp(1000) overflows and this fails.
    B, N, H, d = 1, 16, 1, 16
    k = np.eye(N).reshape(B, N, H, d)
    v = rnd((B, N, H, d), 19)
    perm = np.random.Generator(np.random.PCG64(20)).permutation(N)
    q = k[:, perm].copy()
    o, lse = orc.attn_fwd(q, k, v, 1000.0)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert np.max(np.abs(o - v[:, perm])) <= 1e-12
    assert np.max(np.abs(lse - 1000.0)) <= 1e-12


def check_heads_and_batches_are_independent(orc):
    # Computing all (b, h) at once must equal computing each head alone:
    # catches a wrong head or token stride in the [B, N, H, d] indexing.
    B, N, H, d = 2, 19, 3, 5
    q, k, v = rnd((B, N, H, d), 21), rnd((B, N, H, d), 22), rnd((B, N, H, d), 23)
    o, lse = orc.attn_fwd(q, k, v, 0.45)
    for b in range(B):
        for h in range(H):
            sl = (slice(b, b + 1), slice(None), slice(h, h + 1), slice(None))
            o1, l1 = orc.attn_fwd(q[sl], k[sl], v[sl], 0.45)
            assert np.array_equal(o1[0, :, 0], o[b, :, h])
            assert np.array_equal(l1[0, 0], lse[b, h])


def check_rows_entry_point_matches_full_forward(orc):
    B, N, H, d = 2, 23, 2, 6
    q, k, v = rnd((B, N, H, d), 24), rnd((B, N, H, d), 25), rnd((B, N, H, d), 26)
    o, lse = orc.attn_fwd(q, k, v, 0.3)
    rows = [(0, 0, 0), (1, 1, 22), (1, 0, 7), (0, 1, 13)]
    o_r, lse_r = orc.attn_fwd_rows(q, k, v, 0.3, rows)
    for r, (b, h, i) in enumerate(rows):
        assert np.array_equal(o_r[r], o[b, i, h])
        assert lse_r[r] == lse[b, h, i]


def check_definition_matches_two_pass_form(orc):
    B, N, H, d = 1, 70, 2, 9
    q, k, v = rnd((B, N, H, d), 27), rnd((B, N, H, d), 28), rnd((B, N, H, d), 29)
    o, lse = orc.attn_fwd(q, k, v, 0.33)
    o2, lse2 = orc.attn_fwd_two_pass(q, k, v, 0.33)
    assert np.max(np.abs(o - o2)) <= 64 * N * 2.0 ** -53 * np.max(np.abs(v))
    assert np.max(np.abs(lse - lse2)) <= 1e-14


def check_online_recurrence_bit_equal_with_one_kv_block(orc, block_q):
    # A single K/V block: every rescale multiplies 0 by exp(-inf) = 0 and the
    # sums run in the same order as the two-pass form, so fp64 results agree
    # bit for bit ("only floating-point order differences", YOLO11 page 2.2).
    B, N, H, d = 1, 100, 2, 8
    q, k, v = rnd((B, N, H, d), 30), rnd((B, N, H, d), 31), rnd((B, N, H, d), 32)
    o1, l1 = orc.attn_fwd_two_pass(q, k, v, 0.4)
    o2, l2 = orc.attn_fwd_online(q, k, v, 0.4, block_q, N)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def check_online_recurrence_bit_equal_when_max_is_in_first_block(orc, block_kv):
    # Key 0 dominates every query's scores, so the running max is fixed after
    # the first block and every later alpha is exp(0) = 1 exactly.
    B, N, H, d = 1, 90, 1, 8
    g = np.random.Generator(np.random.PCG64(33))
    q = np.abs(g.standard_normal((B, N, H, d))) + 0.5
    k = g.standard_normal((B, N, H, d)) * 0.1
    k[:, 0] = 10.0
    v = g.standard_normal((B, N, H, d))
    o1, l1 = orc.attn_fwd_two_pass(q, k, v, 0.4)
    o2, l2 = orc.attn_fwd_online(q, k, v, 0.4, 16, block_kv)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def check_online_recurrence_equals_definition_to_rounding(orc, block_q, block_kv):
    B, N, H, d = 2, 150, 2, 8
    q, k, v = rnd((B, N, H, d), 34, 2.0), rnd((B, N, H, d), 35), rnd((B, N, H, d), 36)
    o1, l1 = orc.attn_fwd(q, k, v, 0.5)
    o2, l2 = orc.attn_fwd_online(q, k, v, 0.5, block_q, block_kv)
    bound = 8 * N * 2.0 ** -53 * np.max(np.abs(v))
    assert np.max(np.abs(o1 - o2)) <= bound
    assert np.max(np.abs(l1 - l2)) <= 1e-13


# ---------------------------------------------------------------- backward

def _loss(orc, q, k, v, dout, scale, causal=False):
    o, _ = orc.attn_fwd(q, k, v, scale, causal)
    return float(np.sum(o * dout))


def check_backward_matches_central_finite_differences(orc, B, N, H, d):
    q, k, v = rnd((B, N, H, d), 40), rnd((B, N, H, d), 41), rnd((B, N, H, d), 42)
    dout = rnd((B, N, H, d), 43)
    scale = 0.7
    dq, dk, dv = orc.attn_bwd(q, k, v, dout, scale)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (_loss(orc, args_p["q"], args_p["k"], args_p["v"], dout, scale)
                       - _loss(orc, args_m["q"], args_m["k"], args_m["v"], dout, scale)) / (2 * h)
        err = np.max(np.abs(fd - g))
        assert err <= 1e-6 * max(1.0, np.max(np.abs(g))), (name, err)


def check_score_gradient_rows_sum_to_zero(orc):
    B, N, H, d = 2, 21, 2, 5
    q, k, v, dout = (rnd((B, N, H, d), s) for s in (44, 45, 46, 47))
    ds = orc.attn_dscores(q, k, v, dout, 0.5)
    assert np.max(np.abs(ds.sum(-1))) <= 1e-13


def check_backward_closed_forms(orc):
    # N = 1: O = V regardless of Q and K, so dV = dO and dQ = dK = 0.
    B, N, H, d = 2, 1, 3, 4
    q, k, v, dout = (rnd((B, N, H, d), s) for s in (48, 49, 50, 51))
    dq, dk, dv = orc.attn_bwd(q, k, v, dout, 0.9)
    assert np.array_equal(dv, dout)
    assert np.max(np.abs(dq)) == 0.0 and np.max(np.abs(dk)) == 0.0
    # Q = 0: P = 1/N everywhere, so dV_j = mean_i dO_i and dK = scale dS^T Q = 0.
    B, N, H, d = 1, 13, 2, 3
    q = np.zeros((B, N, H, d))
    k, v, dout = (rnd((B, N, H, d), s) for s in (52, 53, 54))
    dq, dk, dv = orc.attn_bwd(q, k, v, dout, 0.9)
    assert np.max(np.abs(dv - dout.mean(axis=1, keepdims=True))) <= 1e-14
    assert np.max(np.abs(dk)) == 0.0


def check_backward_row_ranges_partition_the_full_backward(orc):
    # dQ rows come out exact from their own range; dK and dV are sums over
    # rows, so the pieces of any partition of [0, N) add up to the whole.
    B, N, H, d = 1, 30, 2, 4
    q, k, v, dout = (rnd((B, N, H, d), s) for s in (55, 56, 57, 58))
    full = orc.attn_bwd(q, k, v, dout, 0.6)
    parts = [orc.attn_bwd_rows(q, k, v, dout, 0.6, a, b) for a, b in ((0, 7), (7, 8), (8, 30))]
    assert np.array_equal(sum(p[0] for p in parts), full[0])
    for g in (1, 2):
        assert np.max(np.abs(sum(p[g] for p in parts) - full[g])) <= 1e-13


# ----------------------------------------------------------- page fixtures

def test_page_printed_shapes():
    from attn_inputs import WORKLOADS
    items = {it["id"]: it for it in json.load(open(os.path.join(GOLDEN, "page_shapes.json")))["items"]}
    a = items["llm_n8192_d128"]
    assert a["N"] * a["d"] == a["qkv_elements"]
    assert a["N"] * a["N"] == a["score_elements"]
    assert a["score_elements"] // a["qkv_elements"] == a["ratio"]
    w4 = WORKLOADS["c4"]
    assert (w4.N, w4.d) == (a["N"], a["d"])
    b = items["yolo11_n400_block64"]
    assert -(-b["N"] // b["block"]) == b["blocks"]
    c = items["yolo11_map20"]
    assert c["map"][0] * c["map"][1] == c["N"] == WORKLOADS["c1"].N == WORKLOADS["c2"].N
    assert c["N"] ** 2 == c["score_elements"]
    e = items["yolov13_neck_map80_c256"]
    w3 = WORKLOADS["c3"]
    assert e["map"][0] * e["map"][1] == e["N"] == w3.N and w3.H * w3.d == e["C"]
    f = items["yolov12_stage1_map160"]
    assert f["map"][0] * f["map"][1] == f["N"]
    assert f["qkv_width"] == 3 * f["C"]
    w6 = WORKLOADS["y12s1"]
    assert (w6.N, w6.H * w6.d) == (f["N"], f["C"])


# ------------------------------------------------- tests on the real oracle

# Every check above, in order; tests/test_oracle_mutants.py reruns the same
# list against oracle copies with planted mistakes.
# ------------------------------------------------------------ causal mask
# LLM explainer page, section 7.1: the causal mask hides every future position
# from a query.  Row i sees keys j <= i.

def check_causal_first_row_is_first_value(orc):
    # row 0 sees only key 0: O_0 = V_0, LSE_0 = scale q_0 . k_0
    B, N, H, d = 2, 9, 2, 5
    q, k, v = rnd((B, N, H, d), 60), rnd((B, N, H, d), 61), rnd((B, N, H, d), 62)
    o, lse = orc.attn_fwd(q, k, v, 0.6, causal=True)
    assert np.array_equal(o[:, 0], v[:, 0])
    expect = 0.6 * np.einsum("bhx,bhx->bh", q[:, 0], k[:, 0])
    assert np.max(np.abs(lse[:, :, 0] - expect)) <= 1e-14


def check_causal_rows_equal_attention_over_their_prefix(orc):
    # brute force: causal row i is ordinary attention of q_i over keys and
    # values 0..i (a problem of i + 1 positions, computed without the mask)
    B, N, H, d = 1, 12, 2, 4
    q, k, v = rnd((B, N, H, d), 63), rnd((B, N, H, d), 64), rnd((B, N, H, d), 65)
    o, lse = orc.attn_fwd(q, k, v, 0.8, causal=True)
    for i in range(N):
        op, lp = orc.attn_fwd(q[:, :i + 1], k[:, :i + 1], v[:, :i + 1], 0.8)
        assert np.max(np.abs(o[:, i] - op[:, i])) <= 1e-14, i
        assert np.max(np.abs(lse[:, :, i] - lp[:, :, i])) <= 1e-14, i
    # the last row sees every key: it matches the unmasked forward
    o_full, lse_full = orc.attn_fwd(q, k, v, 0.8)
    assert np.max(np.abs(o[:, -1] - o_full[:, -1])) <= 1e-14


def check_causal_probabilities_are_lower_triangular(orc):
    q, k = rnd((1, 23, 2, 6), 66), rnd((1, 23, 2, 6), 67)
    p = orc.attn_probs(q, k, 0.9, causal=True)
    upper = np.triu(np.ones((23, 23), dtype=bool), 1)
    assert np.all(p[..., upper] == 0.0)
    assert np.all(p[..., ~upper] > 0.0)
    assert np.max(np.abs(p.sum(-1) - 1.0)) <= 1e-12


def check_causal_backward_matches_central_finite_differences(orc):
    B, N, H, d = 1, 6, 2, 3
    q, k, v = rnd((B, N, H, d), 68), rnd((B, N, H, d), 69), rnd((B, N, H, d), 70)
    dout = rnd((B, N, H, d), 71)
    scale = 0.7
    dq, dk, dv = orc.attn_bwd(q, k, v, dout, scale, causal=True)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (_loss(orc, args_p["q"], args_p["k"], args_p["v"], dout, scale, True)
                       - _loss(orc, args_m["q"], args_m["k"], args_m["v"], dout, scale, True)) / (2 * h)
        err = np.max(np.abs(fd - g))
        assert err <= 1e-6 * max(1.0, np.max(np.abs(g))), (name, err)
    # the last key is seen by the last query only: dV_{N-1} = P_{N-1,N-1} dO_{N-1}
    p = orc.attn_probs(q, k, scale, causal=True)
    expect = p[0, :, N - 1, N - 1][:, None] * dout[0, N - 1]
    assert np.max(np.abs(dv[0, N - 1] - expect)) <= 1e-14



def _numpy_attention(q, k, v, dout, scale, causal):
    """Attention and its gradients written with numpy's einsum and exp in
    fp64, independently of the C oracle: the definition (YOLO11 page,
    section 1.2) and the chain rule through softmax."""
    N = q.shape[1]
    s = scale * np.einsum("bihx,bjhx->bhij", q, k)
    if causal:
        s = np.where(np.tril(np.ones((N, N), dtype=bool)), s, -np.inf)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=-1, keepdims=True)
    p = e / z
    o = np.einsum("bhij,bjhx->bihx", p, v)
    lse = (m + np.log(z))[..., 0]
    dv = np.einsum("bhij,bihx->bjhx", p, dout)
    dp = np.einsum("bihx,bjhx->bhij", dout, v)
    dd = (p * dp).sum(axis=-1, keepdims=True)
    ds = p * (dp - dd)
    dq = scale * np.einsum("bhij,bjhx->bihx", ds, k)
    dk = scale * np.einsum("bhij,bihx->bjhx", ds, q)
    return o, lse, dq, dk, dv


def check_numpy_restatement_agrees(orc):
    # N <= 64: the C oracle and an independent numpy restatement agree to
    # 1e-12 on O, the LSE and all three gradients, with and without the mask
    for seed, (B, N, H, d), causal in [(80, (2, 64, 3, 16), False), (81, (1, 33, 2, 64), True),
                                       (82, (3, 1, 1, 8), False), (83, (1, 50, 4, 32), True)]:
        q, k, v, dout = (rnd((B, N, H, d), seed + 10 * i) for i in range(4))
        scale = 1.0 / math.sqrt(d)
        o, lse = orc.attn_fwd(q, k, v, scale, causal=causal)
        grads = orc.attn_bwd(q, k, v, dout, scale, causal=causal)
        want = _numpy_attention(q, k, v, dout, scale, causal)
        for got, ref in zip((o, lse, *grads), want):
            assert np.max(np.abs(got - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))

CHECKS = [check_probability_rows_sum_to_one, check_zero_queries_give_mean_of_values, check_single_key_gives_its_value, check_constant_values_give_that_value, check_hand_worked_one_dimensional_case, check_shift_of_every_key_leaves_output_and_shifts_lse, check_permutations, check_one_hot_dominance_at_large_scale, check_heads_and_batches_are_independent, check_rows_entry_point_matches_full_forward, check_definition_matches_two_pass_form, check_online_recurrence_bit_equal_with_one_kv_block, check_online_recurrence_bit_equal_when_max_is_in_first_block, check_online_recurrence_equals_definition_to_rounding, check_backward_matches_central_finite_differences, check_score_gradient_rows_sum_to_zero, check_backward_closed_forms, check_backward_row_ranges_partition_the_full_backward, check_causal_first_row_is_first_value, check_causal_rows_equal_attention_over_their_prefix, check_causal_probabilities_are_lower_triangular, check_causal_backward_matches_central_finite_differences, check_numpy_restatement_agrees]

def test_probability_rows_sum_to_one():
    check_probability_rows_sum_to_one(ORC)


def test_zero_queries_give_mean_of_values():
    check_zero_queries_give_mean_of_values(ORC)


def test_single_key_gives_its_value():
    check_single_key_gives_its_value(ORC)


def test_constant_values_give_that_value():
    check_constant_values_give_that_value(ORC)


def test_hand_worked_one_dimensional_case():
    check_hand_worked_one_dimensional_case(ORC)


def test_shift_of_every_key_leaves_output_and_shifts_lse():
    check_shift_of_every_key_leaves_output_and_shifts_lse(ORC)


def test_permutations():
    check_permutations(ORC)


def test_one_hot_dominance_at_large_scale():
    check_one_hot_dominance_at_large_scale(ORC)


def test_heads_and_batches_are_independent():
    check_heads_and_batches_are_independent(ORC)


def test_rows_entry_point_matches_full_forward():
    check_rows_entry_point_matches_full_forward(ORC)


def test_definition_matches_two_pass_form():
    check_definition_matches_two_pass_form(ORC)


@pytest.mark.parametrize("block_q", [1, 7, 64, 128])
def test_online_recurrence_bit_equal_with_one_kv_block(block_q):
    check_online_recurrence_bit_equal_with_one_kv_block(ORC, block_q)


@pytest.mark.parametrize("block_kv", [1, 7, 64])
def test_online_recurrence_bit_equal_when_max_is_in_first_block(block_kv):
    check_online_recurrence_bit_equal_when_max_is_in_first_block(ORC, block_kv)


@pytest.mark.parametrize("block_q,block_kv", [(1, 1), (16, 5), (64, 64), (128, 32)])
def test_online_recurrence_equals_definition_to_rounding(block_q, block_kv):
    check_online_recurrence_equals_definition_to_rounding(ORC, block_q, block_kv)


@pytest.mark.parametrize("B,N,H,d", [(1, 5, 2, 3), (1, 8, 1, 4), (1, 1, 2, 2)])
def test_backward_matches_central_finite_differences(B, N, H, d):
    check_backward_matches_central_finite_differences(ORC, B, N, H, d)


def test_score_gradient_rows_sum_to_zero():
    check_score_gradient_rows_sum_to_zero(ORC)


def test_backward_closed_forms():
    check_backward_closed_forms(ORC)


def test_backward_row_ranges_partition_the_full_backward():
    check_backward_row_ranges_partition_the_full_backward(ORC)


def test_causal_first_row_is_first_value():
    check_causal_first_row_is_first_value(ORC)


def test_causal_rows_equal_attention_over_their_prefix():
    check_causal_rows_equal_attention_over_their_prefix(ORC)


def test_causal_probabilities_are_lower_triangular():
    check_causal_probabilities_are_lower_triangular(ORC)


def test_causal_backward_matches_central_finite_differences():
    check_causal_backward_matches_central_finite_differences(ORC)


def test_numpy_restatement_agrees():
    check_numpy_restatement_agrees(ORC)


def test_c1_unrounded_draws_report():
    # Workload C1 draws fp32 inputs; the GPU receives them rounded to bf16
    # and parity is measured against the oracle on those rounded values.
    # Informational: the effect of that rounding on the exact result, which
    # bench.py reports beside the GPU error.  It stays below the output bar.
    import attn_inputs
    w = attn_inputs.WORKLOADS["c1"]
    raw = attn_inputs.draw_fp32(w.B, w.N, w.H, w.d, w.seed, count=3)
    rounded = attn_inputs.draw_workload(w, count=3)
    o_raw, lse_raw = ORC.attn_fwd(*(x.astype(np.float64) for x in raw), w.scale)
    o_rnd, lse_rnd = ORC.attn_fwd(*(attn_inputs.to_f64(t) for t in rounded), w.scale)
    d_o, d_l = np.max(np.abs(o_rnd - o_raw)), np.max(np.abs(lse_rnd - lse_raw))
    assert 0.0 < d_o < 2e-2 and 0.0 < d_l < 1e-2, (d_o, d_l)
