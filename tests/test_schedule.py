"""Host logic of the forward's work decomposition (no GPU needed).

fa_fwd_plan and fa_fwd_plan_pieces run the same C++ code that the forward
kernels use to decide which (unit, K/V tile) steps each block processes and
how the pieces of a unit cut across blocks are merged.  These tests check,
for many shapes and SM counts, that every step of every unit is processed
exactly once, that each cut unit has exactly one merging piece whose peers
are exactly the blocks that hold its other pieces, and that a block only ever
waits for blocks after it (so the waits cannot form a cycle).
"""
import pytest

import exact_attention_144_b200 as fa

WHOLE, PARTIAL, MERGE = 0, 1, 2

SHAPES = [
    # (B, H, N, d): the workloads, the N sweep, ragged tails, few and many units
    (1, 2, 400, 64), (32, 4, 400, 64), (1, 1, 6400, 256), (1, 8, 8192, 128),
    (1, 8, 1024, 64), (1, 8, 2048, 64), (1, 8, 4096, 64), (1, 8, 8192, 64), (4, 8, 4096, 64),
    (1, 10, 2000, 64), (1, 20, 2000, 64), (1, 10, 4096, 64), (1, 3, 8192, 64), (2, 3, 5000, 128), (1, 1, 1, 64), (3, 1, 129, 128),
    (1, 7, 4097, 64), (2, 16, 4096, 128), (1, 1, 100000, 64), (8, 16, 2048, 64),
    (1, 1, 400, 96), (2, 4, 1600, 96), (1, 8, 8192, 96),  # d = 96: the d = 128 tile shapes
]
SMS = [148, 132, 7, 1]


def all_pieces(B, H, N, d, sms):
    plan = fa.fa_fwd_plan(B, H, N, d, sms)
    return plan, [fa.fa_fwd_plan_pieces(B, H, N, d, sms, blk) for blk in range(plan["grid"])]


@pytest.mark.parametrize("sms", SMS)
@pytest.mark.parametrize("shape", SHAPES)
def test_every_step_once_and_merges_acyclic(shape, sms):
    B, H, N, d = shape
    plan, blocks = all_pieces(B, H, N, d, sms)
    assert 1 <= plan["grid"] <= sms
    n_units, n_kvt, n_split = plan["n_units"], plan["n_kv_tiles"], plan["n_split"]
    n_qt = -(-N // plan["unit_rows"])
    assert n_units == B * H * n_qt * n_split
    assert n_kvt == -(-N // plan["kv_tile_rows"])
    seen = {}  # (b, h, qt, K/V tile) -> block
    for blk, pieces in enumerate(blocks):
        for idx, (u, t0, t1, kind, peer0, npeer) in enumerate(pieces):
            assert 0 <= u < n_units and 0 <= t0 < t1 <= n_kvt
            qt, bh = u % n_qt, u // (n_qt * n_split)
            for t in range(t0, t1):
                key = (bh, qt, t)
                assert key not in seen, f"step {key} processed twice"
                seen[key] = blk
            if kind == PARTIAL:
                assert plan["balanced"] and idx == 0 and t0 > 0
            elif kind == MERGE:
                assert plan["balanced"] and idx == len(pieces) - 1 and t0 == 0 and t1 < n_kvt
                assert peer0 == blk + 1 and npeer >= 1  # waits only on later blocks
            else:
                assert kind == WHOLE
                if plan["balanced"]:
                    assert (t0, t1) == (0, n_kvt)
    # every K/V tile of every Q unit of every (batch, head), nothing else
    assert set(seen) == {(bh, qt, t) for bh in range(B * H) for qt in range(n_qt)
                         for t in range(n_kvt)}
    if plan["balanced"]:
        holders = {}
        for (bh, qt, t), blk in seen.items():
            holders.setdefault(bh * n_qt + qt, set()).add(blk)
        for blk, pieces in enumerate(blocks):
            for (u, t0, t1, kind, peer0, npeer) in pieces:
                # merge peers are exactly the blocks holding the unit's other pieces
                if kind == MERGE:
                    assert holders[u] == {blk} | set(range(peer0, peer0 + npeer))
                elif kind == WHOLE:
                    assert holders[u] == {blk}
        # each block has at most one partial slot, used by its first piece only
        for pieces in blocks:
            assert sum(1 for p in pieces if p[3] == PARTIAL) <= 1
    else:
        # round-robin: unit u runs on block u mod grid, each unit once
        units = sorted(p[0] for pieces in blocks for p in pieces)
        assert units == list(range(n_units))
        for blk, pieces in enumerate(blocks):
            assert all(p[0] % plan["grid"] == blk for p in pieces)


@pytest.mark.parametrize("shape", SHAPES)
def test_balanced_ranges_are_even(shape):
    B, H, N, d = shape
    plan, blocks = all_pieces(B, H, N, d, 148)
    if not plan["balanced"]:
        return
    steps = [sum(t1 - t0 for (_, t0, t1, *_rest) in pieces) for pieces in blocks]
    assert max(steps) - min(steps) <= 1
    assert plan["grid"] == 148 and plan["n_split"] == 1 and plan["kernel"] == 1


def test_workload_plans():
    # the training workload and the long-sequence workload leave a partial last
    # wave (512 and 256 units on 148 SMs) and take the balanced schedule
    for shape in [(4, 8, 4096, 64), (1, 8, 8192, 128), (1, 8, 8192, 64)]:
        plan = fa.fa_fwd_plan(*shape, 148)
        assert plan["balanced"] == 1 and plan["grid"] == 148, plan
        assert plan["scratch_bytes"] == 4 * (148 * 256 * shape[3] + 148 * 256 + 148)
    # the neck workload (one head, d = 256): 50 Q tiles, K/V range split in two
    plan = fa.fa_fwd_plan(1, 1, 6400, 256, 148)
    assert (plan["kernel"], plan["n_split"], plan["n_units"], plan["balanced"]) == (0, 2, 100, 0)
    assert plan["kv_tile_rows"] == 128
    # the detector deep stage: short units (4 K/V tiles) stay round-robin
    plan = fa.fa_fwd_plan(32, 4, 400, 64, 148)
    assert (plan["kernel"], plan["n_units"], plan["balanced"], plan["n_split"]) == (1, 256, 0, 1)
    # one long head (the YOLOv12 stage-1 map, d = 96): 100 units of 200 K/V
    # tiles leave 48 SMs idle round-robin, and long units are worth cutting
    plan = fa.fa_fwd_plan(1, 1, 25600, 96, 148)
    assert (plan["kernel"], plan["n_units"], plan["balanced"], plan["grid"]) == (1, 100, 1, 148)
    # fewer units than SMs but short ones (32 K/V tiles) stay whole
    plan = fa.fa_fwd_plan(1, 8, 4096, 64, 148)
    assert (plan["n_units"], plan["balanced"], plan["grid"]) == (128, 0, 128)
    # a single short head: one 128-row tile kernel unit per tile
    plan = fa.fa_fwd_plan(1, 2, 128, 64, 148)
    assert (plan["kernel"], plan["unit_rows"], plan["n_units"]) == (0, 128, 2)


def test_plan_rejects_bad_arguments():
    for args in [(0, 1, 1, 64, 148), (1, 0, 1, 64, 148), (1, 1, 0, 64, 148), (1, 1, 1, 64, 0)]:
        with pytest.raises(fa.FAError) as e:
            fa.fa_fwd_plan(*args)
        assert e.value.status == fa.FA_ERR_SHAPE
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_plan(1, 1, 64, 80, 148)
    assert e.value.status == fa.FA_ERR_HEADDIM
    with pytest.raises(fa.FAError):
        fa.fa_fwd_plan_pieces(1, 1, 64, 64, 148, 5)  # block past the grid


# ------------------------------------------------------------------ causal
CAUSAL = 1


@pytest.mark.parametrize("sms", [148, 7, 1])
@pytest.mark.parametrize("shape", SHAPES)
def test_causal_units_cover_up_to_their_diagonal(shape, sms):
    # with the causal mask a unit of query rows [a, b) needs exactly the K/V
    # tiles holding keys 0 .. b-1; every unit runs once, whole, on one block
    B, H, N, d = shape
    plan = fa.fa_fwd_plan(B, H, N, d, sms, CAUSAL)
    assert plan["balanced"] == 0 and plan["n_split"] == 1 and plan["scratch_bytes"] == 0
    ur, bn = plan["unit_rows"], plan["kv_tile_rows"]
    n_qt = -(-N // ur)
    assert plan["n_units"] == B * H * n_qt
    seen = {}
    for blk in range(plan["grid"]):
        for (u, t0, t1, kind, peer0, npeer) in fa.fa_fwd_plan_pieces(B, H, N, d, sms, blk, CAUSAL):
            assert kind == 0 and u not in seen
            seen[u] = (t0, t1)
    assert sorted(seen) == list(range(plan["n_units"]))
    for u, (t0, t1) in seen.items():
        qt = n_qt - 1 - u // (B * H)  # longest units first
        assert (t0, t1) == (0, -(-min(N, (qt + 1) * ur) // bn)), (u, qt, t0, t1)


def test_causal_waves_balance_the_load():
    # 256 units of 2..64 K/V tiles on 148 blocks: alternating the direction of
    # each wave keeps every block within 8 tiles of the mean
    B, H, N, d = 1, 8, 8192, 128
    plan = fa.fa_fwd_plan(B, H, N, d, 148, CAUSAL)
    loads = [sum(t1 - t0 for (_, t0, t1, *_r) in fa.fa_fwd_plan_pieces(B, H, N, d, 148, b, CAUSAL))
             for b in range(plan["grid"])]
    assert sum(loads) == B * H * sum(2 * qt + 2 for qt in range(32))
    assert max(loads) - sum(loads) / len(loads) <= 8


def test_unknown_flags_are_rejected():
    with pytest.raises(fa.FAError) as e:
        fa.fa_fwd_plan(1, 1, 64, 64, 148, 2)
    assert e.value.status == fa.FA_ERR_FLAGS


# ------------------------------------------------------------ backward
def test_backward_split_plans():
    # one 384-thread block per SM: the split is taken when it fills the waves
    # clearly better, never for causal batches, and keeps >= 8 query tiles a block
    plan = lambda *a, **k: fa.fa_bwd_plan(*a, **k)  # noqa: E731
    assert plan(4, 8, 4096, 64, 148) == {"n_split": 1, "grid": 1024}    # 99 % of 7 waves
    assert plan(1, 8, 8192, 128, 148) == {"n_split": 2, "grid": 1024}   # 512 blocks: 86 %
    assert plan(1, 1, 25600, 96, 148) == {"n_split": 2, "grid": 400}    # 200 blocks: 68 %
    assert plan(1, 1, 25600, 96, 148, CAUSAL)["n_split"] == 1
    assert plan(1, 2, 2048, 64, 148)["n_split"] == 2                    # 16 query tiles
    assert plan(3, 5, 200, 64, 148)["n_split"] == 1                     # 2 query tiles
    for B, H, N, d in [(1, 1, 1, 64), (2, 3, 5000, 128), (1, 7, 4097, 96), (8, 16, 2048, 64)]:
        p = plan(B, H, N, d, 148)
        n_q = -(-N // (128 if d == 64 else 64))
        assert p["n_split"] == 1 or n_q // p["n_split"] >= 8
        assert p["grid"] == -(-N // 128) * H * B * p["n_split"]
    # d = 256: two blocks per key tile (one per half of d), and the split
    # on top: 100 blocks -> 4 shares of each key tile's query range
    assert plan(1, 1, 6400, 256, 148) == {"n_split": 4, "grid": 400}
    assert plan(1, 1, 6400, 256, 148, CAUSAL) == {"n_split": 1, "grid": 100}
    with pytest.raises(fa.FAError):
        plan(1, 1, 64, 512, 148)
    with pytest.raises(fa.FAError):
        plan(1, 1, 64, 64, 148, 2)
