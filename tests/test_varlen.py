"""Variable-length batches: B sequences of different lengths packed along one
token axis (the YOLOv12 image page's flash_attn_varlen_* form).  Each
sequence is compared with the fp64 oracle run on that sequence alone, forward
and backward, with and without the causal mask; lengths include 0, 1, tile
edges and ragged tails, and a sequence longer than every other."""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from tests.gpu_helpers import err_stats, grad_ok, o_ok, to64, GRAD_MAX, LSE_MAX, O_MAX, O_MEAN

pytestmark = pytest.mark.gpu

LENGTHS = [129, 1, 400, 0, 1000, 257, 128, 64]


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_attention_144_b200 as fa
    fa.fa_get_device_status(clear=True)
    yield fa
    assert fa.fa_get_device_status() == 0, "a kernel gave up a bounded wait"


def packed(lengths, H, d, dtype, seed):
    total = sum(lengths)
    q, k, v, do = attn_inputs.draw(1, total, H, d, dtype, seed, 4, device="cuda")
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device="cuda")
    return [t[0].contiguous() for t in (q, k, v, do)], cu, total


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,dtype", [(64, "bf16"), (96, "fp16"), (128, "fp16"), (256, "bf16")])
def test_varlen_forward_per_sequence(fa, d, dtype, causal):
    H = 2
    (q, k, v, _), cu, total = packed(LENGTHS, H, d, dtype, 1900 + d)
    scale = 1.0 / math.sqrt(d)
    flags = fa.FA_FLAG_CAUSAL if causal else 0
    o, lse = fa.fa_fwd_varlen(q, k, v, cu, max(LENGTHS), scale=scale, flags=flags)
    torch.cuda.synchronize()
    start = 0
    for n in LENGTHS:
        if n:
            sl = slice(start, start + n)
            o_ref, lse_ref = oracle.attn_fwd(to64(q[sl])[None], to64(k[sl])[None],
                                             to64(v[sl])[None], scale, causal=causal)
            eo = err_stats(to64(o[sl])[None], o_ref)
            el = err_stats(lse[:, sl].cpu().double().numpy()[None], lse_ref)
            assert o_ok(eo), (n, eo)
            assert el["max"] <= LSE_MAX, (n, el)
        start += n


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [64, 96, 128, 256])
def test_varlen_backward_per_sequence(fa, d, causal):
    H = 2
    (q, k, v, do), cu, total = packed(LENGTHS, H, d, "bf16", 2000 + d)
    scale = 1.0 / math.sqrt(d)
    flags = fa.FA_FLAG_CAUSAL if causal else 0
    o, lse = fa.fa_fwd_varlen(q, k, v, cu, max(LENGTHS), scale=scale, flags=flags)
    dq, dk, dv = fa.fa_bwd_varlen(q, k, v, o, do, lse, cu, max(LENGTHS), scale=scale, flags=flags)
    torch.cuda.synchronize()
    start = 0
    for n in LENGTHS:
        if n:
            sl = slice(start, start + n)
            ref = oracle.attn_bwd(to64(q[sl])[None], to64(k[sl])[None], to64(v[sl])[None],
                                  to64(do[sl])[None], scale, causal=causal)
            for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
                s = err_stats(to64(g[sl])[None], r)
                assert grad_ok(s, name), (n, name, s)
        start += n


def test_varlen_many_sequences_and_uncovered_tail(fa):
    # 40 sequences of random lengths; tokens past cu_seqlens[B] belong to no
    # sequence and are left untouched
    rng = np.random.default_rng(7)
    lengths = [int(x) for x in rng.integers(1, 700, size=40)]
    H, d = 3, 64
    (q, k, v, do), cu, total = packed(lengths + [50], H, d, "bf16", 2100)
    cu = cu[:-1].contiguous()  # drop the last sequence: its 50 tokens are uncovered
    o = torch.full_like(q, 5.0)
    lse = torch.full((H, total), 5.0, device="cuda")
    fa.fa_fwd_varlen(q, k, v, cu, max(lengths), o=o, lse=lse)
    dq, dk, dv = (torch.full_like(q, 5.0) for _ in range(3))
    fa.fa_bwd_varlen(q, k, v, o, do, lse, cu, max(lengths), dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    covered = sum(lengths)
    for t in (o, dq, dk, dv):
        assert bool((t[covered:] == 5.0).all())
        assert torch.isfinite(t[:covered].float()).all()
    assert bool((lse[:, covered:] == 5.0).all())
    start = 0
    for n in lengths[:5]:
        sl = slice(start, start + n)
        o_ref, _ = oracle.attn_fwd(to64(q[sl])[None], to64(k[sl])[None], to64(v[sl])[None],
                                   1.0 / 8.0)
        assert err_stats(to64(o[sl])[None], o_ref)["max"] <= O_MAX
        start += n
