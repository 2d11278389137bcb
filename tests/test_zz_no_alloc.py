"""fa_bwd_noalloc: the backward pass for callers that cannot allocate.

Some hosts must not call the device allocator at all: plugin runtimes that
hand every kernel a fixed memory plan made ahead of time, code that runs
while allocation is forbidden or unsafe (inside another runtime's critical
section, or where an allocation could trigger a synchronisation the caller
cannot afford).  fa_bwd_noalloc runs the same backward kernels as fa_bwd but
takes its scratch from a fixed buffer compiled into the library.

These tests call it through the C ABI, twice in a row (the buffer keeps the
previous call's contents, so the second call shows that every call clears
what must start at zero), and check that
  * its gradients match the fp64 oracle within the gradient bars;
  * dK and dV are bitwise those of fa_bwd wherever fa_bwd takes one block
    per key tile (both paths then run the same kernel on the same inputs,
    and dK, dV are written by one block each); dQ is reduced across key
    tiles in no fixed order, so it is compared within the bars;
  * the call requests no scratch from the library's memory pool (its
    allocation counter does not move) and maps no device memory (the
    device's free memory is unchanged across a warm call).

This file is collected last on purpose; it also passes when run on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from tests.gpu_helpers import err_stats, grad_ok, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_attention_144_b200 as fa
    oracle.build()
    return fa


def _call_noalloc(lib, q, k, v, o, dout, lse, dq, dk, dv, scale):
    B, N, H, d = q.shape
    stream = torch.cuda.current_stream().cuda_stream
    return lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), B, H, N, d, ctypes.c_float(scale), stream)


@pytest.mark.parametrize("B,N,H", [(2, 1000, 4), (1, 129, 3)])
def test_matches_oracle_and_fa_bwd_on_two_calls_in_a_row(fa, B, N, H):
    d = 64
    scale = float(np.float32(1.0 / np.sqrt(d)))
    q, k, v, dout = attn_inputs.draw(B, N, H, d, "bf16", 900 + N, 4, device="cuda")
    o, lse = fa.fa_fwd(q, k, v, scale=scale)
    want = fa.fa_bwd(q, k, v, o, dout, lse, scale=scale)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    one_block_per_key_tile = fa.fa_bwd_plan(B, H, N, d, sms)["n_split"] == 1
    ref = oracle.attn_bwd(to64(q), to64(k), to64(v), to64(dout), scale)
    lib = fa.lib()
    for _ in range(2):
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        rc = _call_noalloc(lib, q, k, v, o, dout, lse, *got, scale)
        assert rc == fa.FA_OK, fa.fa_status_string(rc)
        torch.cuda.synchronize()
        for name, g, w, r in zip(("dq", "dk", "dv"), got, want, ref):
            assert torch.isfinite(g.float()).all(), name
            s = err_stats(to64(g), r)
            assert grad_ok(s, name), (name, s)
            if name != "dq" and one_block_per_key_tile:
                assert torch.equal(g, w), name
            else:
                assert grad_ok(err_stats(to64(g), to64(w)), name + " vs fa_bwd")
    assert fa.fa_get_device_status() == 0


def test_allocates_nothing(fa):
    B, N, H, d = 2, 777, 3, 64
    scale = 0.125
    q, k, v, dout = attn_inputs.draw(B, N, H, d, "bf16", 1777, 4, device="cuda")
    o, lse = fa.fa_fwd(q, k, v, scale=scale)
    got = [torch.empty_like(q) for _ in range(3)]
    lib = fa.lib()
    # a warm call first: the first call in a context may load the library's
    # device code (which holds the fixed buffer) and look up its address
    assert _call_noalloc(lib, q, k, v, o, dout, lse, *got, scale) == fa.FA_OK
    torch.cuda.synchronize()
    allocs0 = fa.fa_scratch_allocs()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(2):
        assert _call_noalloc(lib, q, k, v, o, dout, lse, *got, scale) == fa.FA_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert fa.fa_scratch_allocs() == allocs0
    assert free1 == free0
    # the counter does see the allocating path
    fa.fa_bwd(q, k, v, o, dout, lse, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_scratch_allocs() == allocs0 + 1


def test_rejects_problems_larger_than_its_buffer(fa):
    # 64 heads x 8192 tokens need 64 * 8192 * (4 * 64 + 8) bytes = 132 MiB of
    # scratch, more than the 64 MiB buffer: refused before any launch.
    B, N, H, d = 1, 8192, 64, 64
    t = [torch.zeros((B, N, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(8)]
    lse = torch.zeros((B, H, N), dtype=torch.float32, device="cuda")
    q, k, v, o, dout, dq, dk, dv = t
    launches = fa.fa_kernel_launches()
    rc = _call_noalloc(fa.lib(), q, k, v, o, dout, lse, dq, dk, dv, 0.125)
    assert rc == fa.FA_ERR_SCRATCH
    assert "64 MiB" in fa.fa_status_string(rc)
    assert fa.fa_kernel_launches() == launches
    torch.cuda.synchronize()
    assert bool((dq == 0).all()) and bool((dk == 0).all())
