"""fa_bwd_noalloc: the backward pass for callers that cannot allocate.

Some hosts (plugin runtimes with their own static memory plan, code running
where allocation is forbidden or unsafe) must not call the device allocator.
fa_bwd_noalloc runs the same backward kernels as fa_bwd but takes its scratch
from a fixed buffer compiled into the library.  These tests call it through
the C ABI and check it against fa_bwd, on two calls in a row (the buffer keeps
the previous call's contents, so the second call shows the reset works).

This file is collected last on purpose; it also passes when run on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import attn_inputs
from tests.gpu_helpers import GRAD_MAX

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_attention_144_b200 as fa
    return fa


def _call_noalloc(lib, q, k, v, o, dout, lse, dq, dk, dv, scale):
    B, N, H, d = q.shape
    stream = torch.cuda.current_stream().cuda_stream
    return lib.fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                              dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                              dv.data_ptr(), B, H, N, d, ctypes.c_float(scale), stream)


@pytest.mark.parametrize("B,N,H", [(2, 1000, 4), (1, 129, 3)])
def test_matches_fa_bwd_on_two_calls_in_a_row(fa, B, N, H):
    d = 64
    scale = float(np.float32(1.0 / np.sqrt(d)))
    q, k, v, dout = attn_inputs.draw(B, N, H, d, "bf16", 900 + N, 4, device="cuda")
    o, lse = fa.fa_fwd(q, k, v, scale=scale)
    want = fa.fa_bwd(q, k, v, o, dout, lse, scale=scale)
    lib = fa.lib()
    for _ in range(2):
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        rc = _call_noalloc(lib, q, k, v, o, dout, lse, *got, scale)
        assert rc == fa.FA_OK, fa.fa_status_string(rc)
        torch.cuda.synchronize()
        for g, w in zip(got, want):
            assert torch.isfinite(g.float()).all()
            assert (g.float() - w.float()).abs().max().item() <= GRAD_MAX
    assert fa.fa_get_device_status() == 0


def test_rejects_problems_larger_than_its_buffer(fa):
    # 64 heads x 8192 tokens need 64 * 8192 * (4 * 64 + 8) bytes = 132 MiB of
    # scratch, more than the 64 MiB buffer: refused before any launch.
    B, N, H, d = 1, 8192, 64, 64
    t = [torch.zeros((B, N, H, d), dtype=torch.bfloat16, device="cuda") for _ in range(8)]
    lse = torch.zeros((B, H, N), dtype=torch.float32, device="cuda")
    q, k, v, o, dout, dq, dk, dv = t
    rc = _call_noalloc(fa.lib(), q, k, v, o, dout, lse, dq, dk, dv, 0.125)
    assert rc == fa.FA_ERR_SCRATCH
    assert "64 MiB" in fa.fa_status_string(rc)
    torch.cuda.synchronize()
    assert bool((dq == 0).all()) and bool((dk == 0).all())
