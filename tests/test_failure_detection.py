"""Failure detection without a GPU fault.

A device-side wait on a barrier that nothing completes gives up after its
limit, records a status the host can read, and returns; the context stays
usable and a normal call afterwards still matches the oracle.
"""
import math

import numpy as np
import pytest
import torch

import attn_inputs
import oracle
from tests.gpu_helpers import O_MAX, err_stats, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_attention_144_b200 as fa
    return fa


def test_bounded_wait_gives_up_and_reports(fa):
    status = fa.fa_selftest_bounded_wait(20000)  # 20 ms limit
    assert status & 0xFF == 0x5A          # the timeout code
    assert (status >> 8) & 0xFF == 0x7F   # the self-test's wait site
    assert fa.fa_get_device_status() == 0  # the self-test clears the word again


def test_device_usable_after_a_timeout(fa):
    fa.fa_selftest_bounded_wait(5000)
    q, k, v = attn_inputs.draw(1, 130, 2, 64, "bf16", 801, 3, device="cuda")
    o, lse = fa.forward(q, k, v, scale=0.125)
    torch.cuda.synchronize()
    o_ref, _ = oracle.attn_fwd(to64(q), to64(k), to64(v), 0.125)
    assert err_stats(to64(o), o_ref)["max"] <= O_MAX
    assert fa.fa_get_device_status() == 0


def test_errors_leave_outputs_untouched(fa):
    q, k, v = attn_inputs.draw(1, 64, 1, 64, "bf16", 802, 3, device="cuda")
    o = torch.full_like(q, 7.0)
    lse = torch.full((1, 1, 64), 3.0, device="cuda")
    lib = fa.lib()
    import ctypes
    rc = lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                    1, 1, 64, 80, ctypes.c_float(0.1), None)
    assert rc == fa.FA_ERR_HEADDIM
    rc = lib.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr() + 2, lse.data_ptr(),
                    1, 1, 64, 64, ctypes.c_float(0.1), None)
    assert rc == fa.FA_ERR_ALIGN
    torch.cuda.synchronize()
    assert bool((o == 7.0).all()) and bool((lse == 3.0).all())
    with pytest.raises(TypeError):
        fa.fa_fwd(q.half(), k.half(), v.half())
