"""Packed Q, K, V ([B, N, 3, H, d], the flash_attn_qkvpacked_func layout the
YOLOv12 image page calls): the same kernels read Q, K, V through a token
stride of 3*H*d and write dQ, dK, dV into a packed gradient, so results must
be bitwise those of the unpacked entry points on the three slices."""
import math

import pytest
import torch

import attn_inputs
import oracle
from tests.gpu_helpers import err_stats, grad_ok, to64, GRAD_MAX, O_MAX

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_attention_144_b200 as fa
    return fa


@pytest.mark.parametrize("B,N,H,d,dtype,causal", [
    (2, 300, 3, 64, "bf16", False), (1, 1000, 2, 128, "fp16", False), (1, 257, 2, 256, "bf16", False),
    (2, 513, 2, 64, "bf16", True), (1, 400, 4, 128, "bf16", True), (1, 700, 2, 96, "fp16", False),
    (2, 300, 1, 96, "bf16", True), (1, 2048, 2, 64, "bf16", False)])
def test_packed_equals_unpacked(fa, B, N, H, d, dtype, causal):
    q, k, v, dout = attn_inputs.draw(B, N, H, d, dtype, 1800 + N + d, 4, device="cuda")
    qkv = torch.stack([q, k, v], dim=2).contiguous()  # [B, N, 3, H, d]
    scale = 1.0 / math.sqrt(d)
    flags = fa.FA_FLAG_CAUSAL if causal else 0
    o_p, lse_p = fa.fa_fwd_qkvpacked(qkv, scale=scale, flags=flags)
    o_u, lse_u = fa.fa_fwd_ex(q, k, v, scale=scale, flags=flags)
    torch.cuda.synchronize()
    assert torch.equal(o_p, o_u) and torch.equal(lse_p, lse_u)
    o_ref, _ = oracle.attn_fwd(to64(q), to64(k), to64(v), scale, causal=causal)
    assert err_stats(to64(o_p), o_ref)["max"] <= O_MAX
    guard = torch.full((2 * qkv.numel(),), -7.0, dtype=qkv.dtype, device="cuda")
    dqkv = guard[:qkv.numel()].view(qkv.shape)
    fa.fa_bwd_qkvpacked(qkv, o_p, dout, lse_p, dqkv=dqkv, scale=scale, flags=flags)
    grads = fa.fa_bwd_ex(q, k, v, o_u, dout, lse_u, scale=scale, flags=flags)
    torch.cuda.synchronize()
    assert bool((guard[qkv.numel():] == -7.0).all()), "write past the end of dqkv"
    # dK, dV are owned by one block each: bitwise equal; dQ is reduced across
    # key tiles in no fixed order, so only equal to rounding
    assert torch.equal(dqkv[:, :, 1], grads[1]) and torch.equal(dqkv[:, :, 2], grads[2])
    assert (dqkv[:, :, 0].float() - grads[0].float()).abs().max().item() <= 1e-2
    ref = oracle.attn_bwd(to64(q), to64(k), to64(v), to64(dout), scale, causal=causal)
    for i, r in enumerate(ref):
        assert grad_ok(err_stats(to64(dqkv[:, :, i]), r))
