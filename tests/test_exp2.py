"""The FMA-pipe base-2 exponential that the forward softmax uses for part of
each row's columns (the rest go through the hardware ex2).

It is range reduction plus a degree-3 polynomial written for this library;
these tests hold it to its stated error bound against the exact 2^x (fp64)
and against CUDA's own exp2 on the same inputs.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_attention_144_b200 as fa
    return fa


def test_relative_error_bound(fa):
    # every softmax argument range: x = s*c - m <= 8 (rescale threshold), and far below 0
    x = torch.cat([torch.linspace(-125.0, 127.0, 2_000_001),
                   torch.linspace(-1.0, 1.0, 100_001),
                   torch.tensor([0.0, -0.5, 0.5, -1.5, 1.5, -124.5, 8.0])]).cuda()
    y = fa.fa_selftest_exp2(x).double().cpu().numpy()
    ref = np.exp2(x.double().cpu().numpy())
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 1e-4, rel.max()
    # against CUDA's own exp2 on the same float inputs
    cuda = torch.exp2(x).double().cpu().numpy()
    assert np.abs(y / cuda - 1.0).max() <= 1e-4


def test_exact_at_integers(fa):
    # f = 0 at integers: the result is the polynomial's constant term times 2^n
    n = torch.arange(-120, 120, dtype=torch.float32).cuda()
    y = fa.fa_selftest_exp2(n).double().cpu().numpy()
    assert np.abs(y / np.exp2(n.double().cpu().numpy()) - 1.0).max() <= 1e-4


def test_very_negative_inputs_stay_tiny_and_finite(fa):
    x = torch.tensor([-125.5, -126.0, -127.0, -150.0, -1e4, -3.0e38, float("-inf")]).cuda()
    y = fa.fa_selftest_exp2(x).cpu().numpy()
    assert np.all(np.isfinite(y)) and np.all(y > 0.0) and np.all(y <= 2.0 ** -124)


def test_odd_count_and_errors(fa):
    x = torch.tensor([1.0, 2.0, 3.0]).cuda()
    y = fa.fa_selftest_exp2(x).cpu().numpy()
    assert np.allclose(y, [2.0, 4.0, 8.0], rtol=1e-4)
    with pytest.raises(TypeError):
        fa.fa_selftest_exp2(x.double())
