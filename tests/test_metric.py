"""The parity metric's bf16 storage allowance is exactly the RNE rounding bound."""
import numpy as np
import torch

from kda_testlib import bf16_half_ulp, rel_err


def test_half_ulp_values():
    np.testing.assert_array_equal(bf16_half_ulp([1.0, 1.5, -1.99, 0.75, 4.0]),
                                  [2.0 ** -8, 2.0 ** -8, 2.0 ** -8, 2.0 ** -9, 2.0 ** -6])


def test_rounding_never_exceeds_allowance():
    # fp32 values rounded once to bf16, as the kernels store their outputs
    x = (torch.randn(200000) * torch.exp(torch.randn(200000) * 3)).to(torch.float64)
    r = x.to(torch.float32).to(torch.bfloat16).to(torch.float64)
    d = (r - x).abs().numpy()
    assert np.all(d <= bf16_half_ulp(r.numpy()))
    assert rel_err(r.numpy(), x.numpy(), stored_as="bf16") == 0.0
    assert rel_err(r.numpy(), x.numpy()) > 0.0


def test_allowance_does_not_hide_real_errors():
    x = np.linspace(-3, 3, 1001)
    r = torch.tensor(x).to(torch.bfloat16).to(torch.float64).numpy()
    r[500] += 0.1                      # a computation error well above one ulp
    assert rel_err(r, x, stored_as="bf16") > 0.05


def test_two_stored_roundings_of_one_value_compare_equal():
    """Two outputs each rounded once to bf16 from nearby exact values may sit
    one ulp apart; with both storages allowed they compare as equal."""
    x = np.array([1.0 + 2.0 ** -8, 3.0 + 2.0 ** -7, -0.75 - 2.0 ** -10])
    eps = 1e-6
    to_bf16 = lambda t: torch.tensor(t, dtype=torch.float32).to(torch.bfloat16).double().numpy()
    a, b = to_bf16(x + eps * np.abs(x)), to_bf16(x - eps * np.abs(x))
    assert np.any(a != b)
    assert rel_err(a, b, stored_as="bf16", both_stored=True) == 0.0
    assert rel_err(a, b, stored_as="bf16") > 0.0
