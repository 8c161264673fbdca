"""The test helpers themselves: the bf16 rounding that the output comparison
accepts, pinned against torch's conversion and against hand-worked ties."""
import numpy as np
import torch

from tests._util import assert_close_out, round_bf16


def test_round_bf16_matches_torch_on_fp32_values():
    # fp32 inputs: torch's fp32 -> bf16 conversion rounds once, to nearest even
    g = torch.Generator().manual_seed(0)
    x = torch.randn(200000, generator=g) * torch.exp2(torch.randint(-20, 20, (200000,),
                                                                    generator=g).float())
    want = x.to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(round_bf16(x.double().numpy()), want)


def test_round_bf16_ties_go_to_even():
    u = 2.0 ** -7  # bf16 spacing in [1, 2)
    cases = {1 + u / 2: 1.0,            # tie between 1 and 1 + u: the even one is 1
             1 + 3 * u / 2: 1 + 2 * u,  # tie between 1 + u and 1 + 2u
             -(1 + u / 2): -1.0,
             2.375 - u: 2.375,          # spacing 2u above 2: the tie goes to 2 + 24 * 2u
             4.0625: 4.0625, 0.0: 0.0}
    for x, want in cases.items():
        assert round_bf16(np.float64(x)) == want, x


def test_close_out_accepts_only_the_correctly_rounded_value_beyond_tolerance():
    want = np.array([4.05, 1.0])
    ok = np.array([round_bf16(4.05), 1.005])  # 4.0625 is 0.0125 away, but correctly rounded
    assert_close_out(ok, want, 1e-2)
    bad = np.array([4.03125, 1.0])            # the other neighbour of 4.05: rejected
    try:
        assert_close_out(bad, want, 1e-2)
    except AssertionError:
        pass
    else:
        raise AssertionError("a wrongly rounded element was accepted")
    try:
        assert_close_out(np.array([4.0625, 1.02]), want, 1e-2)
    except AssertionError:
        pass
    else:
        raise AssertionError("an element beyond the tolerance was accepted")
