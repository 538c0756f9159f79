"""The CPU oracle against what the format, libraries and exact arithmetic fix."""
import numpy as np
import pytest

import oracle_pins as P  # noqa: E402


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_tolerance_rule_admits_bf16_rounding_and_rejects_one_ulp_more():
    import oracle
    rng = np.random.default_rng(1)
    y_ref = rng.standard_normal(10000) * 10.0
    s_abs = np.abs(y_ref) * 3.0
    import torch
    y_bf16 = torch.from_numpy(y_ref).to(torch.bfloat16).double().numpy()
    assert oracle.within_tolerance(y_bf16, y_ref, s_abs).all()
    # a relative error of 2^-6 is outside the rule unless s_abs is huge
    bad = y_ref * (1 + 2.0 ** -6)
    assert not oracle.within_tolerance(bad, y_ref, np.abs(y_ref)).any()
