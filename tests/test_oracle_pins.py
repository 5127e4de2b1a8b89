"""The fp64 oracle against its pins (CPU only)."""
import pytest

import oracle
from oracle_pins import ALL_PINS


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(oracle.default())


def test_oracle_reproduces_closed_form_golden_cases():
    """The worked examples of tests/golden/closed_form_cases.txt (answers derived in closed
    form, see the file) reproduced by the oracle to 1e-12."""
    import os
    import numpy as np
    import mla_workloads as W
    import oracle
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "closed_form_cases.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert len(rows) == 4
    kv = np.zeros((1, 64, 1, W.D_QK), dtype=np.float32)
    kv[0, 0, 0, :512] = 1.0
    kv[0, 1, 0, :512] = 2.0
    kv[0, 1, 0, 512] = 1.0
    kv_bits = W.f32_to_bf16_bits(kv)
    for name, s_q, causal, scale, qi, lse_ref, o_ref in rows:
        s_q, causal, qi = int(s_q), bool(int(causal)), int(qi)
        q = np.zeros((1, s_q, 1, W.D_QK), dtype=np.float32)
        q[..., 512] = 1.0
        o, lse = oracle.mla_decode(W.f32_to_bf16_bits(q), kv_bits, np.zeros((1, 1), np.int32),
                                   np.array([2], np.int32), W.D_V, causal, float(scale))
        assert abs(lse[0, 0, qi] - float(lse_ref)) < 1e-12, name
        assert np.all(np.abs(o[0, qi, 0] - float(o_ref)) < 1e-12), name
