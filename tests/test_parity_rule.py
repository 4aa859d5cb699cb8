"""The comparison rule's unit in the last place, against the number formats themselves
(numpy's float16 spacing; the next bfloat16 by incrementing the bit pattern), on CPU."""
import numpy as np
import torch

from tests.parity import ulp


def test_f16_ulp_equals_numpy_spacing():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.uniform(-60000, 60000, 5000), rng.uniform(-1, 1, 5000), 2.0 ** np.arange(-14, 16)])
    h = np.abs(x.astype(np.float16))
    # normal range, below the largest finite value (whose numpy spacing is inf: the next value overflows)
    h = h[(h >= np.float16(2.0 ** -14)) & (h < np.float16(65504))]
    assert np.array_equal(ulp("f16", h.astype(np.float64)), np.spacing(h).astype(np.float64))
    assert ulp("f16", np.array([1e-6]))[0] == 2.0 ** -24            # subnormal spacing


def test_bf16_ulp_equals_the_step_to_the_next_value():
    rng = np.random.default_rng(4)
    x = torch.from_numpy(np.concatenate([rng.normal(0, 1, 5000), rng.normal(0, 1e30, 2000),
                                         2.0 ** np.arange(-126, 120, 7)])).abs().to(torch.bfloat16)
    bits = x.view(torch.int16)
    nxt = (bits + 1).view(torch.bfloat16)                          # the next representable value up
    step = (nxt.double() - x.double()).numpy()
    assert np.array_equal(ulp("bf16", x.double().numpy()), step)
