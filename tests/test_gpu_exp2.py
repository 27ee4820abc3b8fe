"""The FMA-pipe 2^x polynomial used for part of the forward's exponentials,
held to its error bound against float64 over the argument range the softmax
produces (x <= 8 after the lazy running-max shift)."""

import numpy as np
import pytest
import torch

from exact_attention_121_b200 import _lib

pytestmark = pytest.mark.gpu

# degree-4 fit (exp2_poly_fit.py): 2.9e-6 in float32 Horner form; the
# argument split x = n + f is exact, the exponent add is exact
REL_BOUND = 3.5e-6


def _run(x):
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    yd = torch.empty_like(xd)
    code = _lib.load().fa_selftest_exp2_poly(xd.data_ptr(), yd.data_ptr(), xd.numel(),
                                              torch.cuda.current_stream().cuda_stream)
    assert code == 0
    torch.cuda.synchronize()
    return yd.cpu().numpy().astype(np.float64)


def test_exp2_poly_within_bound():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-125.0, 8.0, 200_001), rng.uniform(-2.0, 2.0, 100_000),
                        np.arange(-125, 9, dtype=np.float64), np.arange(-125, 8) + 0.5,
                        np.array([0.0, -0.0, 1e-7, -1e-7, 0.49999997, -0.49999997, 7.9999995])])
    x = x.astype(np.float32).astype(np.float64)
    y = _run(x)
    rel = np.abs(y / np.exp2(x) - 1.0)
    assert rel.max() <= REL_BOUND, (rel.max(), x[rel.argmax()])
    # integers are exact powers of two (p(0) = 1)
    ints = np.arange(-125, 9, dtype=np.float64)
    np.testing.assert_array_equal(_run(ints), np.exp2(ints))


def test_exp2_poly_clamps_small_arguments():
    y = _run(np.array([-126.0, -200.0, -1e30, -np.inf]))
    np.testing.assert_allclose(y, np.exp2(-125.0), rtol=REL_BOUND)
