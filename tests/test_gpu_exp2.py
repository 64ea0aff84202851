"""The FMA-pipe exponential of the attention softmax (exp2_poly2, reached through the
fpx_diag_exp2 diagnostic) against 2^x in fp64: relative error <= 7.5e-5, the bound its Remez fit
(csrc/exp2_poly_fit.py) reports, on a dense grid over the softmax's range, including integers,
half-integers (the rounding boundary of the range reduction) and the lower clamp."""
import numpy as np
import pytest
import torch

import dynamic_block_sparse_pooled_b200 as fpx

pytestmark = pytest.mark.gpu


def run(x: np.ndarray) -> np.ndarray:
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    yd = torch.empty_like(xd)
    rc = fpx.load().fpx_diag_exp2(xd.data_ptr(), yd.data_ptr(), xd.numel(),
                                  torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    return yd.cpu().numpy().astype(np.float64)


def test_exp2_poly_relative_error_over_the_softmax_range():
    grid = np.linspace(-125.0, 8.0, 4_000_001, dtype=np.float64)
    special = np.concatenate([np.arange(-125, 9), np.arange(-125, 8) + 0.5,
                              np.arange(-125, 8) + 0.5 - 2.0 ** -20,
                              np.arange(-125, 8) + 0.5 + 2.0 ** -20])
    x = np.concatenate([grid, special]).astype(np.float32)
    y = run(x)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(y - want) / want
    assert rel.max() <= 7.5e-5, (rel.max(), x[np.argmax(rel)])
    # odd length: the last, unpaired element goes through the same code
    assert np.abs(run(x[:7]) / np.exp2(x[:7].astype(np.float64)) - 1).max() <= 7.5e-5


def test_exp2_poly_clamps_below_the_range():
    x = np.array([-125.0, -125.5, -126.0, -140.0, -1e4, -np.inf], np.float32)
    y = run(x)
    assert np.all(y > 0) and np.all(np.isfinite(y))
    assert np.all(y <= 2.0 ** -125 * 1.0001)  # a vanishing weight, never a larger value


def test_exp2_diag_argument_checks():
    lib = fpx.load()
    assert lib.fpx_diag_exp2(None, None, 0, None) == 0
    assert lib.fpx_diag_exp2(None, None, 4, None) == -1
    assert lib.fpx_diag_exp2(None, None, -1, None) == -1
