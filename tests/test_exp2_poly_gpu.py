"""The softmax's software base-2 exponential (FMA-pipe polynomial) against float64 2^x."""

import numpy as np
import pytest
import torch

import attention_tiled_attn_b200 as attn
from attention_tiled_attn_b200 import build as attn_build

pytestmark = pytest.mark.gpu

BOUND = 1.02e-4 + 4e-7  # fitted polynomial bound + float32 evaluation rounding


def test_exp2_poly_relative_error():
    attn_build.build()
    x = np.concatenate([np.linspace(-125.999, 8.0, 2_000_001), np.arange(-125, 9, dtype=np.float64),
                        np.arange(-125, 9) + 0.5, [-0.5, 0.5, 1e-8, -1e-8]]).astype(np.float32)
    y = attn.exp2_poly_eval(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= BOUND, rel.max()
    assert np.all(np.isfinite(y)) and np.all(y > 0)


def test_exp2_poly_flushes_below_minus_126():
    """2^-126 is the smallest normal float; below it (a masked -inf logit included)
    the result is exactly 0, so a row that sees no key sums to 0."""
    x = np.array([-126.0, -126.5, -200.0, -1e30, -np.inf], dtype=np.float32)
    y = attn.exp2_poly_eval(torch.from_numpy(x).cuda()).cpu().numpy()
    assert y[0] == np.float32(2.0 ** -126)
    assert np.all(y[1:] == 0.0)


def test_exp2_poly_odd_length():
    x = torch.tensor([0.0, 1.0, -1.0], device="cuda")
    y = attn.exp2_poly_eval(x).cpu().numpy()
    assert np.allclose(y, [1.0, 2.0, 0.5], rtol=BOUND)
