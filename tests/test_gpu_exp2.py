"""The prefill kernel's FMA-pipe exponential (2^t = 2^n p(t - n), a fitted degree-5 p) against
2^t in double precision: relative error within 4e-7 over the range the softmax feeds it, and the
documented clamp below -30."""
import numpy as np
import pytest
import torch

from bit_block_scaled_nvfp4_b200 import api

pytestmark = pytest.mark.gpu


def test_exp2_relative_error_bound():
    g = torch.Generator().manual_seed(11)
    grid = torch.linspace(-30.0, 9.0, 1 << 20)
    rand = torch.rand(1 << 20, generator=g) * 39.0 - 30.0
    special = torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, 8.807354922057604, -29.999, 0.49999997, -0.49999997, 3.5])
    t = torch.cat([grid, rand, special]).float()
    if t.numel() % 2:
        t = t[:-1]
    got = api.selftest_exp2(t.cuda()).cpu().double().numpy()
    want = np.exp2(t.double().numpy())
    rel = np.abs(got / want - 1.0)
    assert rel.max() <= 4e-7, rel.max()


def test_exp2_clamps_below():
    t = torch.tensor([-31.0, -100.0, float("-inf"), -1e30], dtype=torch.float32)
    got = api.selftest_exp2(t.cuda()).cpu().double().numpy()
    assert np.all(np.abs(got / 2.0 ** -30 - 1.0) <= 4e-7)


def test_exp2_rejects_odd_length():
    with pytest.raises(Exception):
        api.selftest_exp2(torch.zeros(3, device="cuda"))
