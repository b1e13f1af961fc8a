"""The attention softmax's FMA-pipe exponential (a share of its 2^x runs on the FMA
pipe instead of the special-function unit), through its diagnostic entry point, against
exp2 in fp64: relative error within 1e-4 over [-125, 0], the range the softmax uses."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_exp2_poly_matches_exp2():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_token_pruning_rmsnorm_b200 import _lib
    lib = _lib.load()
    rng = np.random.default_rng(11)
    x = np.concatenate([-125.0 * rng.random(200001), -rng.random(100000), np.arange(-125, 1, dtype=np.float64),
                        np.arange(-125, 0) + 0.5, [0.0, -0.0, -1e-30, -0.49999997, -0.5, -0.50000006]])
    x = x.astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    y = torch.empty_like(xd)
    _lib.check(lib.tg_selftest_exp2(xd.data_ptr(), y.data_ptr(), x.size, None))
    torch.cuda.synchronize()
    got = y.cpu().numpy().astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() <= 1e-4, (rel.max(), x[np.argmax(rel)])
    # below -125 the input is clamped: a tiny normal number, never more than 2^-124
    xd = torch.tensor([-125.5, -127.0, -200.0, -1e30, float("-inf")], device="cuda")
    y = torch.empty_like(xd)
    _lib.check(lib.tg_selftest_exp2(xd.data_ptr(), y.data_ptr(), 5, None))
    torch.cuda.synchronize()
    assert (y.cpu().numpy() <= 2.0 ** -124).all() and (y.cpu().numpy() > 0).all()
