"""The fp64 exponential of the block discovery (Tang's table-driven method,
for arguments <= 0) against CUDA's own exp on the same device and against
Python's math.exp: relative error <= 1e-14 on [-700, 0]; e^0 = 1 exactly;
-inf and arguments below -700 give 0."""
import math

import numpy as np
import pytest
import torch

import sparse_attention_long_head_b200 as vs

pytestmark = pytest.mark.gpu


def _run(x: np.ndarray) -> np.ndarray:
    xd = torch.from_numpy(x).cuda()
    y = torch.empty_like(xd)
    vs.vs_selftest_exp(xd, y)
    torch.cuda.synchronize()
    return y.cpu().numpy()


def test_relative_error_against_library_exp(cuda_device):
    rng = np.random.default_rng(5)
    x = np.concatenate([-rng.exponential(3.0, 200000), -rng.uniform(0, 700, 200000),
                        -np.linspace(0, 1e-3, 5001), -np.arange(0, 700) * math.log(2) / 32 * 23])
    x = x[x >= -700.0]
    y = _run(x)
    ref_dev = torch.exp(torch.from_numpy(x).cuda()).cpu().numpy()
    rel = np.abs(y - ref_dev) / ref_dev
    assert rel.max() <= 1e-14, rel.max()
    idx = rng.choice(x.size, 2000, replace=False)
    ref_host = np.array([math.exp(v) for v in x[idx]])
    assert (np.abs(y[idx] - ref_host) / ref_host).max() <= 1e-14


def test_special_arguments(cuda_device):
    x = np.array([0.0, -0.0, -np.inf, -700.0, -700.0000001, -745.0, -1e300])
    y = _run(x)
    assert y[0] == 1.0 and y[1] == 1.0
    assert y[2] == 0.0 and y[4] == 0.0 and y[5] == 0.0 and y[6] == 0.0
    assert abs(y[3] - math.exp(-700.0)) <= 1e-14 * math.exp(-700.0)
