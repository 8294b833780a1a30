"""GPU parity of the dense projections around the MTLA path (``mtla_linear``,
the tcgen05 GEMM) and of the layer built from them, against the float64
oracle on the same seeded bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import np64, rel_err
from kv_cache_mtla_b200 import mtla

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    torch.cuda.synchronize()
    mtla.get_device_status()
    yield
    assert mtla.get_device_status() == mtla.OK


def _bf16_randn(g, *shape, scale=1.0):
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(300, 200, 520), (1, 64, 64), (4096, 512, 512), (128, 32, 512),
                                   (257, 1000, 8), (16, 288, 512), (1000, 129, 136)])
def test_linear_matches_oracle(M, N, K):
    """y = x W^T: partial row and column tiles (M, N not multiples of the
    128 x 64/128/256 output tiles), K below one 64-column box and not a multiple
    of it, every tile width. The result is bf16 (rounding <= 2^-8 relative), so
    the bound is 8e-3 of max|y|."""
    g = torch.Generator().manual_seed(M * 7 + N * 3 + K)
    x = _bf16_randn(g, M, K)
    w = _bf16_randn(g, N, K, scale=K ** -0.5)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    mtla.linear(x.cuda(), w.cuda(), y)
    ref = oracle.linear(x.float().numpy(), w.float().numpy())
    assert rel_err(np64(y), ref) <= 8e-3
