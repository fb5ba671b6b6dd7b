"""Seeded random shapes through the C ABI against the fp64 oracle.

Each case draws T, d, N, Z, K, I, the dtype, the weight layout and the
dispatch mode, so the shape-dependent paths are crossed at many points: the
split-K router (its split count depends on T, E and d), the one-CTA dispatch
layout (T <= 256) against the chunked one, the small-batch route's cluster
forms and the dispatch layout it builds (gather mode, T <= 256), the top-K's
fused count reduce (<= 16 CTAs), tensor-core against CUDA-core GEMMs, the
token-tile configurations, partial feature blocks and ragged segments.  bf16 cases whose shape the tensor-core backward takes also
run the backward pass.
"""
import numpy as np
import pytest

from mixture_experts_layer_30_b200 import binding as B
from tests import test_gpu_backward as TB
from tests import test_gpu_layer as TL

pytestmark = pytest.mark.gpu


def _draw(case):
    rng = np.random.default_rng(1000 + case)
    dtype = "bf16" if case % 3 else "f32"
    T = int(rng.choice([1, 5, 31, 64, 200, 256, 257, 511, 600, 1200]))
    if dtype == "bf16":
        d = int(rng.choice([64, 128, 256, 384, 512, 72, 136]))
        I = int(rng.choice([64, 128, 256, 384, 40]))
    else:
        d = int(rng.choice([16, 64, 100, 128]))
        I = int(rng.choice([8, 32, 64, 96]))
    N = int(rng.choice([1, 3, 8, 16, 40, 130]))
    Z = int(rng.choice([0, 1, 4, 8, 40]))
    E = N + Z
    K = int(rng.integers(1, min(E, 12) + 1))
    tiled = dtype == "bf16" and d % 128 == 0 and I % 128 == 0 and bool(rng.integers(0, 2))
    mode = ["split", "ffn", "gather"][int(rng.integers(0, 3))]
    bias = rng.uniform(-0.05, 0.05, E) if rng.integers(0, 2) else None
    return dict(T=T, d=d, N=N, Z=Z, K=K, I=I, dtype=dtype, tiled=tiled, mode=mode, bias=bias)


@pytest.mark.parametrize("case", range(40))
def test_random_shape_forward(case):
    c = _draw(case)
    shape, L = TL._small(c["T"], c["d"], c["N"], c["Z"], c["K"], c["I"], c["dtype"],
                         seed=2000 + case, bias=c["bias"])
    if c["tiled"]:
        shape.weight_layout = B.WEIGHTS_TILED
    TL._run_and_check(shape, c["dtype"], L, c["N"], c["K"], split_ffn=c["mode"] == "split",
                      fused_gather=c["mode"] == "gather")


def _draw_bwd(case):
    """bf16 shapes the tensor-core backward takes: d, I multiples of 128, E of 8."""
    rng = np.random.default_rng(5000 + case)
    T = int(rng.choice([1, 17, 64, 256, 300, 700]))
    d = int(rng.choice([128, 256, 384, 640]))
    I = int(rng.choice([128, 256, 384]))
    N, Z = [(8, 0), (12, 4), (16, 8), (40, 8), (64, 32), (100, 4)][int(rng.integers(0, 6))]
    K = int(rng.integers(1, min(N + Z, 10) + 1))
    tiled = bool(rng.integers(0, 2))
    bias = rng.uniform(-0.05, 0.05, N + Z) if rng.integers(0, 2) else None
    gamma = float(rng.choice([1.0, 0.7, 2.0]))
    return dict(T=T, d=d, N=N, Z=Z, K=K, I=I, tiled=tiled, bias=bias, gamma=gamma)


@pytest.mark.parametrize("case", range(10))
def test_random_shape_backward(case):
    c = _draw_bwd(case)
    shape, L = TB._small(c["T"], c["d"], c["N"], c["Z"], c["K"], c["I"], "bf16",
                         seed=3000 + case, bias=c["bias"], w_std=0.03)
    if c["tiled"]:
        shape.weight_layout = B.WEIGHTS_TILED
    TB.check_backward(shape, "bf16", L, c["N"], c["K"], gamma=c["gamma"], seed=case)
