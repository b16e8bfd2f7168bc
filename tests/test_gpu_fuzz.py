"""Seeded random shapes through the BF16 and E4M3 forwards, every token against the oracle.

Shapes are drawn from the supported set (d a multiple of 256, I a multiple of 128, E a
multiple of 4 and of the group count, up to 32 groups, top_k <= 8 and <= topk_group * E /
n_group), with and without weight normalisation, so that group sizes, lane runs of the
selection and ragged m-tiles combine in ways the hand-picked cases do not.
"""
import dataclasses

import numpy as np
import pytest
import torch

from sparse_moe_transformer_fp32_b200 import workloads as W
from tests import gpu_helpers as H
from tests.test_gpu_parity import _check_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    from sparse_moe_transformer_fp32_b200 import beam_moe as bm
    from sparse_moe_transformer_fp32_b200 import build
    build.build()
    bm.lib()
    yield
    torch.cuda.empty_cache()


def _shape(i: int) -> dict:
    rng = np.random.default_rng(1000 + i)
    while True:
        G = int(rng.choice([1, 2, 3, 4, 5, 8, 16, 32]))
        per = int(rng.integers(1, 9))
        E = G * per
        if E % 4 or E > 256:
            continue
        Gk = int(rng.integers(1, G + 1))
        k = int(rng.integers(1, min(8, Gk * per) + 1))
        return dict(T=int(rng.integers(1, 301)), d=int(rng.choice([256, 512, 768])), E=E,
                    n_group=G, topk_group=Gk, top_k=k, I=int(rng.choice([128, 256, 384])),
                    norm_topk_prob=i % 4 != 3, seed=100 + i)


@pytest.mark.parametrize("i", range(20))
def test_random_shape_bf16_and_e4m3(i):
    wl = dataclasses.replace(W.WORKLOADS["tiny"], name=f"fuzz{i}", **_shape(i))
    case = H.make_case(wl)
    weights = H.device_weights(wl)
    out, idx, w, _ = H.run_forward(case, weights)
    _check_routing(case, idx, w)
    ref = H.oracle_out(case, weights, range(wl.T), batch=64)
    H.assert_close_out(out.float().cpu().numpy(), ref, f"{wl.name} bf16 {_shape(i)}")
    fp8 = H.device_weights_fp8(weights)
    out8, idx8, w8, _ = H.run_forward_fp8(case, fp8)
    _check_routing(case, idx8, w8)
    ref8 = H.oracle_out_fp8(case, weights, range(wl.T), fp8, batch=64)
    H.assert_close_out(out8.float().cpu().numpy(), ref8, f"{wl.name} e4m3 {_shape(i)}")
