"""Targeted checks of the tcgen05 prefill kernel: small problems (one CTA, a
few tiles, ragged tails) for every head dim, each compared with the oracle;
SDPA_DEBUG=1 makes every call synchronise and report a timed-out in-kernel
wait as SDPA_ERR_TIMEOUT, and the counters must show the tcgen05 kernel ran."""
import numpy as np
import pytest
import torch

import scaled_dot_product_14_b200 as S
from scaled_dot_product_14_b200 import inputs as I

from gpu_util import run_and_check

pytestmark = pytest.mark.gpu

DIMS = [(64, 64), (72, 72), (80, 80), (96, 96), (128, 128), (192, 128), (256, 256), (512, 512)]


@pytest.fixture(scope="module", autouse=True)
def built():
    from scaled_dot_product_14_b200 import build
    import oracle
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


@pytest.fixture(autouse=True)
def debug_sync(monkeypatch):
    monkeypatch.setenv("SDPA_DEBUG", "1")


def tc_launches():
    return S.sdpa_get_counters()["prefill_tcgen05_launches"]


@pytest.mark.parametrize("D,Dv", DIMS)
def test_single_cta(D, Dv):
    c = I.make_case(2000 + D, 1, 1, 1, 128, 128, D, Dv, dtype=I.BF16)
    n0 = tc_launches()
    run_and_check(c, label=f"one CTA D={D}")
    assert tc_launches() == n0 + 1


@pytest.mark.parametrize("D,Dv", DIMS)
@pytest.mark.parametrize("L", [9, 200, 384, 1000])
@pytest.mark.parametrize("mask", ["none", "causal"])
def test_few_tiles(D, Dv, L, mask):
    c = I.make_case(2100 + D + L, 1, 4, 2, L, L, D, Dv, dtype=I.BF16, mask=mask)
    run_and_check(c, label=f"D={D} L={L} {mask}")


@pytest.mark.parametrize("D,Dv", [(64, 64), (128, 128), (512, 512)])
@pytest.mark.parametrize("mask", ["additive", "bool"])
def test_masks_fp16(D, Dv, mask):
    c = I.make_case(2200 + D, 2, 4, 1, 300, 257, D, Dv, dtype=I.F16, mask=mask)
    run_and_check(c, label=f"fp16 D={D} {mask}")


def test_no_device_error_left():
    st, code = S.sdpa_check_device_error(torch.cuda.current_stream().cuda_stream)
    assert st == 0 and code == 0
