"""sdpa_forward_noalloc, the entry point for callers that cannot allocate device
memory at call time (a memory manager that owns the whole GPU, or a decode
loop that must not pay for cudaMalloc / cudaFree).  Its split-K partials live in
a fixed array compiled into the library.  This file is named to be collected
last, so a run that stops at the first failure has run every other test."""
import numpy as np
import pytest
import torch

import scaled_dot_product_14_b200 as S
from scaled_dot_product_14_b200 import inputs as I

from gpu_util import GpuCase, TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from scaled_dot_product_14_b200 import build
    build.build()
    assert torch.cuda.is_available()


def run_noalloc(g: GpuCase) -> int:
    c = g.c
    out_ptr = g.out_buf.data_ptr() + g.pad * g.out_buf.element_size()
    return S.sdpa_forward_noalloc(g.q.data_ptr(), g.k.data_ptr(), g.v.data_ptr(), out_ptr, c.B, c.Hq, c.Hkv,
                                  c.Lq, c.Lk, c.Dqk, c.Dv, c.all_strides16, c.scale, c.mask_kind,
                                  None if g.mask is None else g.mask.data_ptr(),
                                  None if g.mask is None else c.mask_strides, c.dtype,
                                  torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("shape", [
    dict(seed=1001, B=1, Hq=32, Hkv=8, Lq=1, Lk=4096, D=256, dtype=I.BF16, mask="decode_additive"),
    dict(seed=1002, B=1, Hq=32, Hkv=4, Lq=1, Lk=4096, D=512, dtype=I.BF16, mask="none"),
    dict(seed=1009, B=2, Hq=16, Hkv=2, Lq=4, Lk=1000, D=128, dtype=I.F16, mask="causal"),
])
def test_noalloc_matches_sdpa_forward_on_two_calls(shape):
    c = I.make_case(shape["seed"], shape["B"], shape["Hq"], shape["Hkv"], shape["Lq"], shape["Lk"], shape["D"],
                    dtype=shape["dtype"], mask=shape["mask"])
    ref_case = GpuCase(c)
    assert ref_case.run() == 0
    ref = ref_case.output()
    tmax, tmean = TOL[c.dtype]
    for call in range(2):
        g = GpuCase(c)
        st = run_noalloc(g)
        assert st == 0, S.sdpa_error_string(st)
        got = g.output()                      # also checks nothing was written outside out
        assert np.isfinite(got).all()
        err = np.abs(got - ref)
        assert err.max() <= tmax and err.mean() <= tmean, (call, err.max(), err.mean())


def test_noalloc_rejects_what_it_does_not_cover(monkeypatch):
    c = I.make_case(1010, 1, 8, 2, 64, 64, 128, dtype=I.BF16)          # prefill shape
    g = GpuCase(c)
    assert run_noalloc(g) == 1                                          # SDPA_ERR_INVALID_ARG
    c32 = I.make_case(1011, 1, 8, 2, 1, 64, 128, dtype=I.F32)           # fp32 decode
    assert run_noalloc(GpuCase(c32)) == 1
    # With the split count sdpa_forward picks on a 148-SM GPU the partials stay
    # under 4 MiB, so force 4096 splits: 32 rows x 4096 x 257 floats do not fit.
    monkeypatch.setenv("SDPA_DECODE_SPLITS", "4096")
    big = I.make_case(1012, 1, 32, 8, 1, 65536, 256, dtype=I.BF16)
    gb = GpuCase(big)
    assert run_noalloc(gb) == 10                                        # SDPA_ERR_TOO_LARGE
    torch.cuda.synchronize()
    assert np.isnan(gb.out_buf.float().cpu().numpy()).all()             # nothing was launched
