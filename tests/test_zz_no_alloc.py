"""sdpa_forward_noalloc, the decode entry point for callers that cannot allocate
device memory when they call attention: a process whose memory manager already
owns the whole GPU (a caching allocator or a serving runtime with a fixed
budget, where a foreign cudaMalloc fails or fragments it), or a decode loop that
must not pay for cudaMalloc / cudaFree, which can synchronise the device.  Its
split-K partials live in a fixed array compiled into the library.

Each case runs on a stream that sdpa_forward has never used, so no split-K
workspace of the library exists for it, and checks two calls in a row against
the float64 oracle.  Across the second call the device's free memory and the
library's workspace bytes must not change.  This file is named to be collected
last, so a run that stops at the first failure has run every other test."""
import numpy as np
import pytest
import torch

import scaled_dot_product_14_b200 as S
from scaled_dot_product_14_b200 import inputs as I

from gpu_util import GpuCase, compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from scaled_dot_product_14_b200 import build
    import oracle
    build.build()
    oracle.build()
    assert torch.cuda.is_available()


def run_noalloc(g: GpuCase, stream) -> int:
    c = g.c
    out_ptr = g.out_buf.data_ptr() + g.pad * g.out_buf.element_size()
    return S.sdpa_forward_noalloc(g.q.data_ptr(), g.k.data_ptr(), g.v.data_ptr(), out_ptr, c.B, c.Hq, c.Hkv,
                                  c.Lq, c.Lk, c.Dqk, c.Dv, c.all_strides16, c.scale, c.mask_kind,
                                  None if g.mask is None else g.mask.data_ptr(),
                                  None if g.mask is None else c.mask_strides, c.dtype, stream.cuda_stream)


@pytest.mark.parametrize("shape", [
    dict(seed=1001, B=1, Hq=32, Hkv=8, Lq=1, Lk=4096, D=256, dtype=I.BF16, mask="decode_additive"),
    dict(seed=1002, B=1, Hq=32, Hkv=4, Lq=1, Lk=4096, D=512, dtype=I.BF16, mask="none"),
    dict(seed=1009, B=2, Hq=16, Hkv=2, Lq=4, Lk=1000, D=128, dtype=I.F16, mask="causal"),
])
def test_noalloc_matches_oracle_on_two_calls_without_allocating(shape):
    c = I.make_case(shape["seed"], shape["B"], shape["Hq"], shape["Hkv"], shape["Lq"], shape["Lk"], shape["D"],
                    dtype=shape["dtype"], mask=shape["mask"])
    stream = torch.cuda.Stream()                 # never used by sdpa_forward
    cases = [GpuCase(c), GpuCase(c)]             # every torch allocation happens before the calls
    torch.cuda.synchronize()
    ws0 = S.sdpa_workspace_bytes()
    assert run_noalloc(cases[0], stream) == 0, S.sdpa_last_cuda_error()
    stream.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert run_noalloc(cases[1], stream) == 0, S.sdpa_last_cuda_error()
    stream.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device free memory changed across a call: {free0} -> {free1}"
    assert S.sdpa_workspace_bytes() == ws0
    rows = None if c.Lk * c.B * c.Hq * c.Lq <= 2 ** 20 else I.sample_rows(shape["seed"], c.B, c.Hq, c.Lq, 16)
    for call, g in enumerate(cases):
        got = g.output()                         # also checks nothing was written outside out
        assert np.isfinite(got).all()
        compare(c, got, rows, label=f"noalloc call {call}")
    assert np.array_equal(cases[0].output(), cases[1].output())


def test_noalloc_rejects_what_it_does_not_cover(monkeypatch):
    stream = torch.cuda.Stream()
    c = I.make_case(1010, 1, 8, 2, 64, 64, 128, dtype=I.BF16)          # prefill shape
    assert run_noalloc(GpuCase(c), stream) == 1                         # SDPA_ERR_INVALID_ARG
    c32 = I.make_case(1011, 1, 8, 2, 1, 64, 128, dtype=I.F32)           # fp32 decode
    assert run_noalloc(GpuCase(c32), stream) == 1
    mla = I.make_case(1013, 1, 4, 1, 1, 300, 40, 32, dtype=I.BF16)     # absorbed-MLA dims: CUDA-core kernels only
    gm = GpuCase(mla)
    assert run_noalloc(gm, stream) == 1
    # With the split count sdpa_forward picks on a 148-SM GPU the partials stay
    # under 4 MiB, so force 4096 splits: 32 rows x 4096 x 257 floats do not fit.
    monkeypatch.setenv("SDPA_DECODE_SPLITS", "4096")
    big = I.make_case(1012, 1, 32, 8, 1, 65536, 256, dtype=I.BF16)
    gb = GpuCase(big)
    assert run_noalloc(gb, stream) == 10                                # SDPA_ERR_TOO_LARGE
    torch.cuda.synchronize()
    assert np.isnan(gb.out_buf.float().cpu().numpy()).all()             # nothing was launched
    assert np.isnan(gm.out_buf.float().cpu().numpy()).all()
