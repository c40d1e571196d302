"""Helpers for the GPU parity tests: run a seeded case through the C ABI and
compare with the float64 oracle on the same stored inputs.

Tolerances: fp32 max-abs <= 1e-5; fp16 / bf16 max-abs <= 2e-2 and mean-abs
<= 2e-3, with the inputs already rounded to the dtype before the oracle sees
them (the oracle widens the very same stored values)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import scaled_dot_product_14_b200 as S
from scaled_dot_product_14_b200 import inputs as I

TOL = {I.F32: (1e-5, 1e-5), I.F16: (2e-2, 2e-3), I.BF16: (2e-2, 2e-3)}
TORCH_DT = {I.F32: torch.float32, I.F16: torch.float16, I.BF16: torch.bfloat16}


def to_device(storage: np.ndarray, dtype: int) -> torch.Tensor:
    """Flat storage array -> 1-D CUDA tensor of the dtype (bit-exact)."""
    if dtype == I.F32:
        t = torch.from_numpy(np.ascontiguousarray(storage, dtype=np.float32))
    else:
        t = torch.from_numpy(np.ascontiguousarray(storage).view(np.int16)).view(TORCH_DT[dtype])
    return t.cuda()


def out_extent(c: I.Case) -> int:
    so = c.out_strides
    return (c.B - 1) * so[0] + (c.Hq - 1) * so[1] + (c.Lq - 1) * so[2] + (c.Dv - 1) * so[3] + 1 if c.B and c.Hq and c.Lq else 1


class GpuCase:
    """Device copies of a case, a NaN-prefilled output buffer, and a runner."""

    def __init__(self, c: I.Case, out_pad: int = 64):
        self.c = c
        self.q = to_device(c.q, c.dtype)
        self.k = to_device(c.k, c.dtype)
        self.v = to_device(c.v, c.dtype)
        self.mask = None
        if c.mask is not None:
            self.mask = (torch.from_numpy(c.mask).cuda() if c.mask_kind == I.MASK_BOOL
                         else to_device(c.mask, c.dtype))
        self.pad = out_pad
        n = out_extent(c) + 2 * out_pad
        self.out_buf = torch.full((n,), float("nan"), dtype=TORCH_DT[c.dtype], device="cuda")

    def run(self, stream=None) -> int:
        c = self.c
        out_ptr = self.out_buf.data_ptr() + self.pad * self.out_buf.element_size()
        s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        if c.mask_kind == I.MASK_SLIDING:
            return S.sdpa_forward_window(self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(), out_ptr,
                                         c.B, c.Hq, c.Hkv, c.Lq, c.Lk, c.Dqk, c.Dv, c.all_strides16, c.scale,
                                         c.window, c.dtype, s)
        return S.sdpa_forward(self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(), out_ptr,
                              c.B, c.Hq, c.Hkv, c.Lq, c.Lk, c.Dqk, c.Dv, c.all_strides16, c.scale, c.mask_kind,
                              None if self.mask is None else self.mask.data_ptr(),
                              None if self.mask is None else c.mask_strides, c.dtype, s)

    def output(self) -> np.ndarray:
        """float64 [B, Hq, Lq, Dv] from the strided output; checks the guard bands stay NaN."""
        c = self.c
        torch.cuda.synchronize()
        buf = self.out_buf.float().cpu().numpy().astype(np.float64)
        assert np.isnan(buf[:self.pad]).all() and np.isnan(buf[len(buf) - self.pad:]).all(), "wrote outside out"
        body = buf[self.pad:]
        so = c.out_strides
        idx = (np.arange(c.B)[:, None, None, None] * so[0] + np.arange(c.Hq)[None, :, None, None] * so[1]
               + np.arange(c.Lq)[None, None, :, None] * so[2] + np.arange(c.Dv)[None, None, None, :] * so[3])
        return body[idx]


def oracle_rows(c: I.Case, rows=None):
    return oracle.sdpa_rows(c.q, c.k, c.v, B=c.B, Hq=c.Hq, Hkv=c.Hkv, Lq=c.Lq, Lk=c.Lk, Dqk=c.Dqk, Dv=c.Dv,
                            strides=c.strides, scale=c.scale, dtype=c.dtype, mask_kind=c.mask_kind, mask=c.mask,
                            mask_strides=c.mask_strides, rows=rows, window=c.window)


def compare(c: I.Case, got: np.ndarray, rows=None, label=""):
    """got: float64 [B,Hq,Lq,Dv].  rows: optional (n,3) sample; else every row."""
    ref = oracle_rows(c, rows)
    if rows is None:
        g = got.reshape(-1, c.Dv)
    else:
        g = got[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert np.isfinite(g).all(), f"{label}: non-finite output"
    err = np.abs(g - ref)
    mx, mean = float(err.max()), float(err.mean())
    tmax, tmean = TOL[c.dtype]
    assert mx <= tmax and mean <= tmean, f"{label}: max-abs {mx:.3e} (tol {tmax}), mean-abs {mean:.3e} (tol {tmean})"
    return mx, mean


def run_and_check(c: I.Case, rows=None, label="", expect_path=None):
    g = GpuCase(c)
    st = g.run()
    assert st == 0, f"{label}: status {st} {S.sdpa_error_string(st)} {S.sdpa_last_cuda_error()}"
    got = g.output()
    if rows is None:
        assert np.isfinite(got).all(), f"{label}: NaN left in the output (unwritten rows?)"
    return compare(c, got, rows, label), got
