"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/sdpa.h declares, and its validation (shared by
sdpa_supported and sdpa_forward) returns the documented statuses before any
CUDA call."""
import ctypes
import re

import pytest

import scaled_dot_product_14_b200 as S
from scaled_dot_product_14_b200 import inputs as I


@pytest.fixture(scope="module")
def lib():
    from scaled_dot_product_14_b200 import build
    build.build()
    return S.lib()


def declared_functions():
    text = open(S.HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sdpa_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "sdpa_forward" in names and "sdpa_supported" in names
    for n in names:
        assert hasattr(lib, n), n


def test_abi_version(lib):
    assert S.sdpa_abi_version() == 2


def strides16(layout, B, Hq, Hkv, Lq, Lk, Dqk, Dv):
    return (I.strides_for(layout, B, Hq, Lq, Dqk) + I.strides_for(layout, B, Hkv, Lk, Dqk)
            + I.strides_for(layout, B, Hkv, Lk, Dv) + I.strides_for(layout, B, Hq, Lq, Dv))


def sup(B=1, Hq=32, Hkv=8, Lq=1, Lk=4096, Dqk=256, Dv=None, layout="bhld", mask_kind=0, mask_strides=None,
        dtype=2, strides=None):
    Dv = Dqk if Dv is None else Dv
    st = strides if strides is not None else strides16(layout, B, Hq, Hkv, Lq, Lk, Dqk, Dv)
    return S.sdpa_supported(B, Hq, Hkv, Lq, Lk, Dqk, Dv, st, mask_kind, mask_strides, dtype)


@pytest.mark.parametrize("D,Dv", [(64, 64), (72, 72), (80, 80), (96, 96), (128, 128), (192, 128), (256, 256), (512, 512),
                                  (40, 32)])
@pytest.mark.parametrize("dtype", [0, 1, 2])
@pytest.mark.parametrize("layout", ["bhld", "blhd"])
def test_supported_head_dims_both_paths(lib, D, Dv, dtype, layout):
    assert sup(Lq=1, Dqk=D, Dv=Dv, dtype=dtype, layout=layout) == (0, S.SDPA_PATH_DECODE)
    assert sup(Lq=8, Dqk=D, Dv=Dv, dtype=dtype, layout=layout) == (0, S.SDPA_PATH_DECODE)
    assert sup(Lq=9, Dqk=D, Dv=Dv, dtype=dtype, layout=layout) == (0, S.SDPA_PATH_PREFILL)
    assert sup(Lq=8192, Lk=8192, Dqk=D, Dv=Dv, dtype=dtype, layout=layout) == (0, S.SDPA_PATH_PREFILL)


@pytest.mark.parametrize("D,Dv", [(32, 32), (48, 48), (192, 192), (128, 64), (256, 128), (512, 256), (100, 100),
                                  (40, 40), (32, 40), (40, 24)])
def test_unsupported_head_dims_are_errors(lib, D, Dv):
    assert sup(Dqk=D, Dv=Dv)[0] == 2


def test_invalid_arguments(lib):
    assert sup(Hq=30, Hkv=8)[0] == 1          # Hq % Hkv != 0
    assert sup(Hkv=0, Hq=0)[0] == 1
    assert sup(B=-1)[0] == 1
    assert sup(dtype=3)[0] == 1
    assert sup(mask_kind=5)[0] == 1
    assert sup(mask_kind=S.SDPA_MASK_ADDITIVE, mask_strides=None)[0] == 1


def test_stride_rules(lib):
    st = list(strides16("bhld", 1, 32, 8, 1, 4096, 256, 256))
    bad = list(st); bad[3] = 2                  # d-stride must be 1
    assert sup(strides=bad)[0] == 3
    bad = list(st); bad[6] = 257                 # k l-stride * 2 bytes not a multiple of 16
    assert sup(strides=bad)[0] == 3
    bad = list(st); bad[5] = -256 * 4096         # negative head stride
    assert sup(strides=bad)[0] == 3
    ok = list(st); ok[2] = 7                     # q l-stride irrelevant when Lq == 1
    assert sup(strides=ok)[0] == 0
    assert sup(mask_kind=S.SDPA_MASK_BOOL, mask_strides=(0, 0, 0, 1))[0] == 0
    assert sup(mask_kind=S.SDPA_MASK_BOOL, mask_strides=(0, 0, -1, 1))[0] == 3
    # fp32 D=72 [B,L,H,D]: 288-byte rows are 16-byte multiples
    assert sup(Dqk=72, dtype=0, layout="blhd", Lq=100, Lk=100)[0] == 0


def test_empty_problems_take_no_path(lib):
    assert sup(B=0) == (0, S.SDPA_PATH_NONE)
    assert sup(Lq=0) == (0, S.SDPA_PATH_NONE)
    assert sup(Hq=0) == (0, S.SDPA_PATH_NONE)


def test_too_large(lib):
    assert sup(B=70000)[0] == 10
    assert sup(Lk=1 << 31)[0] == 10


def test_forward_rejects_before_touching_cuda(lib):
    S.sdpa_reset_counters()
    st = strides16("bhld", 1, 4, 2, 16, 16, 64, 64)
    args = dict(B=1, Hq=4, Hkv=2, Lq=16, Lk=16, Dqk=64, Dv=64, strides=st, scale=0.125, mask_kind=0, mask=None,
                mask_strides=None, dtype=2, stream=None)
    call = lambda **kw: S.sdpa_forward(*[kw.get(n, args.get(n, 4096 if n in "qkvout" else None)) for n in
                                        ["q", "k", "v", "out"]], **{n: kw.get(n, args[n]) for n in args})
    assert call(Dqk=100, Dv=100) == 2
    assert call(q=0) == 9                                  # null q
    assert call(q=4096 + 8) == 4                           # misaligned
    assert call(mask_kind=S.SDPA_MASK_BOOL, mask=None, mask_strides=(0, 0, 16, 1)) == 9
    assert call(mask_kind=S.SDPA_MASK_NONE, mask=4096) == 9
    assert call(scale=float("nan")) == 1
    assert call(B=0) == 0                                  # empty: OK, nothing launched
    c = S.sdpa_get_counters()
    assert c["calls"] == 7 and c["rejected_calls"] == 6 and c["empty_calls"] == 1
    assert c["calls"] == c["prefill_calls"] + c["decode_calls"] + c["empty_calls"] + c["rejected_calls"]


def test_error_strings(lib):
    for code in range(0, 11):
        assert S.sdpa_error_string(code) and S.sdpa_error_string(code) != "unknown status"
    assert S.sdpa_error_string(99) == "unknown status"


def test_package_fails_loudly_without_library(monkeypatch, tmp_path):
    import importlib
    monkeypatch.setattr(S, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(S, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        S.lib()


def test_debug_hooks_validate_their_arguments(lib):
    assert S.sdpa_debug_set(S.SDPA_DEBUG_WAIT_LIMIT_NS, 0) == 0
    assert S.sdpa_debug_set(S.SDPA_DEBUG_DECODE_BARRIER_EXTRA, 0) == 0
    assert S.sdpa_debug_set(S.SDPA_DEBUG_DECODE_BARRIER_EXTRA, -1) == 1
    assert S.sdpa_debug_set(S.SDPA_DEBUG_DECODE_BARRIER_EXTRA, 5000) == 1
    assert S.sdpa_debug_set(S.SDPA_DEBUG_FAIL_ALLOCS, -3) == 1
    assert S.sdpa_debug_set(S.SDPA_DEBUG_FAIL_ALLOCS, 0) == 0
    assert S.sdpa_debug_set(77, 1) == 1
    assert S.sdpa_workspace_bytes() >= 0


def _noalloc(B=1, Hq=4, Hkv=1, Lq=1, Lk=64, Dqk=40, Dv=32, dtype=2, ptr=4096):
    st = strides16("bhld", B, Hq, Hkv, Lq, Lk, Dqk, Dv)
    return S.sdpa_forward_noalloc(ptr, ptr, ptr, ptr, B, Hq, Hkv, Lq, Lk, Dqk, Dv, st, Dqk ** -0.5, 0, None, None,
                                  dtype, None)


def test_noalloc_rejects_uncovered_cases_before_any_cuda_call(lib):
    """sdpa_forward_noalloc decides every argument status on the host before it
    touches CUDA, so these run without a GPU: the absorbed-MLA dims (40, 32),
    which have no tensor-core decode kernel, are refused (once they reached the
    split planner with an empty shape), as are fp32, prefill lengths and null
    or misaligned pointers."""
    assert _noalloc(Dqk=40, Dv=32, dtype=2) == 1
    assert _noalloc(Dqk=40, Dv=32, dtype=1) == 1
    assert _noalloc(Dqk=256, Dv=256, dtype=0) == 1
    assert _noalloc(Dqk=256, Dv=256, Lq=9, Lk=9) == 1
    assert _noalloc(Dqk=100, Dv=100) == 2
    assert _noalloc(Dqk=256, Dv=256, ptr=0) == 9
    assert _noalloc(Dqk=256, Dv=256, ptr=4096 + 2) == 4
    assert _noalloc(Dqk=256, Dv=256, B=0) == 0


def test_sliding_window_kind_is_validated_on_the_host(lib):
    assert sup(mask_kind=S.SDPA_MASK_SLIDING) == (0, S.SDPA_PATH_DECODE)
    assert sup(mask_kind=S.SDPA_MASK_SLIDING, Lq=100, Lk=100) == (0, S.SDPA_PATH_PREFILL)
    assert sup(mask_kind=5)[0] == 1
    st = strides16("bhld", 1, 4, 2, 16, 16, 64, 64)
    # window < 1 is refused before any CUDA call
    assert S.sdpa_forward_window(4096, 4096, 4096, 4096, 1, 4, 2, 16, 16, 64, 64, st, 0.125, 0, 2, None) == 1
