"""The pins must be sharp: each plausible mistake planted in a copy of the
oracle's C source (compiled on the CPU into a temporary library) must make at
least one pin fail.  Every mutant keeps its memory accesses in bounds."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle as O
from scaled_dot_product_14_b200 import inputs as I

from test_oracle import _page1, _torch_ref, full, logical

MUTANTS = {
    "gqa_mapping_modulo": ("const int64_t g = h / n_rep;", "const int64_t g = h % Hkv;"),
    "causal_top_left": ("if (j > i + (Lk - Lq)) sj = -INFINITY;", "if (j > i) sj = -INFINITY;"),
    "causal_reversed": ("if (j > i + (Lk - Lq)) sj = -INFINITY;", "if (j < i + (Lk - Lq)) sj = -INFINITY;"),
    "scale_dropped": ("double sj = scale * dot;", "double sj = dot;"),
    "mask_subtracted": ("sj += oracle_load(mask, midx, dtype);", "sj -= oracle_load(mask, midx, dtype);"),
    "bool_polarity": ("if (((const uint8_t*)mask)[midx] == 0) sj = -INFINITY;",
                      "if (((const uint8_t*)mask)[midx] != 0) sj = -INFINITY;"),
    "k_reversed_d": ("j * sk[2] + d * sk[3]", "j * sk[2] + (Dqk - 1 - d) * sk[3]"),
    "no_normalise": ("for (int64_t e = 0; e < Dv; ++e) o[e] /= l;", ";"),
    "mask_lq_index_dropped": ("i * (mask_st ? mask_st[2] : 0)", "0"),
    "bf16_low_half": ("uint32_t bits = ((uint32_t)b) << 16;", "uint32_t bits = ((uint32_t)b) << 15;"),
    "mask_scaled": ("sj += oracle_load(mask, midx, dtype);", "sj += scale * oracle_load(mask, midx, dtype);"),
    "causal_off_by_one": ("if (j > i + (Lk - Lq)) sj = -INFINITY;", "if (j >= i + (Lk - Lq)) sj = -INFINITY;"),
    "v_from_kv_head_zero": ("g * sv[1] + j * sv[2]", "0 * sv[1] + j * sv[2]"),
    "q_from_kv_head": ("b * sq[0] + h * sq[1]", "b * sq[0] + g * sq[1]"),
    "dot_over_dv": ("for (int64_t d = 0; d < Dqk; ++d) {", "for (int64_t d = 0; d < (Dv < Dqk ? Dv : Dqk); ++d) {"),
    "empty_row_guard_dropped": ("if (l > 0.0) {", "{"),
    "window_off_by_one": ("if (j > own || j <= own - window) sj = -INFINITY;",
                          "if (j > own || j < own - window) sj = -INFINITY;"),
    "window_not_causal": ("if (j > own || j <= own - window) sj = -INFINITY;",
                          "if (j <= own - window) sj = -INFINITY;"),
    "window_top_left": ("const int64_t own = i + (Lk - Lq);", "const int64_t own = i;"),
}


def _pins_hold() -> bool:
    """A compact set of pins; True if all hold for the currently loaded oracle."""
    try:
        import json
        gold = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "mlx3585_linspace.json")))["printed"]
        x, C, C_blhd, M, G = _page1(O)
        if abs(np.abs(G - M).max() - gold["manual_vs_fused_max_diff"]) > 6e-8:
            return False
        if abs(np.abs(G - C_blhd).max() - gold["manual_vs_pytorch_fused_max_diff"]) > 6e-8:
            return False
        for mask in ["none", "additive", "bool", "causal"]:
            c = I.make_case(77, 1, 4, 2, 6, 6, 64, dtype=I.BF16, mask=mask)
            if c.mask_kind == I.MASK_BOOL:
                c.mask.reshape(c.Lq, c.Lk)[:, 0] = 1
            if np.abs(full(O, c) - _torch_ref(c)).max() > 1e-12:
                return False
        # Dqk != Dv: the score sum runs over Dqk, the output over Dv
        c = I.make_case(79, 1, 4, 2, 5, 7, 192, 128, dtype=I.BF16)
        if np.abs(full(O, c) - _torch_ref(c)).max() > 1e-12:
            return False
        # bottom-right causal with Lq > Lk: queries 0..2 see no key and give exact zeros
        c = I.make_case(80, 1, 2, 2, 6, 3, 64, dtype=I.F32, mask="causal")
        o = full(O, c)
        if not (np.all(o[:, :, :3] == 0.0) and np.isfinite(o).all()):
            return False
        # causal with Lq != Lk: the query chunk [3, 4) of a Lq = 4 problem
        c = I.make_case(78, 1, 2, 2, 4, 9, 64, dtype=I.F32, mask="causal")
        last = full(O, c)[:, :, 3:4]
        from test_oracle import with_values
        sub = I.make_case(78, 1, 2, 2, 1, 9, 64, dtype=I.F32, mask="causal")
        sub = with_values(sub, q=logical(c, "q")[:, :, 3:4], k=logical(c, "k"), v=logical(c, "v"))
        if np.abs(full(O, sub) - last).max() > 1e-12:
            return False
        # sliding window of one key, Lq < Lk: every row is its own key's V row
        c = I.make_case(81, 1, 2, 1, 3, 7, 64, dtype=I.F32, mask="sliding", window=1)
        o, v = full(O, c), logical(c, "v")
        if not all(np.array_equal(o[0, h, i], v[0, 0, i + 4]) for h in range(2) for i in range(3)):
            return False
        return True
    except ValueError:
        return False


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, oracle_mod, name):
    src = open(os.path.join(os.path.dirname(O.__file__), "sdpa_oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "mut.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(path), "-lm"])
    saved = O._load()
    lib = ctypes.CDLL(str(so))
    lib.oracle_sdpa_rows.restype = saved.oracle_sdpa_rows.restype
    lib.oracle_sdpa_rows.argtypes = saved.oracle_sdpa_rows.argtypes
    O._lib = lib
    try:
        assert not _pins_hold(), f"mutant {name} slipped through every pin"
    finally:
        O._lib = saved


def test_unmutated_oracle_passes_the_same_pins(oracle_mod):
    assert _pins_hold()
