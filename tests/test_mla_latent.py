"""Absorbed multi-head latent attention (MLA) decode on the small fixture of
mlxcel issue #1065 ("f32 matmul and single-query SDPA lose ~fp16 precision on
M5"), section "Why this is a precision problem": num_heads 4, kv_lora_rank 32,
qk_nope_head_dim 16, qk_rope_head_dim 8, v_head_dim 12, and the failing test
"absorbed attention respects an additive causal mask".

In the absorbed form the key up-projection is folded into the query
(q_abs = [q_nope . W_uk, q_rope]), every head attends over one shared latent
cache K = [c | k_rope] (Hkv = 1, Dqk = 32 + 8 = 40), and the values are the
latent columns c themselves (Dv = 32), passed as a strided alias of K; the
value up-projection W_uv is applied to the attention output afterwards.  The
scale is (qk_nope + qk_rope)^-0.5.

CPU: the oracle's absorbed result, up-projected, must equal the explicit
(non-absorbed) attention written out in numpy with per-head keys and values.
GPU: the library against the oracle, decode and prefill, with V aliasing K.
"""
import dataclasses

import numpy as np
import pytest

from scaled_dot_product_14_b200 import inputs as I

HEADS, RANK, NOPE, ROPE, VDIM = 4, 32, 16, 8, 12
DQK, DV = RANK + ROPE, RANK
SCALE = float(np.float32((NOPE + ROPE) ** -0.5))


def causal_additive(Lq, Lk):
    """0 where key j is visible to query i (bottom-right: j <= i + Lk - Lq), -inf elsewhere."""
    i = np.arange(Lq)[:, None]
    j = np.arange(Lk)[None, :]
    return np.where(j <= i + (Lk - Lq), 0.0, -np.inf)


def mla_parts(seed, Lq, Lk, dyadic=False):
    """Latent cache, rope keys, projections and queries.  dyadic: entries in
    {-1, -1/2, 0, 1/2, 1}, so every product and the absorbed query are exact in fp32."""
    rng = np.random.default_rng(seed)

    def draw(*shape):
        if dyadic:
            return rng.integers(-2, 3, size=shape).astype(np.float64) / 2.0
        return rng.standard_normal(shape).astype(np.float32).astype(np.float64)

    return dict(c=draw(Lk, RANK), k_rope=draw(Lk, ROPE), w_uk=draw(HEADS, NOPE, RANK),
                w_uv=draw(HEADS, VDIM, RANK), q_nope=draw(HEADS, Lq, NOPE), q_rope=draw(HEADS, Lq, ROPE))


def absorbed_case(parts, dtype=I.F32, mask=True) -> I.Case:
    """The absorbed problem as one library call: q [1, H, Lq, 40], K [1, 1, Lk, 40],
    V = the first 32 columns of K (same buffer, same strides)."""
    H, Lq, _ = parts["q_nope"].shape
    Lk = parts["c"].shape[0]
    q_abs = np.concatenate([np.einsum("hin,hnr->hir", parts["q_nope"], parts["w_uk"]), parts["q_rope"]], axis=2)
    kbuf = np.concatenate([parts["c"], parts["k_rope"]], axis=1)
    q = I.to_storage(q_abs.astype(np.float32).reshape(-1), dtype)
    k = I.to_storage(kbuf.astype(np.float32).reshape(-1), dtype)
    qs = tuple(I.strides_for("bhld", 1, H, Lq, DQK))
    ks = tuple(I.strides_for("bhld", 1, 1, Lk, DQK))
    os_ = tuple(I.strides_for("bhld", 1, H, Lq, DV))
    c = I.Case(1, H, 1, Lq, Lk, DQK, DV, dtype, q, k, k, qs + ks + ks, os_, SCALE)
    if mask:
        m = causal_additive(Lq, Lk).astype(np.float32).reshape(-1)
        c = dataclasses.replace(c, mask_kind=I.MASK_ADDITIVE, mask=I.to_storage(m, dtype),
                                mask_strides=(0, 0, Lk, 1))
    return c


def explicit_attention(parts, mask=True):
    """Non-absorbed MLA attention in float64: per-head keys [c W_uk^T | k_rope],
    per-head values c W_uv^T, materialised scores; returns [H, Lq, VDIM]."""
    H, Lq, _ = parts["q_nope"].shape
    Lk = parts["c"].shape[0]
    out = np.zeros((H, Lq, VDIM))
    add = causal_additive(Lq, Lk) if mask else np.zeros((Lq, Lk))
    for h in range(H):
        k_nope = parts["c"] @ parts["w_uk"][h].T                   # [Lk, NOPE]
        v = parts["c"] @ parts["w_uv"][h].T                        # [Lk, VDIM]
        s = SCALE * (parts["q_nope"][h] @ k_nope.T + parts["q_rope"][h] @ parts["k_rope"].T) + add
        for i in range(Lq):
            row = s[i]
            if np.all(np.isneginf(row)):
                continue
            p = np.exp(row - row.max())
            out[h, i] = (p / p.sum()) @ v
    return out


def oracle_absorbed(oracle_mod, c):
    return oracle_mod.sdpa_full(c.q, c.k, c.v, B=c.B, Hq=c.Hq, Hkv=c.Hkv, Lq=c.Lq, Lk=c.Lk, Dqk=c.Dqk,
                                Dv=c.Dv, strides=c.strides, scale=c.scale, dtype=c.dtype,
                                mask_kind=c.mask_kind, mask=c.mask, mask_strides=c.mask_strides)


@pytest.mark.parametrize("Lq,Lk", [(1, 1), (1, 9), (4, 4), (4, 9), (16, 33)])
@pytest.mark.parametrize("mask", [True, False])
def test_absorbed_equals_explicit_attention(oracle_mod, Lq, Lk, mask):
    """Folding W_uk into the query and W_uv after the softmax changes nothing:
    the oracle's absorbed latent output, up-projected, equals the explicit
    per-head attention (exact inputs, float64 on both sides)."""
    parts = mla_parts(90 + Lq * 7 + Lk, Lq, Lk, dyadic=True)
    c = absorbed_case(parts, mask=mask)
    lat = oracle_absorbed(oracle_mod, c)[0]                        # [H, Lq, 32]
    got = np.einsum("hir,hvr->hiv", lat, parts["w_uv"])
    ref = explicit_attention(parts, mask=mask)
    assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_absorbed_value_alias_is_the_latent_prefix(oracle_mod):
    """With one visible key the latent output is that key's first 32 columns:
    V is read through K's strides, not a copy."""
    parts = mla_parts(97, 4, 9, dyadic=True)
    c = absorbed_case(parts)
    lat = oracle_absorbed(oracle_mod, c)[0]
    # bottom-right causal: query 0 of 4 over 9 keys sees keys 0..5; none of them alone,
    # so use Lq = Lk = 1 for the closed form
    one = absorbed_case(mla_parts(98, 1, 1, dyadic=True))
    lat1 = oracle_absorbed(oracle_mod, one)[0]
    kb = I.storage_to_f32(one.k, one.dtype).reshape(1, DQK)
    assert np.array_equal(lat1[:, 0, :], np.broadcast_to(kb[0, :DV], (HEADS, DV)))
    assert np.isfinite(lat).all()


# ---------------------------------------------------------------------------- GPU
@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [I.F32, I.BF16, I.F16])
@pytest.mark.parametrize("Lk", [1, 7, 64, 300, 4096])
def test_mla_decode_gpu(dtype, Lk):
    import scaled_dot_product_14_b200 as S
    from gpu_util import GpuCase, compare
    c = absorbed_case(mla_parts(1950 + Lk, 1, Lk), dtype=dtype)
    g = GpuCase(c)
    g.v = g.k                                  # V is the latent prefix of K on the device too
    assert g.run() == 0
    compare(c, g.output(), label=f"mla decode Lk={Lk}")
    assert S.sdpa_last_launch_count() >= 1


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [I.F32, I.BF16])
def test_mla_chunked_matches_unchunked_gpu(dtype):
    """The failing case of the page: four queries with the additive causal mask,
    run whole and one query at a time over the visible key prefix."""
    from gpu_util import GpuCase, compare, TOL
    Lq, Lk = 4, 300
    parts = mla_parts(1960, Lq, Lk)
    c = absorbed_case(parts, dtype=dtype)
    g = GpuCase(c)
    g.v = g.k
    assert g.run() == 0
    full = g.output()
    compare(c, full, label="mla unchunked")
    tmax, _ = TOL[dtype]
    for a in range(Lq):
        sub_parts = dict(parts, q_nope=parts["q_nope"][:, a:a + 1], q_rope=parts["q_rope"][:, a:a + 1],
                         c=parts["c"][:Lk - Lq + a + 1], k_rope=parts["k_rope"][:Lk - Lq + a + 1])
        sc = absorbed_case(sub_parts, dtype=dtype)
        sg = GpuCase(sc)
        sg.v = sg.k
        assert sg.run() == 0
        part = sg.output()
        compare(sc, part, label=f"mla chunk {a}")
        assert np.abs(part[:, :, 0] - full[:, :, a]).max() <= 2 * tmax


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", [I.F32, I.BF16])
def test_mla_prefill_gpu(dtype):
    """Many queries at once (prefill path) over the same latent cache."""
    from gpu_util import GpuCase, compare
    c = absorbed_case(mla_parts(1970, 100, 333), dtype=dtype)
    g = GpuCase(c)
    g.v = g.k
    assert g.run() == 0
    compare(c, g.output(), label="mla prefill")
