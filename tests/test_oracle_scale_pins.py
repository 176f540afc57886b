"""Pins of the oracle's per-vector scales (CPU).

The LSE README's "KV cache formats" table gives fp8/bf8 "with scales" 512
extra bytes per token over the 8-bit elements: one FP32 scale per (token, kv
head) of K and of V, the vector times its scale being the key or value.  The
oracle reads them from a block per fragment ([kv_head][token]).  Pinned here:

* against torch float64 SDPA on the generator's logical vectors times the
  scales the generator drew (so the oracle reads back what the layout writer
  wrote, for chain and tree rows, both 8-bit formats, a wide scale range);
* unit scales give the unscaled result bit for bit;
* power-of-two scales give, bit for bit, the result of an FP32 cache holding
  the scaled values (a different decoder and no scale array);
* V scales times 4 multiply the output by 4 and leave lse unchanged;
  K scales times 1/4 equal Q times 1/4;
* a zero V scale keeps the key's weight in the denominator.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from verify_attention_paged_b200 import workloads as wl
from conftest import to_problem
from test_oracle_pins import sdpa_reference

FP8 = ["e4m3", "e5m2"]


def scaled_case(dtype, seed, spread=6.0, tree=True, tpf=8):
    return wl.small_case(dtype, [37, 64, 5, 16], [3, 1, 5, 2], n_q_heads=8, n_kv_heads=2,
                         head_dim=16, tokens_per_fragment=tpf, tree=tree, seed=seed,
                         scaled=True, scale_spread=spread, magnitude_spread=spread)


def with_scales(w, scales):
    return wl.Workload(**{**w.__dict__, "scales": scales})


@pytest.mark.parametrize("dtype", FP8)
@pytest.mark.parametrize("tree", [False, True])
def test_scaled_matches_library_sdpa(dtype, tree):
    w = scaled_case(dtype, seed=61, tree=tree)
    live = ~np.isnan(w.scales)
    assert np.ptp(np.log2(w.scales[live])) > 6  # the scales span a wide range
    out, lse = orc.attention(to_problem(w))
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    np.testing.assert_allclose(out, sdpa_reference(w), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("dtype", FP8)
def test_unit_scales_are_bitwise_unscaled(dtype):
    w = wl.small_case(dtype, [37, 20], [3, 4], n_q_heads=4, n_kv_heads=2, head_dim=8,
                      tokens_per_fragment=8, tree=True, seed=62)
    n = len(w.chunks) * (w.chunk_bytes // w.fragment_bytes) * w.n_kv_heads * \
        w.tokens_per_fragment
    a = orc.attention(to_problem(w))
    b = orc.attention(to_problem(with_scales(w, np.ones(n, np.float32))))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def _f32_copy_scaled(w):
    """An FP32 cache with the same page tables whose vectors are the stored
    8-bit vectors times their scales (exact for power-of-two scales), built
    from the fragments through torch's FP8 -> FP32 conversion."""
    T = w.tokens_per_fragment
    Hkv, D = w.n_kv_heads, w.head_dim
    fpc = w.chunk_bytes // w.fragment_bytes
    fb32 = w.fragment_bytes * 4
    chunks = [np.full(fb32 * fpc, 0xFF, np.uint8) for _ in w.chunks]
    tdt = wl.TORCH_DTYPES[w.dtype]
    for f in range(len(w.chunks) * fpc):
        c, o = divmod(f, fpc)
        raw = torch.from_numpy(w.chunks[c][o * w.fragment_bytes:(o + 1) * w.fragment_bytes].copy())
        vals = raw.view(tdt).to(torch.float32).reshape(T, Hkv, D)
        sc = torch.from_numpy(w.scales[f * Hkv * T:(f + 1) * Hkv * T].reshape(Hkv, T).T.copy())
        vals = vals * torch.nan_to_num(sc, nan=1.0)[:, :, None]
        chunks[c][o * fb32:(o + 1) * fb32] = vals.contiguous().view(torch.uint8).reshape(-1).numpy()
    return wl.Workload(**{**w.__dict__, "dtype": "f32", "chunks": chunks, "fragment_bytes": fb32,
                          "chunk_bytes": fb32 * fpc, "scales": None})


@pytest.mark.parametrize("dtype", FP8)
def test_power_of_two_scales_equal_an_fp32_cache(dtype):
    w = wl.small_case(dtype, [37, 64, 5], [3, 1, 5], n_q_heads=6, n_kv_heads=3, head_dim=16,
                      tokens_per_fragment=8, tree=True, seed=63)
    rng = np.random.default_rng(5)
    n = len(w.chunks) * (w.chunk_bytes // w.fragment_bytes) * w.n_kv_heads * \
        w.tokens_per_fragment
    w = with_scales(w, np.exp2(rng.integers(-12, 8, n)).astype(np.float32))
    a = orc.attention(to_problem(w))
    b = orc.attention(to_problem(_f32_copy_scaled(w)))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_constant_scales():
    w = scaled_case("e4m3", seed=64, spread=0.0)
    base_out, base_lse = orc.attention(to_problem(w))
    T, Hkv = w.tokens_per_fragment, w.n_kv_heads
    is_v = np.zeros_like(w.scales, bool)
    for f in w.v_pages[w.v_pages >= 0]:
        is_v[f * Hkv * T:(f + 1) * Hkv * T] = True
    # V scales times 4 (exact in FP32): output times 4 bit for bit, lse unchanged
    s2 = np.where(is_v, w.scales * 4, w.scales).astype(np.float32)
    out, lse = orc.attention(to_problem(with_scales(w, s2)))
    assert np.array_equal(out, 4 * base_out)
    assert np.array_equal(lse, base_lse)
    # K scales times 0.25 (exact): the same as Q times 0.25
    s3 = np.where(is_v, w.scales, w.scales * 0.25).astype(np.float32)
    out3, lse3 = orc.attention(to_problem(with_scales(w, s3)))
    out4, lse4 = orc.attention(to_problem(w, q=(w.q * 0.25).astype(np.float32)))
    np.testing.assert_allclose(out3, out4, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse3, lse4, rtol=1e-12, atol=1e-14)


def test_zero_v_scale_keeps_the_key_in_the_denominator():
    # one sequence, one row, two keys: the second key's V scale is 0, so
    # out = sigma(x0 - x1) V0 and lse is unchanged
    w = wl.small_case("e4m3", [2], [1], n_q_heads=1, n_kv_heads=1, head_dim=8,
                      tokens_per_fragment=8, seed=65, scaled=True)
    T = w.tokens_per_fragment
    f1 = int(w.v_pages[0, 0])
    s = w.scales.copy()
    s[f1 * T + 1] = 0.0
    out, lse = orc.attention(to_problem(with_scales(w, s)))
    base_out, base_lse = orc.attention(to_problem(w))
    k = [w.logical_k[0][j, 0].to(torch.float64).numpy() * w.logical_k_scale[0][j, 0]
         for j in range(2)]
    v0 = w.logical_v[0][0, 0].to(torch.float64).numpy() * w.logical_v_scale[0][0, 0]
    q = w.q[0, 0].astype(np.float64)
    x = [w.scale * float(q @ kj) for kj in k]
    p0 = 1.0 / (1.0 + np.exp(x[1] - x[0]))
    np.testing.assert_allclose(out[0, 0], p0 * v0, rtol=1e-13, atol=1e-15)
    assert lse[0, 0] == base_lse[0, 0]


def test_scale_array_must_cover_the_arena():
    w = scaled_case("e5m2", seed=66)
    with pytest.raises(orc.OracleError):
        orc.attention(to_problem(with_scales(w, w.scales[:-1])))


def test_scaled_contiguous_cache_is_bitwise_equal():
    # relaying the fragments (and their scale blocks) into identity tables
    # leaves the scaled problem unchanged, bit for bit
    w = scaled_case("e5m2", seed=67)
    c = wl.contiguous_copy(w)
    a = orc.attention(to_problem(w))
    b = orc.attention(to_problem(c))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert np.isnan(c.scales).sum() == np.isnan(w.scales).sum()
