"""Pins for the float64 oracle, against things other than itself.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a wrong page or head lookup, a
wrong bit in a decoder) fails at least one of them:

* a library routine on the special case it covers: torch's float64
  scaled_dot_product_attention on the dense, gathered keys (no paging);
* closed forms: one key gives that key's V and its score as lse; two keys
  give the logistic mix; Q = 0 gives the mean of the visible V rows and
  lse = ln(count); constant V gives that constant;
* invariants: any other fragment placement gives bit-identical output;
  split-then-merge equals unsplit; a parent-chain tree equals the chain mask;
  duplicated query heads of a group agree; output is linear in V;
* codecs: every FP8 code and every 16-bit code decodes like torch's cast;
* the pages' own worked numbers: the bytes-per-token table of the LSE README.
"""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import expit

from oracle import oracle as orc
from verify_attention_paged_b200 import workloads as wl
from conftest import to_problem

DTYPES = ["f32", "f16", "bf16", "e4m3", "e5m2"]
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def sdpa_reference(w):
    """torch float64 SDPA per sequence on dense gathered K/V (library routine)."""
    G = w.n_q_heads // w.n_kv_heads
    outs = []
    for s in range(w.n_seqs):
        L = int(w.seq_lens[s])
        r0, r1 = int(w.row_offsets[s]), int(w.row_offsets[s + 1])
        R = r1 - r0
        C = L - R
        k = w.logical_k[s].to(torch.float64)
        v = w.logical_v[s].to(torch.float64)
        if w.scales is not None:  # per-vector scales, as the generator drew them
            k = k * torch.from_numpy(w.logical_k_scale[s]).to(torch.float64)[:, :, None]
            v = v * torch.from_numpy(w.logical_v_scale[s]).to(torch.float64)[:, :, None]
        k = k.repeat_interleave(G, dim=1).permute(1, 0, 2)
        v = v.repeat_interleave(G, dim=1).permute(1, 0, 2)
        q = torch.from_numpy(w.q[r0:r1].astype(np.float64)).permute(1, 0, 2)
        mask = torch.zeros((R, L), dtype=torch.bool)
        mask[:, :C] = True
        for r in range(R):
            m = int(w.row_masks[r0 + r]) if w.row_masks is not None else (1 << (r + 1)) - 1
            for i in range(R):
                if (m >> i) & 1:
                    mask[r, C + i] = True
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask,
                                                             scale=w.scale)
        outs.append(o.permute(1, 0, 2).numpy())
    return np.concatenate(outs, axis=0)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("tree", [False, True])
def test_matches_library_sdpa(dtype, tree):
    w = wl.small_case(dtype, [37, 64, 5, 16], [3, 1, 5, 2], n_q_heads=8, n_kv_heads=2,
                      head_dim=16, tokens_per_fragment=8, tree=tree, seed=11)
    out, lse = orc.attention(to_problem(w))
    ref = sdpa_reference(w)
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "e4m3"])
def test_mha_and_single_head_group(dtype):
    # G = 1 (MHA) and G = Hq (MQA) both agree with the library routine
    for hq, hkv in ((4, 4), (6, 1)):
        w = wl.small_case(dtype, [29, 3], [2, 3], n_q_heads=hq, n_kv_heads=hkv, head_dim=8,
                          tokens_per_fragment=4, seed=3)
        out, _ = orc.attention(to_problem(w))
        np.testing.assert_allclose(out, sdpa_reference(w), rtol=1e-12, atol=1e-13)


def test_single_key_closed_form():
    for dtype in DTYPES:
        w = wl.small_case(dtype, [1], [1], n_q_heads=4, n_kv_heads=2, head_dim=16,
                          tokens_per_fragment=4, seed=5)
        out, lse = orc.attention(to_problem(w))
        k = w.logical_k[0].to(torch.float64).numpy()[0]   # [Hkv, D]
        v = w.logical_v[0].to(torch.float64).numpy()[0]
        for h in range(4):
            g = h // 2
            assert np.array_equal(out[0, h], v[g])      # exactly that V
            x = w.scale * float(np.dot(w.q[0, h].astype(np.float64), k[g]))
            assert lse[0, h] == pytest.approx(x, rel=1e-14, abs=1e-14)


def test_two_key_closed_form():
    w = wl.small_case("f32", [2], [1], n_q_heads=2, n_kv_heads=1, head_dim=16,
                      tokens_per_fragment=1, seed=9)
    out, lse = orc.attention(to_problem(w))
    k = w.logical_k[0].to(torch.float64).numpy()[:, 0]
    v = w.logical_v[0].to(torch.float64).numpy()[:, 0]
    for h in range(2):
        q = w.q[0, h].astype(np.float64)
        x0, x1 = w.scale * q @ k[0], w.scale * q @ k[1]
        want = expit(x0 - x1) * v[0] + expit(x1 - x0) * v[1]
        np.testing.assert_allclose(out[0, h], want, rtol=1e-13, atol=1e-14)
        assert lse[0, h] == pytest.approx(np.logaddexp(x0, x1), rel=1e-14)


@pytest.mark.parametrize("dtype", DTYPES)
def test_zero_query_gives_mean_of_visible_values(dtype):
    w = wl.small_case(dtype, [50, 9], [4, 3], n_q_heads=4, n_kv_heads=2, head_dim=8,
                      tokens_per_fragment=8, tree=True, seed=21)
    q0 = np.zeros_like(w.q)
    out, lse = orc.attention(to_problem(w, q=q0))
    for s in range(w.n_seqs):
        L = int(w.seq_lens[s]); r0 = int(w.row_offsets[s]); R = int(w.row_offsets[s + 1]) - r0
        C = L - R
        v = w.logical_v[s].to(torch.float64).numpy()
        for r in range(R):
            m = int(w.row_masks[r0 + r])
            vis = list(range(C)) + [C + i for i in range(R) if (m >> i) & 1]
            for h in range(4):
                np.testing.assert_allclose(out[r0 + r, h], v[vis, h // 2].mean(axis=0),
                                           rtol=1e-12, atol=1e-13)
                assert lse[r0 + r, h] == pytest.approx(math.log(len(vis)), rel=1e-14)


def test_constant_values_give_that_constant():
    w = wl.small_case("bf16", [40], [2], n_q_heads=4, n_kv_heads=2, head_dim=8,
                      tokens_per_fragment=8, seed=2)
    # overwrite every live V byte pattern with bf16(0.75) = 0x3F40
    chunks = [c.copy() for c in w.chunks]
    T = w.tokens_per_fragment
    fpc = w.chunk_bytes // w.fragment_bytes
    row = w.n_kv_heads * w.head_dim * 2
    for p in range(math.ceil(40 / T)):
        c, off = divmod(int(w.v_pages[0, p]), fpc)
        n = min(T, 40 - p * T)
        view = chunks[c][off * w.fragment_bytes: off * w.fragment_bytes + n * row]
        view.view(np.uint16)[:] = 0x3F40
    out, _ = orc.attention(to_problem(w, chunks=chunks))
    np.testing.assert_allclose(out, 0.75, rtol=1e-14, atol=0)


def _replace_fragments(w, seed):
    """Same logical content, every fragment moved to a fresh random slot."""
    rng = np.random.default_rng(seed)
    fpc = w.chunk_bytes // w.fragment_bytes
    n_frag = fpc * len(w.chunks)
    perm = rng.permutation(n_frag)          # old id -> new id
    chunks = [np.full_like(c, 0xFF) for c in w.chunks]
    fb = w.fragment_bytes
    for old in range(n_frag):
        new = int(perm[old])
        oc, oo = divmod(old, fpc)
        nc, no = divmod(new, fpc)
        chunks[nc][no * fb:(no + 1) * fb] = w.chunks[oc][oo * fb:(oo + 1) * fb]
    remap = lambda t: np.where(t >= 0, perm[np.maximum(t, 0)], -1).astype(np.int32)  # noqa
    return chunks, remap(w.k_pages), remap(w.v_pages)


@pytest.mark.parametrize("dtype", DTYPES)
def test_fragment_placement_invariance_is_bitwise(dtype):
    w = wl.small_case(dtype, [70, 33, 8], [2, 4, 1], n_q_heads=6, n_kv_heads=3, head_dim=16,
                      tokens_per_fragment=8, tree=True, seed=4)
    out, lse = orc.attention(to_problem(w))
    chunks, kp, vp = _replace_fragments(w, seed=99)
    out2, lse2 = orc.attention(to_problem(w, chunks=chunks, k_pages=kp, v_pages=vp))
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "e5m2"])
def test_contiguous_cache_is_bitwise_equal(dtype):
    # the identity page table over a contiguous cache (the fragment-addressing
    # A/B's other arm) holds the same problem: identical oracle bits
    w = wl.small_case(dtype, [70, 33, 8], [2, 4, 1], n_q_heads=6, n_kv_heads=3, head_dim=16,
                      tokens_per_fragment=8, tree=True, seed=4)
    c = wl.contiguous_copy(w)
    nk = int(sum((w.seq_lens + 7) // 8))
    live = c.k_pages >= 0
    assert np.array_equal(np.sort(c.k_pages[live]), np.arange(nk))
    assert np.array_equal(np.sort(c.v_pages[live]), np.arange(nk, 2 * nk))
    out, lse = orc.attention(to_problem(w))
    out2, lse2 = orc.attention(to_problem(c))
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("kp", [1, 3, 8, 16, 1000])
def test_split_equals_unsplit(dtype, kp):
    w = wl.small_case(dtype, [70, 33, 8], [2, 4, 1], n_q_heads=4, n_kv_heads=2, head_dim=8,
                      tokens_per_fragment=8, tree=True, seed=6)
    out, lse = orc.attention(to_problem(w))
    out_s, lse_s = orc.attention_split(to_problem(w), kp)
    np.testing.assert_allclose(out_s, out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse_s, lse, rtol=1e-12, atol=1e-13)


def test_parent_chain_tree_equals_chain():
    w = wl.small_case("f16", [30, 12], [5, 3], n_q_heads=4, n_kv_heads=2, head_dim=8,
                      tokens_per_fragment=8, seed=8)
    assert w.row_masks is None  # chain by default
    masks = []
    for R in (5, 3):
        m = 0
        for i in range(R):
            m |= 1 << i          # parent[i] = i - 1: ancestors are all earlier rows
            masks.append(m)
    out_c, lse_c = orc.attention(to_problem(w))
    out_t, lse_t = orc.attention(to_problem(w, row_masks=np.array(masks, np.uint64)))
    assert np.array_equal(out_c, out_t) and np.array_equal(lse_c, lse_t)


def test_all_roots_tree_sees_context_and_self():
    # every draft hangs off the context: row r of a tree with all parents -1
    # must equal a one-row decode of a sequence holding only the context + row r
    w = wl.small_case("bf16", [25], [4], n_q_heads=2, n_kv_heads=1, head_dim=8,
                      tokens_per_fragment=4, seed=12)
    masks = np.array([1 << i for i in range(4)], np.uint64)
    out, _ = orc.attention(to_problem(w, row_masks=masks))
    C = 21
    k = w.logical_k[0].to(torch.float64).numpy()[:, 0]
    v = w.logical_v[0].to(torch.float64).numpy()[:, 0]
    for r in range(4):
        keys = list(range(C)) + [C + r]
        for h in range(2):
            x = w.scale * (k[keys] @ w.q[r, h].astype(np.float64))
            p = np.exp(x - x.max())
            np.testing.assert_allclose(out[r, h], (p[:, None] * v[keys]).sum(0) / p.sum(),
                                       rtol=1e-12, atol=1e-13)


def test_duplicated_heads_agree():
    w = wl.small_case("e5m2", [45], [3], n_q_heads=6, n_kv_heads=2, head_dim=16,
                      tokens_per_fragment=8, seed=13)
    q = w.q.copy()
    q[:, 1] = q[:, 0]          # heads 0 and 1 are in group 0
    q[:, 5] = q[:, 3]          # heads 3 and 5 are in group 1
    out, lse = orc.attention(to_problem(w, q=q))
    assert np.array_equal(out[:, 0], out[:, 1]) and np.array_equal(out[:, 3], out[:, 5])
    assert not np.allclose(out[:, 0], out[:, 3])   # different kv heads differ


def test_linear_in_values_for_fp32():
    w = wl.small_case("f32", [33], [2], n_q_heads=2, n_kv_heads=1, head_dim=8,
                      tokens_per_fragment=4, seed=14)
    T = w.tokens_per_fragment
    fpc = w.chunk_bytes // w.fragment_bytes
    row = w.head_dim * 4

    def with_v(scale_a, add_b):
        chunks = [c.copy() for c in w.chunks]
        for p in range(math.ceil(33 / T)):
            c, off = divmod(int(w.v_pages[0, p]), fpc)
            n = min(T, 33 - p * T)
            f = chunks[c][off * w.fragment_bytes: off * w.fragment_bytes + n * row].view(np.float32)
            f[:] = f * scale_a + add_b
        return orc.attention(to_problem(w, chunks=chunks))[0]

    base = with_v(1.0, 0.0)
    np.testing.assert_allclose(with_v(2.0, 0.0), 2 * base, rtol=1e-12, atol=1e-13)
    # (scalings by 2 and -1 are exact in FP32 storage; a shift would round)
    np.testing.assert_allclose(with_v(-1.0, 0.0), -base, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("dtype,tdt,nbits", [
    ("e4m3", torch.float8_e4m3fn, 8), ("e5m2", torch.float8_e5m2, 8),
    ("f16", torch.float16, 16), ("bf16", torch.bfloat16, 16)])
def test_codec_matches_library_cast(dtype, tdt, nbits):
    codes = np.arange(1 << nbits, dtype=np.int64)
    if nbits == 8:
        t = torch.from_numpy(codes.astype(np.uint8)).view(tdt)
    else:
        t = torch.from_numpy(codes.astype(np.uint16).view(np.int16)).view(tdt)
    want = t.to(torch.float64).numpy()
    got = np.array([orc.decode(dtype, int(c)) for c in codes])
    nan = np.isnan(want)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(want[~nan], got[~nan])


def test_codec_fp32_roundtrip():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(1000).astype(np.float32)
    got = np.array([orc.decode("f32", int(b)) for b in x.view(np.uint32)])
    assert np.array_equal(got, x.astype(np.float64))


def test_kv_bytes_per_token_matches_readme_table():
    with open(os.path.join(GOLDEN, "kv_bytes_per_token.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) == 5
    for fmt, dt, want, scales in rows:
        assert orc.kv_bytes_per_token(dt, 16, 4, 256, bool(int(scales))) == int(want), fmt
    # 32K tokens: 4 GiB for fp32, 2 GiB for the 16-bit formats
    assert orc.kv_bytes_per_token("f32", 16, 4, 256, False) * 32768 == 4 << 30
    assert orc.kv_bytes_per_token("bf16", 16, 4, 256, False) * 32768 == 2 << 30


def test_rejects_bad_input():
    w = wl.small_case("bf16", [20], [2], n_q_heads=4, n_kv_heads=2, head_dim=8,
                      tokens_per_fragment=8, seed=1)
    bad = w.k_pages.copy(); bad[0, 1] = 10 ** 6
    with pytest.raises(orc.OracleError, match="bad page"):
        orc.attention(to_problem(w, k_pages=bad))
    with pytest.raises(orc.OracleError, match="bad mask"):   # row 0 must see itself
        orc.attention(to_problem(w, row_masks=np.array([2, 3], np.uint64)))
    with pytest.raises(orc.OracleError, match="bad mask"):   # row 0 may not see row 1
        orc.attention(to_problem(w, row_masks=np.array([3, 3], np.uint64)))


@pytest.mark.parametrize("dtype", ["f32", "bf16", "e4m3"])
def test_long_query_block_matches_library_sdpa(dtype):
    # a prefill-style block of more than 64 chained rows (no masks): row r
    # sees the context and positions up to its own
    w = wl.small_case(dtype, [300, 90], [150, 70], n_q_heads=4, n_kv_heads=2, head_dim=16,
                      tokens_per_fragment=16, seed=21)
    assert w.row_masks is None and w.max_rows > 64
    out, lse = orc.attention(to_problem(w))
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    np.testing.assert_allclose(out, sdpa_reference(w), rtol=1e-12, atol=1e-13)


def test_long_query_block_in_256_key_windows_equals_unsplit():
    # cutting the keys into 256-key windows (the windows past a row's own
    # position are empty for it and drop out of the merge) changes nothing
    w = wl.small_case("bf16", [700, 300], [200, 100], n_q_heads=4, n_kv_heads=2, head_dim=16,
                      tokens_per_fragment=16, seed=22)
    a = orc.attention(to_problem(w))
    for kp in (256, 64):
        b_ = orc.attention_split(to_problem(w), kp)
        np.testing.assert_allclose(b_[0], a[0], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(b_[1], a[1], rtol=1e-12, atol=1e-13)


def test_masked_rows_stay_limited_to_64():
    w = wl.small_case("bf16", [100], [70], n_q_heads=2, n_kv_heads=1, head_dim=8,
                      tokens_per_fragment=16, seed=23)
    masks = np.array([(1 << min(r + 1, 64)) - 1 for r in range(70)], dtype=np.uint64)
    with pytest.raises(orc.OracleError):
        orc.attention(to_problem(w, row_masks=masks))
