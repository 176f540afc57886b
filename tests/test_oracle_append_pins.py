"""Pins of the oracle's encoder and K/V append (CPU).

The encoder (FP32 -> stored bits) is checked against torch's casts on every
in-range value tried (nearest, ties to even, subnormals), on every code of
each format (decode then encode returns the code), and on the overflow
rules its header states (FP8 saturates, F16/BF16 go to infinity).  The
append is checked against the arena bytes the workload generator wrote with
torch's casts: rewriting a sequence's last keys from their values restores
the same bytes, and nothing else changes.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from verify_attention_paged_b200 import workloads as wl

TORCH = {"f16": torch.float16, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn,
         "e5m2": torch.float8_e5m2}
MAXV = {"f16": 65504.0, "bf16": float(torch.finfo(torch.bfloat16).max), "e4m3": 448.0,
        "e5m2": 57344.0}
# below this magnitude the nearest value is finite (half an ulp past the max)
ROUND_LIMIT = {"f16": 65520.0, "bf16": 3.3961e38, "e4m3": 464.0, "e5m2": 61440.0}


def torch_bits(dtype, x):
    t = torch.from_numpy(np.asarray(x, np.float32)).to(TORCH[dtype])
    if t.element_size() == 1:
        return t.view(torch.uint8).numpy().astype(np.int64)
    return t.view(torch.int16).numpy().astype(np.int64) & 0xFFFF


def encode_all(dtype, x):
    return np.array([orc.encode(dtype, float(v)) for v in x], np.int64)


def sample_values(dtype, n, seed):
    rng = np.random.default_rng(seed)
    # magnitudes across the format's normal and subnormal ranges
    lo = {"f16": -26, "bf16": -140, "e4m3": -11, "e5m2": -18}[dtype]
    hi = np.log2(MAXV[dtype])
    mag = np.exp2(rng.uniform(lo, hi, n))
    x = (mag * np.where(rng.random(n) < 0.5, -1.0, 1.0)).astype(np.float32)
    return x[np.abs(x) < ROUND_LIMIT[dtype]]


@pytest.mark.parametrize("dtype", sorted(TORCH))
def test_encoder_matches_torch_cast_in_range(dtype):
    x = sample_values(dtype, 30000, seed=11)
    assert np.array_equal(encode_all(dtype, x), torch_bits(dtype, x))


@pytest.mark.parametrize("dtype", sorted(TORCH))
def test_encoder_rounds_ties_to_even(dtype):
    # midpoints between adjacent codes (exact in FP32): each goes to the code
    # with the even fraction, as torch's cast does
    codes = np.arange(1, 1 << (8 if TORCH[dtype].itemsize == 1 else 16))
    vals = np.array([orc.decode(dtype, int(c)) for c in codes])
    ok = np.isfinite(vals) & (vals > 0)
    v = np.unique(vals[ok])
    mid = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    exact = mid.astype(np.float64) == (v[:-1] + v[1:]) / 2
    mid = mid[exact & (np.abs(mid) < ROUND_LIMIT[dtype])]
    assert len(mid) > 10
    got = encode_all(dtype, mid)
    assert np.array_equal(got, torch_bits(dtype, mid))
    assert np.all(got % 2 == 0)  # the even neighbour


@pytest.mark.parametrize("dtype,nbits", [("f16", 16), ("bf16", 16), ("e4m3", 8), ("e5m2", 8)])
def test_every_code_round_trips(dtype, nbits):
    for c in range(1 << nbits):
        v = orc.decode(dtype, c)
        if np.isnan(v) or (np.isinf(v) and dtype in ("e4m3", "e5m2")):
            continue  # (the 8-bit formats saturate infinities: see the overflow test)
        assert orc.encode(dtype, v) == c, (dtype, hex(c), v)


@pytest.mark.parametrize("dtype", sorted(TORCH))
def test_overflow_and_nan_rules(dtype):
    big = np.float32(ROUND_LIMIT[dtype] * (1.01 if dtype != "bf16" else 1.0001))
    if dtype == "bf16":
        big = np.float32(np.finfo(np.float32).max)
    top_pos = orc.encode(dtype, MAXV[dtype])
    top_neg = orc.encode(dtype, -MAXV[dtype])
    if dtype in ("e4m3", "e5m2"):
        # saturate at the largest finite value
        assert orc.encode(dtype, float(big)) == top_pos
        assert orc.encode(dtype, -float(big)) == top_neg
        assert orc.decode(dtype, top_pos) == MAXV[dtype]
        assert orc.encode(dtype, float("inf")) == top_pos
    elif dtype == "f16":
        assert orc.encode(dtype, float(big)) == 0x7C00
        assert orc.encode(dtype, -float(big)) == 0xFC00
        assert orc.encode(dtype, float("inf")) == 0x7C00
    # values just below the rounding limit stay finite
    below = np.nextafter(np.float32(ROUND_LIMIT[dtype]), np.float32(0))
    if dtype != "bf16":
        assert orc.encode(dtype, float(below)) == top_pos
    assert np.isnan(orc.decode(dtype, orc.encode(dtype, float("nan"))))
    assert orc.encode(dtype, -0.0) != orc.encode(dtype, 0.0)  # the sign of zero is kept


def test_f32_encoding_is_the_float_bits():
    x = np.array([0.0, -0.0, 1.5, -3.25e-40, 1e30], np.float32)
    for v in x:
        assert orc.encode("f32", float(v)) == int(np.frombuffer(v.tobytes(), np.uint32)[0])


def _append_from_logical(w, n_new):
    """Host copies of w's arena with each sequence's last n_new keys erased
    (0xFF) and rewritten through orc.kv_append from their stored values."""
    chunks = [c.copy() for c in w.chunks]
    T = w.tokens_per_fragment
    fpc = w.chunk_bytes // w.fragment_bytes
    es = wl.ELEM_SIZE[w.dtype]
    row = w.n_kv_heads * w.head_dim * es
    before, offs, ks, vs = [], [0], [], []
    for s in range(w.n_seqs):
        L = int(w.seq_lens[s])
        m = min(n_new, L)
        before.append(L - m)
        offs.append(offs[-1] + m)
        for j in range(L - m, L):
            for table in (w.k_pages, w.v_pages):
                c, off = divmod(int(table[s, j // T]), fpc)
                b = off * w.fragment_bytes + (j % T) * row
                chunks[c][b:b + row] = 0xFF
        ks.append(w.logical_k[s][L - m:L].to(torch.float32).numpy())
        vs.append(w.logical_v[s][L - m:L].to(torch.float32).numpy())
    k_new = np.concatenate(ks) if ks else np.zeros((0, w.n_kv_heads, w.head_dim), np.float32)
    v_new = np.concatenate(vs) if vs else np.zeros((0, w.n_kv_heads, w.head_dim), np.float32)
    st = orc.kv_append(chunks, w.chunk_bytes, w.fragment_bytes, w.dtype, w.n_kv_heads,
                       w.head_dim, w.k_pages, w.v_pages, np.array(before, np.int32),
                       np.array(offs, np.int32), k_new, v_new)
    return chunks, st, np.array(before, np.int32), np.array(offs, np.int32), k_new, v_new


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16", "e4m3", "e5m2"])
def test_append_restores_the_generator_bytes(dtype):
    # the generator wrote every key with torch's cast; rewriting the last
    # keys of each sequence from their values gives back the same bytes, in
    # the right fragments, and touches nothing else
    w = wl.small_case(dtype, [40, 9, 1, 33], [1, 2, 1, 3], n_q_heads=4, n_kv_heads=2,
                      head_dim=16, tokens_per_fragment=8, seed=41)
    chunks, st, *_ = _append_from_logical(w, 11)
    assert st == 0
    for a, b in zip(chunks, w.chunks):
        assert np.array_equal(a, b)


def test_append_past_the_page_table_is_reported_and_skipped():
    w = wl.small_case("bf16", [16, 8], [1, 1], n_q_heads=2, n_kv_heads=1, head_dim=8,
                      tokens_per_fragment=8, seed=42)
    chunks = [c.copy() for c in w.chunks]
    # sequence 0 appends 3 keys at 15, 16, 17: pages 1 and 2; the table has 2
    k_new = np.ones((3, 1, 8), np.float32)
    st = orc.kv_append(chunks, w.chunk_bytes, w.fragment_bytes, "bf16", 1, 8, w.k_pages,
                       w.v_pages, np.array([15, 8], np.int32), np.array([0, 3, 3], np.int32),
                       k_new, 2 * k_new)
    assert st == 2
    # key 15 was written (page 1), keys 16 and 17 were not
    fpc = w.chunk_bytes // w.fragment_bytes
    c, off = divmod(int(w.k_pages[0, 1]), fpc)
    b = off * w.fragment_bytes + 7 * 16
    assert np.array_equal(chunks[c][b:b + 16].view(np.uint16),
                          np.full(8, 0x3F80, np.uint16))  # bf16 1.0


@pytest.mark.parametrize("dtype", ["e4m3", "e5m2"])
def test_scaled_append_restores_the_generator_bytes_and_scales(dtype):
    # the generator drew per-vector scales amax / (largest finite value) and
    # stored each vector divided by its scale (FP32 division, torch's cast);
    # re-appending the last keys of each sequence from the same FP32 vectors
    # gives back the same bytes and the same scales, bit for bit
    w = wl.small_case(dtype, [40, 9, 1, 33], [1, 2, 1, 3], n_q_heads=4, n_kv_heads=2,
                      head_dim=16, tokens_per_fragment=8, seed=44, scaled=True,
                      magnitude_spread=4.0)
    chunks = [c.copy() for c in w.chunks]
    scales = w.scales.copy()
    T, Hkv = w.tokens_per_fragment, w.n_kv_heads
    fpc = w.chunk_bytes // w.fragment_bytes
    row = Hkv * w.head_dim
    n_new = 11
    before, offs, ks, vs = [], [0], [], []
    for s in range(w.n_seqs):
        L = int(w.seq_lens[s])
        m = min(n_new, L)
        before.append(L - m)
        offs.append(offs[-1] + m)
        for j in range(L - m, L):
            for table in (w.k_pages, w.v_pages):
                f = int(table[s, j // T])
                c, off = divmod(f, fpc)
                b = off * w.fragment_bytes + (j % T) * row
                chunks[c][b:b + row] = 0xFF
                scales[f * Hkv * T + np.arange(Hkv) * T + j % T] = np.nan
        ks.append(w.logical_k_src[s][L - m:L].numpy())
        vs.append(w.logical_v_src[s][L - m:L].numpy())
    st = orc.kv_append(chunks, w.chunk_bytes, w.fragment_bytes, dtype, Hkv, w.head_dim,
                       w.k_pages, w.v_pages, np.array(before, np.int32),
                       np.array(offs, np.int32), np.concatenate(ks), np.concatenate(vs),
                       scales=scales)
    assert st == 0
    for a, b in zip(chunks, w.chunks):
        assert np.array_equal(a, b)
    assert np.array_equal(scales.view(np.uint32), w.scales.view(np.uint32))


def test_scaled_append_of_a_zero_vector_uses_unit_scale():
    w = wl.small_case("e4m3", [8], [1], n_q_heads=2, n_kv_heads=1, head_dim=8,
                      tokens_per_fragment=8, seed=45, scaled=True)
    chunks = [c.copy() for c in w.chunks]
    scales = w.scales.copy()
    z = np.zeros((1, 1, 8), np.float32)
    st = orc.kv_append(chunks, w.chunk_bytes, w.fragment_bytes, "e4m3", 1, 8, w.k_pages,
                       w.v_pages, np.array([7], np.int32), np.array([0, 1], np.int32), z, z,
                       scales=scales)
    assert st == 0
    for table in (w.k_pages, w.v_pages):
        assert scales[int(table[0, 0]) * 8 + 7] == 1.0
