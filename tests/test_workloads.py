"""The seeded input generator (CPU): page tables name distinct fragments of
the arena, every live key's bytes sit where its table says, every other
byte is the dead pattern (0xFF), per-vector scales exist exactly for live
vectors, and the same seed gives the same bytes."""
import math

import numpy as np
import pytest
import torch

from verify_attention_paged_b200 import workloads as wl


def _live_map(w):
    """Boolean per arena byte: True where a live key's K or V element sits."""
    T = w.tokens_per_fragment
    fpc = w.chunk_bytes // w.fragment_bytes
    row = w.n_kv_heads * w.head_dim * wl.ELEM_SIZE[w.dtype]
    live = [np.zeros(w.chunk_bytes, bool) for _ in w.chunks]
    for s in range(w.n_seqs):
        L = int(w.seq_lens[s])
        for p in range(math.ceil(L / T)):
            n = min(T, L - p * T)
            for table in (w.k_pages, w.v_pages):
                c, o = divmod(int(table[s, p]), fpc)
                live[c][o * w.fragment_bytes:o * w.fragment_bytes + n * row] = True
    return live


@pytest.mark.parametrize("dtype,scaled", [("f32", False), ("bf16", False), ("e4m3", True),
                                          ("e5m2", False)])
def test_tables_bytes_and_dead_pattern(dtype, scaled):
    w = wl.small_case(dtype, [37, 1, 64, 9], [2, 1, 3, 1], n_q_heads=4, n_kv_heads=2,
                      head_dim=16, tokens_per_fragment=8, seed=5, scaled=scaled)
    T = w.tokens_per_fragment
    used = np.concatenate([w.k_pages[w.k_pages >= 0], w.v_pages[w.v_pages >= 0]])
    assert len(np.unique(used)) == len(used)                  # no fragment shared
    for s in range(w.n_seqs):
        n = math.ceil(int(w.seq_lens[s]) / T)
        assert (w.k_pages[s, :n] >= 0).all() and (w.k_pages[s, n:] == -1).all()
        assert (w.v_pages[s, :n] >= 0).all() and (w.v_pages[s, n:] == -1).all()
    live = _live_map(w)
    for c, m in zip(w.chunks, live):
        assert (c[~m] == wl.DEAD_BYTE).all()
    # every live key reads back as the logical vector the generator kept
    fpc = w.chunk_bytes // w.fragment_bytes
    es = wl.ELEM_SIZE[dtype]
    row = w.n_kv_heads * w.head_dim * es
    for s in range(w.n_seqs):
        for j in range(int(w.seq_lens[s])):
            c, o = divmod(int(w.k_pages[s, j // T]), fpc)
            b = o * w.fragment_bytes + (j % T) * row
            want = w.logical_k[s][j].contiguous().view(torch.uint8).reshape(-1).numpy()
            assert np.array_equal(w.chunks[c][b:b + row], want)
    if scaled:
        Hkv = w.n_kv_heads
        has = ~np.isnan(w.scales)
        want = np.zeros_like(has)
        for s in range(w.n_seqs):
            for j in range(int(w.seq_lens[s])):
                for table in (w.k_pages, w.v_pages):
                    f = int(table[s, j // T])
                    want[f * Hkv * T + np.arange(Hkv) * T + j % T] = True
        assert np.array_equal(has, want)
        assert (w.scales[has] > 0).all()


def test_same_seed_same_bytes_and_other_seed_differs():
    a = wl.small_case("bf16", [50, 20], [1, 2], seed=9)
    b = wl.small_case("bf16", [50, 20], [1, 2], seed=9)
    c = wl.small_case("bf16", [50, 20], [1, 2], seed=10)
    assert all(np.array_equal(x, y) for x, y in zip(a.chunks, b.chunks))
    assert np.array_equal(a.q, b.q) and np.array_equal(a.k_pages, b.k_pages)
    assert not np.array_equal(a.q, c.q)


def test_fragment_ab_cases_shapes():
    cases = wl.fragment_ab_cases()
    assert [int(w.seq_lens[0]) for w in cases] == [16384, 68173, 65656]
    assert [w.total_rows for w in cases] == [1, 8, 4]
    for w in cases:
        assert w.dtype == "bf16" and w.fragment_bytes == 256 << 10
        assert w.tokens_per_fragment == 256 and (w.n_q_heads, w.n_kv_heads) == (24, 4)
