"""Seeded synthetic inputs for paged decode / verification attention.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic.  Both the CUDA path's tests and the oracle's tests take
their inputs from here, and it imports neither of them.

Layout it produces (the fragment-addressed cache of the LSE releases page,
v0.4.20 "K/V memory management and automatic split attention"):

* the arena is ``n_chunks`` chunks of ``chunk_bytes`` each, cut into
  fragments of ``fragment_bytes``; fragment id ``f`` lives in chunk
  ``f // (chunk_bytes // fragment_bytes)``;
* a fragment holds ``T`` consecutive tokens of K (or of V) for every kv head,
  token-major: ``[token][kv_head][dim]``;
* sequence ``s`` reaches key ``j`` through ``k_pages[s, j // T]`` (and
  ``v_pages`` for V); K and V use separate fragments;
* fragments are handed out in a shuffled order; unused page-table entries
  hold -1; every byte of the arena not holding a live key is 0xFF, which is
  NaN in all five storage formats, so any read of a dead slot shows up.

The five named workloads follow the benchmark configurations of the
specification: tiny FP32 decode, batched BF16 decode, BF16 chain verify,
long-context FP8 (E4M3) and a mixed FP16 tree-verify batch.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

TORCH_DTYPES = {
    "f32": torch.float32,
    "f16": torch.float16,
    "bf16": torch.bfloat16,
    "e4m3": torch.float8_e4m3fn,
    "e5m2": torch.float8_e5m2,
}
ELEM_SIZE = {"f32": 4, "f16": 2, "bf16": 2, "e4m3": 1, "e5m2": 1}
DEAD_BYTE = 0xFF


@dataclass
class Workload:
    name: str
    dtype: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    fragment_bytes: int
    chunk_bytes: int
    chunks: list                 # list of np.uint8 arrays (host arena)
    k_pages: np.ndarray          # int32 [S, max_pages]
    v_pages: np.ndarray          # int32 [S, max_pages]
    seq_lens: np.ndarray         # int32 [S]
    row_offsets: np.ndarray      # int32 [S + 1]
    row_masks: np.ndarray | None  # uint64 [total_rows]; None means chain
    q: np.ndarray                # float32 [total_rows, Hq, D]
    scale: float
    seed: int
    logical_k: list = field(default_factory=list)  # per seq torch [L, Hkv, D] storage dtype
    logical_v: list = field(default_factory=list)
    parents: list = field(default_factory=list)    # per seq list of draft parents (-1 = root)
    # per-vector FP32 scales, a block of T * Hkv per fragment id ([kv_head]
    # [token] inside it; NaN where no live vector); None means unit scales
    scales: np.ndarray | None = None
    logical_k_scale: list = field(default_factory=list)  # per seq float32 [L, Hkv]
    logical_v_scale: list = field(default_factory=list)
    # scaled: the FP32 vectors before they were divided by their scales
    logical_k_src: list = field(default_factory=list)    # per seq float32 [L, Hkv, D]
    logical_v_src: list = field(default_factory=list)

    @property
    def n_seqs(self) -> int:
        return int(len(self.seq_lens))

    @property
    def max_pages(self) -> int:
        return int(self.k_pages.shape[1])

    @property
    def tokens_per_fragment(self) -> int:
        return self.fragment_bytes // (self.n_kv_heads * self.head_dim * ELEM_SIZE[self.dtype])

    @property
    def total_rows(self) -> int:
        return int(self.row_offsets[-1])

    @property
    def max_rows(self) -> int:
        return int(np.max(np.diff(self.row_offsets))) if self.n_seqs else 0

    def kv_bytes(self) -> int:
        """Bytes of live K and V (every key of every sequence, all kv heads),
        their per-vector scales included."""
        per_vec = self.head_dim * ELEM_SIZE[self.dtype] + (4 if self.scales is not None else 0)
        return int(np.sum(self.seq_lens.astype(np.int64))) * 2 * self.n_kv_heads * per_vec

    def call_bytes(self) -> int:
        """K + V + Q + out bytes of one call (Q and out in FP32)."""
        qo = 2 * self.total_rows * self.n_q_heads * self.head_dim * 4
        return self.kv_bytes() + qo


def _chain_masks(R: int) -> list[int]:
    return [(1 << (r + 1)) - 1 for r in range(R)]


def _tree_masks(parents: list[int]) -> list[int]:
    """Self + ancestors bit masks for a topologically ordered parent list."""
    masks = []
    for i, p in enumerate(parents):
        m = 1 << i
        if p >= 0:
            m |= masks[p]
        masks.append(m)
    return masks


def build(
    name: str,
    dtype: str,
    seq_lens: list[int],
    rows: list[int],
    n_q_heads: int,
    n_kv_heads: int,
    head_dim: int,
    fragment_bytes: int,
    chunk_bytes: int,
    max_pages: int,
    seed: int,
    parents: list[list[int]] | None = None,
    kv_std: float = 1.0,
    q_std: float = 1.0,
    keep_logical: bool = False,
    n_chunks: int | None = None,
    gen: torch.Generator | None = None,
    scaled: bool = False,
    scale_spread: float = 0.0,
    magnitude_spread: float = 0.0,
) -> Workload:
    """Lay out one seeded problem.

    ``rows[s]`` query rows are the last positions of sequence ``s``;
    ``parents[s]`` (optional) gives each draft row's parent row, -1 for a row
    hanging off the cached context; without it the rows form a chain.

    ``scaled`` (8-bit formats) stores every K and V vector with a per-vector
    FP32 scale, amax / (largest finite value of the format), the stored
    elements being the vector divided by it and cast.  ``magnitude_spread``
    first multiplies each vector by 2^u, u uniform in [-spread, spread] (the
    vectors' sizes vary, and their scales with them); ``scale_spread``
    multiplies each scale by 2^u, u uniform in [0, spread] (the scales vary
    over that many binades while the vectors they give back do not: the
    stored elements shrink by the same factor, never past the format's
    largest value).
    """
    g = gen if gen is not None else torch.Generator().manual_seed(seed)
    es = ELEM_SIZE[dtype]
    row_bytes = n_kv_heads * head_dim * es
    assert fragment_bytes % row_bytes == 0 and chunk_bytes % fragment_bytes == 0
    T = fragment_bytes // row_bytes
    fpc = chunk_bytes // fragment_bytes
    S = len(seq_lens)
    pages_needed = [math.ceil(L / T) for L in seq_lens]
    assert all(p <= max_pages for p in pages_needed)
    need = 2 * sum(pages_needed)
    if n_chunks is None:
        n_chunks = max(1, math.ceil(need / fpc))
    assert need <= n_chunks * fpc, "arena too small"

    # shuffled fragment assignment
    perm = torch.randperm(n_chunks * fpc, generator=g)[:need].to(torch.int64).numpy()
    k_pages = np.full((S, max_pages), -1, np.int32)
    v_pages = np.full((S, max_pages), -1, np.int32)
    cursor = 0
    for s in range(S):
        n = pages_needed[s]
        k_pages[s, :n] = perm[cursor:cursor + n]
        v_pages[s, :n] = perm[cursor + n:cursor + 2 * n]
        cursor += 2 * n

    row_offsets = np.zeros(S + 1, np.int32)
    row_offsets[1:] = np.cumsum(rows)
    masks: list[int] = []
    for s in range(S):
        if parents is not None:
            assert len(parents[s]) == rows[s]
            masks += _tree_masks(parents[s])
        else:
            masks += _chain_masks(rows[s])
    row_masks = np.array(masks, dtype=np.uint64) if parents is not None else None

    total_rows = int(row_offsets[-1])
    q = (torch.randn((total_rows, n_q_heads, head_dim), generator=g, dtype=torch.float32)
         * q_std).numpy()

    chunks = [np.full(chunk_bytes, DEAD_BYTE, np.uint8) for _ in range(n_chunks)]
    tdt = TORCH_DTYPES[dtype]
    assert not scaled or es == 1, "per-vector scales go with the 8-bit formats"
    scales = np.full(n_chunks * fpc * n_kv_heads * T, np.nan, np.float32) if scaled else None
    logical_k, logical_v = [], []
    logical_ks, logical_vs = [], []
    src_k, src_v = [], []
    for s in range(S):
        L = seq_lens[s]
        for which, table in (("k", k_pages), ("v", v_pages)):
            x = torch.randn((L, n_kv_heads, head_dim), generator=g, dtype=torch.float32)
            x = x * kv_std
            if scaled:
                if magnitude_spread > 0:
                    u = (torch.rand((L, n_kv_heads, 1), generator=g) * 2 - 1) * magnitude_spread
                    x = x * torch.exp2(u)
                if keep_logical:
                    (src_k if which == "k" else src_v).append(x.clone())
                sc = x.abs().amax(dim=2) / torch.finfo(tdt).max      # [L, Hkv]
                if scale_spread > 0:
                    sc = sc * torch.exp2(torch.rand((L, n_kv_heads), generator=g) * scale_spread)
                sc = torch.where(sc > 0, sc, torch.ones_like(sc))
                x = x / sc[:, :, None]
                sc = sc.numpy()
                if keep_logical:
                    (logical_ks if which == "k" else logical_vs).append(sc)
            x = x.to(tdt)
            if keep_logical:
                (logical_k if which == "k" else logical_v).append(x)
            raw = x.contiguous().view(torch.uint8).reshape(L, row_bytes).numpy()
            for p in range(pages_needed[s]):
                f = int(table[s, p])
                c, off = divmod(f, fpc)
                t0, t1 = p * T, min((p + 1) * T, L)
                base = off * fragment_bytes
                chunks[c][base:base + (t1 - t0) * row_bytes] = raw[t0:t1].reshape(-1)
                if scaled:
                    blk = scales[f * n_kv_heads * T:(f + 1) * n_kv_heads * T].reshape(n_kv_heads, T)
                    blk[:, :t1 - t0] = sc[t0:t1].T

    return Workload(
        name=name, dtype=dtype, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads, head_dim=head_dim,
        fragment_bytes=fragment_bytes, chunk_bytes=chunk_bytes, chunks=chunks,
        k_pages=k_pages, v_pages=v_pages, seq_lens=np.array(seq_lens, np.int32),
        row_offsets=row_offsets, row_masks=row_masks, q=q, scale=1.0 / math.sqrt(head_dim),
        seed=seed, logical_k=logical_k, logical_v=logical_v,
        parents=parents if parents is not None else [], scales=scales,
        logical_k_scale=logical_ks, logical_v_scale=logical_vs, logical_k_src=src_k,
        logical_v_src=src_v)


# ---------------------------------------------------------------------------
# The five benchmark workloads.  Seed = 1234 + index (index 0..4).
# ---------------------------------------------------------------------------

MIB = 1 << 20
KIB = 1 << 10
NAMES = ["tiny_decode", "batched_decode", "chain_verify", "long_fp8", "tree_verify"]


def tiny_decode(keep_logical=False) -> Workload:
    """1 sequence, 1 query row, 4 query heads / 1 kv head, head_dim 64, 512
    keys, FP32 K/V in 16-token pages in random order."""
    return build("tiny_decode", "f32", [512], [1], 4, 1, 64, fragment_bytes=16 * 64 * 4,
                 chunk_bytes=1 * MIB, max_pages=32, seed=1234, keep_logical=keep_logical)


def batched_decode(keep_logical=False) -> Workload:
    """8 sequences, lengths uniform in [1024, 16384], 1 row each, 24/4 heads,
    head_dim 128, BF16 K/V in 256 KiB fragments of one 256 MiB arena."""
    g = torch.Generator().manual_seed(1235)
    lens = torch.randint(1024, 16385, (8,), generator=g).tolist()
    return build("batched_decode", "bf16", lens, [1] * 8, 24, 4, 128,
                 fragment_bytes=256 * KIB, chunk_bytes=256 * MIB, max_pages=64, seed=1235,
                 n_chunks=1, gen=g, keep_logical=keep_logical)


def chain_verify(keep_logical=False) -> Workload:
    """1 sequence, 32768 cached keys + 8 chained draft rows, 24/4 heads,
    head_dim 128, BF16 in 256 KiB fragments."""
    return build("chain_verify", "bf16", [32768 + 8], [8], 24, 4, 128,
                 fragment_bytes=256 * KIB, chunk_bytes=256 * MIB, max_pages=129, seed=1236,
                 n_chunks=1, keep_logical=keep_logical)


def long_fp8(keep_logical=False) -> Workload:
    """1 sequence, 68173 keys (4 chained query rows included), 24/4 heads,
    head_dim 128, FP8 E4M3 cast from N(0, 0.5^2), 512-token fragments;
    capacity 256 pages (131072 keys)."""
    return build("long_fp8", "e4m3", [68173], [4], 24, 4, 128, fragment_bytes=512 * 4 * 128,
                 chunk_bytes=256 * MIB, max_pages=256, seed=1237, kv_std=0.5, n_chunks=1,
                 keep_logical=keep_logical)


def tree_verify(keep_logical=False) -> Workload:
    """16 sequences, context log-uniform in [256, 131072], each with a random
    draft tree of 1..16 nodes, 24/4 heads, head_dim 128, FP16 in 256 KiB
    fragments across several 256 MiB chunks; capacity 513 pages."""
    g = torch.Generator().manual_seed(1238)
    lo, hi = math.log(256), math.log(131072)
    ctx = [int(math.exp(lo + (hi - lo) * float(u)))
           for u in torch.rand(16, generator=g, dtype=torch.float64)]
    nodes = torch.randint(1, 17, (16,), generator=g).tolist()
    parents = []
    for n in nodes:
        parents.append([int(torch.randint(-1, i, (1,), generator=g)) for i in range(n)])
    lens = [c + n for c, n in zip(ctx, nodes)]
    return build("tree_verify", "f16", lens, nodes, 24, 4, 128, fragment_bytes=256 * KIB,
                 chunk_bytes=256 * MIB, max_pages=513, seed=1238, parents=parents, gen=g,
                 keep_logical=keep_logical)


def long_e5m2(keep_logical=False) -> Workload:
    """The long-context FP8 workload with E5M2 storage (the releases page's
    second 8-bit format, "BF8"): 68173 keys incl. 4 chained rows, 24/4 heads,
    head_dim 128, cast from N(0, 0.5^2), 512-token fragments, capacity 256
    pages."""
    return build("long_e5m2", "e5m2", [68173], [4], 24, 4, 128, fragment_bytes=512 * 4 * 128,
                 chunk_bytes=256 * MIB, max_pages=256, seed=1239, kv_std=0.5, n_chunks=1,
                 keep_logical=keep_logical)


def long_fp8_scaled(keep_logical=False) -> Workload:
    """The long-context FP8 (E4M3) workload stored with per-vector FP32
    scales (the README's fp8 "with scales" format): each K and V vector of
    N(0, 0.5^2) values is divided by amax / 448 and cast, its scale kept in
    the fragment's scale block."""
    return build("long_fp8_scaled", "e4m3", [68173], [4], 24, 4, 128,
                 fragment_bytes=512 * 4 * 128, chunk_bytes=256 * MIB, max_pages=256, seed=1243,
                 kv_std=0.5, n_chunks=1, keep_logical=keep_logical, scaled=True)


def prefill_block(keep_logical=False) -> Workload:
    """A long query block (the releases page's prefill chunks of 1024 rows,
    v0.4.14): 1 sequence of 16384 keys whose last 1024 positions are a chain
    of query rows over 15360 cached keys, 24/4 heads, head_dim 128, BF16 in
    256 KiB fragments in shuffled order."""
    return build("prefill_block", "bf16", [16384], [1024], 24, 4, 128,
                 fragment_bytes=256 * KIB, chunk_bytes=256 * MIB, max_pages=64, seed=1244,
                 n_chunks=1, keep_logical=keep_logical)


BUILDERS = {
    "tiny_decode": tiny_decode,
    "batched_decode": batched_decode,
    "chain_verify": chain_verify,
    "long_fp8": long_fp8,
    "tree_verify": tree_verify,
    "long_e5m2": long_e5m2,
    "long_fp8_scaled": long_fp8_scaled,
    "prefill_block": prefill_block,
}
# workloads beyond the five benchmark configurations
EXTRA_NAMES = ["long_e5m2", "long_fp8_scaled", "prefill_block"]


# ---------------------------------------------------------------------------
# Fragment-addressing A/B (LSE releases, v0.4.20, "Validation and
# performance"): the same keys reached through a shuffled page table and
# through an identity one, and split against forced-unsplit attention.
# ---------------------------------------------------------------------------

def contiguous_copy(w: Workload) -> Workload:
    """The same problem with its fragments moved so that every page table is
    the identity on a contiguous run: the K pages of sequence 0, 1, ... come
    first in fragment order, then the V pages, as in an unpaged cache."""
    T = w.tokens_per_fragment
    fpc = w.chunk_bytes // w.fragment_bytes
    n_pages = [math.ceil(int(L) / T) for L in w.seq_lens]
    k_pages = np.full_like(w.k_pages, -1)
    v_pages = np.full_like(w.v_pages, -1)
    nk = sum(n_pages)
    chunks = [np.full(w.chunk_bytes, DEAD_BYTE, np.uint8) for _ in w.chunks]
    fb = w.fragment_bytes
    blk = w.n_kv_heads * T
    scales = None if w.scales is None else np.full_like(w.scales, np.nan)
    cursor = 0
    for s, n in enumerate(n_pages):
        for p in range(n):
            for old_table, new_table, new_id in ((w.k_pages, k_pages, cursor + p),
                                                 (w.v_pages, v_pages, nk + cursor + p)):
                oc, oo = divmod(int(old_table[s, p]), fpc)
                nc, no = divmod(new_id, fpc)
                chunks[nc][no * fb:(no + 1) * fb] = w.chunks[oc][oo * fb:(oo + 1) * fb]
                if scales is not None:
                    old_id = int(old_table[s, p])
                    scales[new_id * blk:(new_id + 1) * blk] = w.scales[old_id * blk:(old_id + 1) * blk]
                new_table[s, p] = new_id
        cursor += n
    return Workload(**{**w.__dict__, "name": w.name + "_contiguous", "chunks": chunks,
                       "k_pages": k_pages, "v_pages": v_pages, "scales": scales})


def fragment_ab_cases() -> list[Workload]:
    """The releases page's fragment-addressing measurements, as BF16 problems
    with 24/4 heads, head_dim 128 and 256 KiB fragments: one query row at 16K
    context; eight chained query rows at 68K (68,173 keys in total); and
    65,656 live keys with four chained query rows, the split-vs-unsplit
    check."""
    common = dict(n_q_heads=24, n_kv_heads=4, head_dim=128, fragment_bytes=256 * KIB,
                  chunk_bytes=256 * MIB)
    return [
        build("frag_16k_decode", "bf16", [16384], [1], max_pages=64, seed=1240, **common),
        build("frag_68k_8rows", "bf16", [68173], [8], max_pages=267, seed=1241, **common),
        build("split_65656_4rows", "bf16", [65656], [4], max_pages=257, seed=1242, **common),
    ]


def small_case(dtype: str, seq_lens, rows, n_q_heads=8, n_kv_heads=2, head_dim=64,
               tokens_per_fragment=16, max_pages=None, seed=7, tree=False, kv_std=1.0,
               keep_logical=True, n_chunks=None, scaled=False, scale_spread=0.0,
               magnitude_spread=0.0, frags_per_chunk=None) -> Workload:
    """A small seeded problem of any shape, for parity and pin tests.
    ``frags_per_chunk`` cuts the arena into chunks of that many fragments
    (enough chunks for every live fragment), so a problem spans many chunks."""
    g = torch.Generator().manual_seed(seed)
    es = ELEM_SIZE[dtype]
    fb = tokens_per_fragment * n_kv_heads * head_dim * es
    need = 2 * sum(math.ceil(L / tokens_per_fragment) for L in seq_lens)
    if max_pages is None:
        max_pages = max(1, max(math.ceil(L / tokens_per_fragment) for L in seq_lens))
    fpc = max(4, need) if frags_per_chunk is None else int(frags_per_chunk)
    if frags_per_chunk is not None and n_chunks is None:
        n_chunks = math.ceil(need / fpc)
    parents = None
    if tree:
        parents = [[int(torch.randint(-1, i, (1,), generator=g)) for i in range(R)] for R in rows]
    return build(f"small_{dtype}", dtype, list(seq_lens), list(rows), n_q_heads, n_kv_heads,
                 head_dim, fragment_bytes=fb, chunk_bytes=fb * fpc, max_pages=max_pages,
                 seed=seed, parents=parents, kv_std=kv_std, keep_logical=keep_logical,
                 n_chunks=n_chunks, gen=g, scaled=scaled, scale_spread=scale_spread,
                 magnitude_spread=magnitude_spread)
