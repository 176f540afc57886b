"""Host-side checks of the C ABI that need no GPU: the library loads and
exports every declared entry point; arena bookkeeping; the split rule; plan
shapes and argument checks; validation of host copies of the inputs."""
import ctypes

import numpy as np
import pytest

from verify_attention_paged_b200 import binding as b
from verify_attention_paged_b200 import workloads as wl

B200 = dict(n_sms=148, smem_optin=232448, ctas_per_sm=2)
FAKE = 1 << 32  # 256-byte-aligned stand-in device address (never dereferenced here)


def test_library_exports_every_declared_symbol():
    declared = b.declared_symbols()
    assert len(declared) >= 17
    for name in declared:
        assert hasattr(b._lib, name), name
        assert hasattr(b, name), f"binding lacks {name}"


def test_status_strings():
    assert b.lse_status_string(0) == "ok"
    assert "fragments" in b.lse_status_string(3)


def test_arena_alloc_free_lowest_first_and_growth():
    a = b.lse_kv_arena_create([FAKE], 1 << 20, 256 << 10, "bf16", 4, 128)
    info = b.lse_kv_arena_query(a)
    assert info["tokens_per_fragment"] == 256 and info["n_fragments"] == 4
    ids = b.lse_kv_arena_alloc(a, 3)
    assert list(ids) == [0, 1, 2]
    b.lse_kv_arena_free(a, [1])
    assert list(b.lse_kv_arena_alloc(a, 1)) == [1]          # free slot reused first
    with pytest.raises(b.LseError, match="out of fragments"):
        b.lse_kv_arena_alloc(a, 2)                           # only 1 free
    assert b.lse_kv_arena_query(a)["n_free"] == 1            # nothing taken
    first = b.lse_kv_arena_add_chunk(a, FAKE * 2)            # grow without moving
    assert first == 4
    assert list(b.lse_kv_arena_alloc(a, 2)) == [3, 4]
    info = b.lse_kv_arena_query(a)
    assert info["n_chunks"] == 2 and info["n_free"] == 3 and info["n_empty_chunks"] == 0
    b.lse_kv_arena_free(a, [4])
    assert b.lse_kv_arena_query(a)["n_empty_chunks"] == 1    # second chunk releasable
    with pytest.raises(b.LseError, match="not in use"):
        b.lse_kv_arena_free(a, [4])                          # double free
    with pytest.raises(b.LseError, match="twice"):
        b.lse_kv_arena_free(a, [0, 0])
    assert b.lse_kv_arena_query(a)["n_free"] == 4            # failed frees took nothing
    b.lse_kv_arena_destroy(a)


@pytest.mark.parametrize("args,msg", [
    (([FAKE], 1 << 20, 256 << 10, "bf16", 4, 96), "head_dim"),
    (([FAKE], 1 << 20, 1000, "bf16", 4, 128), "fragment_bytes"),
    (([FAKE], (1 << 20) + 5, 256 << 10, "bf16", 4, 128), "chunk_bytes"),
    (([FAKE + 16], 1 << 20, 256 << 10, "bf16", 4, 128), "aligned"),
    (([FAKE], 1 << 20, 256 << 10, 9, 4, 128), "dtype"),
])
def test_arena_rejects_bad_arguments(args, msg):
    with pytest.raises(b.LseError, match=msg):
        b.lse_kv_arena_create(*args)


def test_split_rule():
    # one full sequence of 33024 keys, 4 kv heads, 148 SMs x 2 CTAs, tile 128
    n, kp = b.lse_attn_split_rule(33024, 4, 148, 2, 128)
    assert kp % 128 == 0 and n == -(-33024 // kp)
    assert n * 4 <= 2 * 148 + 4 * 2   # about one wave of resident CTAs at full capacity
    # never smaller than a tile, never larger than the (rounded) capacity
    assert b.lse_attn_split_rule(100, 1, 148, 8, 128) == (1, 128)
    assert b.lse_attn_split_rule(10 ** 6 + 1, 1000, 1, 1, 64) == (1, 10 ** 6 // 64 * 64 + 64)
    assert b.lse_attn_split_rule(0, 1, 1, 1, 1)[0] == 0


def _plan_for(w, **lim):
    a = b.lse_kv_arena_create([FAKE * (i + 1) for i in range(len(w.chunks))], w.chunk_bytes,
                              w.fragment_bytes, w.dtype, w.n_kv_heads, w.head_dim)
    p, ws = b.lse_attn_plan_ex(a, w.n_seqs, w.max_rows, w.total_rows, w.n_q_heads,
                               w.max_pages, **(lim or B200))
    return a, p, ws


def test_plan_depends_on_capacity_not_live_lengths():
    w1 = wl.small_case("bf16", [40, 9], [1, 1], max_pages=64, tokens_per_fragment=16)
    w2 = wl.small_case("bf16", [1000, 3], [1, 1], max_pages=64, tokens_per_fragment=16)
    i1 = b.lse_attn_plan_query(_plan_for(w1)[1])
    i2 = b.lse_attn_plan_query(_plan_for(w2)[1])
    assert (i1["n_splits"], i1["keys_per_split"]) == (i2["n_splits"], i2["keys_per_split"])
    cap = 64 * 16
    assert i1["n_splits"] == -(-cap // i1["keys_per_split"])


def test_plan_workspace_size():
    w = wl.small_case("f16", [100, 50, 7], [4, 2, 1], n_q_heads=8, n_kv_heads=2,
                      head_dim=128, max_pages=20)
    _, p, ws = _plan_for(w)
    info = b.lse_attn_plan_query(p)
    n = w.total_rows * 8 * info["n_splits"]
    assert ws >= 256 + n * 128 * 4 + n * 4 and ws % 256 == 0
    assert info["workspace_bytes"] == ws and info["pairs"] == 4 * 4


def test_merge_in_pass_reports_one_launch_plans():
    # lse_attn_forward is one launch (the merge inside the partial pass) on
    # tensor-core plans, a partial launch and a merge launch on CUDA-core ones
    tiny = wl.tiny_decode()
    i_tiny = b.lse_attn_plan_query(_plan_for(tiny)[1])
    assert i_tiny["kernel_name"] == "cuda_core" and i_tiny["merge_in_pass"] == 0
    tc = wl.small_case("bf16", [700], [4], n_q_heads=24, n_kv_heads=4, head_dim=128,
                       tokens_per_fragment=128)
    i_tc = b.lse_attn_plan_query(_plan_for(tc)[1])
    assert i_tc["kernel_name"] == "tcgen05" and i_tc["merge_in_pass"] == 1


def test_plan_rejects_bad_shapes():
    a = b.lse_kv_arena_create([FAKE], 1 << 20, 256 << 10, "bf16", 4, 128)
    for args in [(1, 40000, 40000, 24, 10), (1, 0, 1, 24, 10), (1, 1, 1, 22, 10),
                 (0, 1, 1, 24, 10), (2, 4, 9, 24, 10)]:
        with pytest.raises(b.LseError):
            b.lse_attn_plan_ex(a, *args, **B200)


def test_validate_accepts_generated_workloads_and_flags_faults():
    w = wl.small_case("e4m3", [70, 33, 8], [2, 4, 1], n_q_heads=6, n_kv_heads=3, head_dim=64,
                      tokens_per_fragment=8, tree=True, seed=4)
    _, p, _ = _plan_for(w)
    b.lse_attn_validate(p, w.k_pages, w.v_pages, w.seq_lens, w.row_offsets, w.row_masks)
    bad = w.k_pages.copy(); bad[1, 2] = 10 ** 6
    with pytest.raises(b.LseError, match="unknown"):
        b.lse_attn_validate(p, bad, w.v_pages, w.seq_lens, w.row_offsets, w.row_masks)
    m = w.row_masks.copy(); m[0] = 2
    with pytest.raises(b.LseError, match="misses itself"):
        b.lse_attn_validate(p, w.k_pages, w.v_pages, w.seq_lens, w.row_offsets, m)
    m = w.row_masks.copy(); m[2] = 0b11
    with pytest.raises(b.LseError, match="later row"):
        b.lse_attn_validate(p, w.k_pages, w.v_pages, w.seq_lens, w.row_offsets, m)
    lens = w.seq_lens.copy(); lens[0] = 10 ** 5
    with pytest.raises(b.LseError, match="capacity"):
        b.lse_attn_validate(p, w.k_pages, w.v_pages, lens, w.row_offsets, w.row_masks)
    lens = w.seq_lens.copy(); lens[2] = 0
    with pytest.raises(b.LseError, match="rows"):
        b.lse_attn_validate(p, w.k_pages, w.v_pages, lens, w.row_offsets, w.row_masks)


def test_run_rejects_null_pointers_without_launching():
    w = wl.small_case("bf16", [10], [1])
    _, p, _ = _plan_for(w)
    with pytest.raises(b.LseError, match="NULL"):
        b.lse_attn_run(p, 0, 0, 0, 0, 0, None, 0.1, 0)
    with pytest.raises(b.LseError, match="aligned"):
        b.lse_attn_run(p, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.1, FAKE + 8)
    with pytest.raises(b.LseError, match="finite"):
        b.lse_attn_run(p, FAKE, FAKE, FAKE, FAKE, FAKE, None, float("nan"), FAKE)


def test_per_vector_scales_attach_and_plan():
    a = b.lse_kv_arena_create([FAKE], 1 << 20, 256 << 10, "e4m3", 4, 128)  # T = 512, 4 frags
    need = 4 * 4 * 512
    with pytest.raises(b.LseError, match="need"):
        b.lse_kv_arena_set_scales(a, FAKE, need - 1)
    with pytest.raises(b.LseError, match="aligned"):
        b.lse_kv_arena_set_scales(a, FAKE + 4, need)
    b.lse_kv_arena_set_scales(a, FAKE, need)
    args = (a, 1, 4, 4, 24, 4, 148, 232448)
    p, _ = b.lse_attn_plan_ex(*args)
    info = b.lse_attn_plan_query(p)
    assert info["scaled"] == 1 and info["kernel_name"] == "tcgen05"
    b.lse_kv_arena_set_scales(a, None)
    p0, _ = b.lse_attn_plan_ex(*args)
    info0 = b.lse_attn_plan_query(p0)
    assert info0["scaled"] == 0
    # the scale rows take shared memory from the same ring
    slots = lambda i: i["stages"] + i["v_stages"]  # noqa: E731  (K and V ring slots)
    assert info["smem_bytes"] > info0["smem_bytes"] or slots(info) < slots(info0)
    # a plan runs only on an arena in the state it was made for (checked
    # before any launch)
    with pytest.raises(b.LseError, match="scales"):
        b.lse_attn_run(p, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.1, FAKE)
    b.lse_kv_arena_set_scales(a, FAKE, need)
    with pytest.raises(b.LseError, match="scales"):
        b.lse_attn_run(p0, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.1, FAKE)
    # growth past the scale array is refused at run time
    b.lse_kv_arena_add_chunk(a, FAKE * 2)
    with pytest.raises(b.LseError, match="grew"):
        b.lse_attn_run(p, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.1, FAKE)
    b.lse_attn_plan_destroy(p)
    b.lse_attn_plan_destroy(p0)
    b.lse_kv_arena_destroy(a)


def test_per_vector_scales_only_for_8_bit_arenas():
    a = b.lse_kv_arena_create([FAKE], 1 << 20, 256 << 10, "bf16", 4, 128)
    with pytest.raises(b.LseError, match="8-bit"):
        b.lse_kv_arena_set_scales(a, FAKE, 1 << 20)
    b.lse_kv_arena_destroy(a)


def test_scaled_arena_bytes_per_token_match_the_readme_table():
    # the README's table: fp8/bf8 "with scales" take 33,280 bytes per token
    # for 16 KV layers of four kv heads of 256 dims (K and V).  The library's
    # layout: T tokens of elements per fragment plus the smallest scale array
    # it accepts (one FP32 per token and kv head of each fragment)
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "kv_bytes_per_token.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    want = {r[1]: int(r[2]) for r in rows}
    for dtype in ("e4m3", "e5m2"):
        frag = 256 << 10
        a = b.lse_kv_arena_create([FAKE], 4 * frag, frag, dtype, 4, 256)
        info = b.lse_kv_arena_query(a)
        T, n_frag = info["tokens_per_fragment"], info["n_fragments"]
        need = None
        for n in range(n_frag * 4 * T - 2, n_frag * 4 * T + 2):
            try:
                b.lse_kv_arena_set_scales(a, FAKE, n)
                need = n
                break
            except b.LseError:
                pass
        assert need is not None
        per_token_one_tensor = (frag + need * 4 // n_frag) / T
        assert 16 * 2 * per_token_one_tensor == want[dtype]
        b.lse_kv_arena_destroy(a)


def test_append_argument_checks_without_launching():
    a = b.lse_kv_arena_create([FAKE], 1 << 20, 256 << 10, "e4m3", 4, 128)
    F = FAKE
    with pytest.raises(b.LseError, match="NULL"):
        b.lse_kv_append(a, 1, 4, F, F, 0, F, F, F, 3)
    with pytest.raises(b.LseError, match="n_seqs"):
        b.lse_kv_append(a, 0, 4, F, F, F, F, F, F, 3)
    b.lse_kv_append(a, 1, 4, 0, 0, F, F, F, F, 0)   # nothing to write: no launch, ok
    # a scaled arena that grew past its scale array is refused before launch
    b.lse_kv_arena_set_scales(a, F, 4 * 4 * 512)
    b.lse_kv_arena_add_chunk(a, F * 2)
    with pytest.raises(b.LseError, match="grew"):
        b.lse_kv_append(a, 1, 4, F, F, F, F, F, F, 3)
    b.lse_kv_arena_destroy(a)


@pytest.mark.parametrize("dtype,scaled", [("f16", False), ("bf16", False), ("e4m3", False),
                                          ("e5m2", False), ("e4m3", True), ("e5m2", True)])
def test_planner_sweep_stays_within_device_limits(dtype, scaled):
    # every (group size, rows) the tensor-core kernel takes: a plan that fits
    # the B200's shared memory, a ring of 2-6 stages, row chunks of at most
    # 48 pairs; scaled plans only for the 8-bit formats
    esize = 1 if dtype.startswith("e") else 2
    for T in (8, 16, 64, 128, 512):
        frag = T * 4 * 128 * esize
        a = b.lse_kv_arena_create([FAKE], frag * 8, frag, dtype, 4, 128)
        if scaled:
            b.lse_kv_arena_set_scales(a, FAKE, 8 * 4 * T)
        for hq in (4, 8, 24, 48):
            G = hq // 4
            for rows in (1, 2, 3, 4, 5, 8, 9, 16, 33, 64):
                p, _ = b.lse_attn_plan_ex(a, 2, rows, 2 * rows, hq, 16, **B200)
                info = b.lse_attn_plan_query(p)
                assert info["kernel_name"] == "tcgen05", (dtype, T, hq, rows)
                assert info["smem_bytes"] <= B200["smem_optin"]
                assert 2 <= info["stages"] <= 6 and info["q_slots"] in (1, 2)
                assert info["scaled"] == int(scaled)
                rc = info["rows_per_chunk"]
                assert 1 <= rc <= rows and G * rc <= max(48, G)
                if G * rows <= 48:
                    assert rc == rows
                b.lse_attn_plan_destroy(p)
        b.lse_kv_arena_destroy(a)


@pytest.mark.parametrize("n_chunks", [1, 16, 17, 64])
def test_tensor_core_plan_for_arenas_of_any_chunk_count(n_chunks):
    # every chunk an arena can have gets its TMA descriptor: the planner
    # keeps the tensor-core kernel however many chunks there are, and an
    # arena grown after planning stays within the kernel's reach
    frag = 256 << 10
    a = b.lse_kv_arena_create([FAKE * (i + 1) for i in range(n_chunks)], frag * 4, frag,
                              "bf16", 4, 128)
    p, _ = b.lse_attn_plan_ex(a, 8, 1, 8, 24, 64, **B200, allow_tcgen05=1)
    assert b.lse_attn_plan_query(p)["kernel_name"] == "tcgen05"
    while b.lse_kv_arena_query(a)["n_chunks"] < 64:
        b.lse_kv_arena_add_chunk(a, FAKE * 100)
    with pytest.raises(b.LseError, match="64 chunks"):
        b.lse_kv_arena_add_chunk(a, FAKE * 100)
    b.lse_attn_plan_destroy(p)
    b.lse_kv_arena_destroy(a)


def test_tma_chunk_limit_is_every_chunk_an_arena_can_have():
    text = open(b.HEADER_PATH).read()
    import re
    lim = {k: int(v) for k, v in re.findall(r"#define (LSE_MAX_\w*CHUNKS) (\d+)", text)}
    assert lim["LSE_MAX_TMA_CHUNKS"] == lim["LSE_MAX_CHUNKS"]


def test_long_query_block_plans():
    # more than 64 rows per sequence: the rows-as-M tensor-core pass, for
    # 16-bit and FP8 arenas at head_dim 128; refused (with the reason)
    # elsewhere; it runs through lse_attn_forward only, without masks
    a = b.lse_kv_arena_create([FAKE], 1 << 28, 256 << 10, "bf16", 4, 128)
    p, ws = b.lse_attn_plan_ex(a, 2, 1024, 2048, 24, 64, **B200)
    info = b.lse_attn_plan_query(p)
    assert info["kernel_name"] == "prefill" and info["rows_per_chunk"] == 128
    assert info["smem_bytes"] <= B200["smem_optin"] and 2 <= info["stages"] <= 6
    assert ws >= 148 * 2 * 128 * 129 * 4
    F = FAKE
    with pytest.raises(b.LseError, match="lse_attn_forward"):
        b.lse_attn_run(p, F, F, F, F, F, None, 0.1, F)       # refused before any launch
    with pytest.raises(b.LseError, match="lse_attn_forward"):
        b.lse_attn_merge(p, F, F, F, F)
    with pytest.raises(b.LseError, match="row masks"):
        b.lse_attn_forward(p, F, F, F, F, F, F, 0.1, F, F)
    lens = np.array([1000, 70], np.int32)
    offs = np.array([0, 900, 970], np.int32)
    pages = np.zeros((2, 64), np.int32)
    b.lse_attn_validate(p, pages, pages, lens, offs)
    masks = np.full(970, 1, np.uint64)
    with pytest.raises(b.LseError, match="masks take at most 64"):
        b.lse_attn_validate(p, pages, pages, lens, offs, masks)
    b.lse_attn_plan_destroy(p)
    with pytest.raises(b.LseError, match="tcgen05"):
        b.lse_attn_plan_ex(a, 1, 100, 100, 24, 64, **{**B200, "allow_tcgen05": 0})
    b.lse_kv_arena_destroy(a)
    f = b.lse_kv_arena_create([FAKE], 1 << 20, 64 << 10, "f32", 1, 128)
    with pytest.raises(b.LseError, match="16-bit or FP8"):
        b.lse_attn_plan_ex(f, 1, 100, 100, 8, 64, **B200)
    b.lse_kv_arena_destroy(f)


def test_benchmark_plans_keep_their_ring_depth():
    # the shared-memory budget of the tensor-core pass: the benchmark
    # workloads keep the K/V ring depth that their throughput depends on
    # (K and V tile slots together)
    want = {"batched_decode": 6, "chain_verify": 4, "long_fp8": 10, "tree_verify": 4,
            "long_e5m2": 10}
    for name, slots in want.items():
        w = wl.BUILDERS[name]()
        a, p, _ = _plan_for(w, n_sms=148, smem_optin=232448, ctas_per_sm=0, allow_tcgen05=1)
        info = b.lse_attn_plan_query(p)
        assert info["kernel_name"] == "tcgen05", name
        assert info["stages"] + info["v_stages"] >= slots, (name, info)
        assert 2 <= info["stages"] <= info["v_stages"] <= 8
        b.lse_attn_plan_destroy(p)
        b.lse_kv_arena_destroy(a)
