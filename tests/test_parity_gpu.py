"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle
on the same seeded inputs.  Every test compares every output element: the
small cases with the oracle on one thread, the full-size workloads (in the
launch configuration the benchmark times) with the oracle spread over the
host cores."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from verify_attention_paged_b200 import workloads as wl
from conftest import to_problem
from parity_util import assert_close, lse_tol, oracle_all_outputs

pytestmark = pytest.mark.gpu

DTYPES = ["f32", "f16", "bf16", "e4m3", "e5m2"]


@pytest.fixture(scope="module")
def binding():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from verify_attention_paged_b200 import binding as b
    return b


def gpu_run(b, w, **kw):
    call = b.DeviceCall(w, **kw)
    out, lse = call.run()
    torch.cuda.synchronize()
    err = call.device_error()
    res = out[:w.total_rows].cpu().numpy(), lse[:w.total_rows].cpu().numpy(), call.info
    call.close()
    return res, err


def check_full(b, w, **kw):
    (out, lse, info), err = gpu_run(b, w, **kw)
    assert err == 0, f"device error word {err:#x}"
    ref_out, ref_lse = orc.attention(to_problem(w))
    assert_close(out, ref_out, w.dtype)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=lse_tol(w.dtype) * 4)
    return info


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("tree", [False, True])
def test_small_ragged_all_formats(binding, dtype, tree):
    # lengths span many 32/128-key tiles with ragged tails; rows 1..16
    w = wl.small_case(dtype, [1, 7, 33, 300, 517, 129], [1, 1, 3, 8, 16, 5], n_q_heads=12,
                      n_kv_heads=2, head_dim=128, tokens_per_fragment=16, tree=tree, seed=101)
    check_full(binding, w)


@pytest.mark.parametrize("head_dim", [64, 128, 256])
@pytest.mark.parametrize("groups", [(4, 4), (8, 1), (24, 4)])
def test_head_dims_and_group_sizes(binding, head_dim, groups):
    hq, hkv = groups
    for dtype in ("bf16", "f32"):
        w = wl.small_case(dtype, [200, 45], [4, 2], n_q_heads=hq, n_kv_heads=hkv,
                          head_dim=head_dim, tokens_per_fragment=8, seed=102)
        check_full(binding, w)


def test_rows_at_the_limit_and_tiny_fragments(binding):
    # R = 64 draft rows (the mask limit), 1-token fragments, GQA 3
    w = wl.small_case("f16", [64, 100], [64, 33], n_q_heads=6, n_kv_heads=2, head_dim=64,
                      tokens_per_fragment=1, tree=True, seed=103)
    check_full(binding, w)


def test_idle_sequence_and_drafts_only(binding):
    # an idle sequence (R = 0), one of only draft rows (L = R), one single key
    w = wl.small_case("bf16", [50, 6, 1], [0, 6, 1], n_q_heads=4, n_kv_heads=2, head_dim=64,
                      tokens_per_fragment=4, tree=True, seed=104)
    check_full(binding, w)


def test_capacity_far_above_live_lengths(binding):
    # most planned partitions are empty and must be skipped
    w = wl.small_case("e4m3", [40, 3, 250], [2, 1, 4], n_q_heads=8, n_kv_heads=2,
                      head_dim=128, tokens_per_fragment=16, max_pages=400, seed=105)
    info = check_full(binding, w)
    assert info["n_splits"] * info["keys_per_split"] >= 400 * 16


def test_arena_spanning_several_chunks(binding):
    w = wl.build("multi_chunk", "f16", [700, 90, 333], [3, 1, 2], 8, 2, 64,
                 fragment_bytes=16 * 2 * 64 * 2, chunk_bytes=16 * 2 * 64 * 2 * 24, max_pages=50,
                 seed=106, n_chunks=7)
    assert len(w.chunks) == 7
    check_full(binding, w)


def test_fragment_placement_does_not_change_output(binding):
    from test_oracle_pins import _replace_fragments
    w = wl.small_case("bf16", [300, 77], [3, 2], n_q_heads=8, n_kv_heads=2, head_dim=128,
                      tokens_per_fragment=16, seed=107)
    (out1, lse1, _), e1 = gpu_run(binding, w)
    chunks, kp, vp = _replace_fragments(w, seed=5)
    w2 = wl.Workload(**{**w.__dict__, "chunks": chunks, "k_pages": kp, "v_pages": vp})
    (out2, lse2, _), e2 = gpu_run(binding, w2)
    assert e1 == 0 and e2 == 0
    # same arithmetic in the same order: identical bits
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


def test_contiguous_cache_gives_identical_bits(binding):
    # the releases page reports that fragment addressing left outputs exactly
    # unchanged; here the identity table over a contiguous cache and the
    # shuffled table give the same bits on the tensor-core path
    w = wl.small_case("bf16", [3000, 1500, 77], [1, 4, 2], n_q_heads=24, n_kv_heads=4,
                      head_dim=128, tokens_per_fragment=128, seed=131)
    (out1, lse1, info), e1 = gpu_run(binding, w)
    (out2, lse2, _), e2 = gpu_run(binding, wl.contiguous_copy(w))
    assert e1 == 0 and e2 == 0 and info["kernel_name"] == "tcgen05"
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_forced_unsplit_plan_matches_oracle(binding, dtype):
    # one CTA per kv head (no split of the key range) against the oracle
    w = wl.small_case(dtype, [2900, 1100], [4, 1], n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, seed=132)
    props = torch.cuda.get_device_properties(0)
    limits = dict(n_sms=w.n_kv_heads, smem_optin=props.shared_memory_per_block_optin,
                  ctas_per_sm=0, allow_tcgen05=1)
    info = check_full(binding, w, plan_limits=limits)
    assert info["kernel_name"] == "tcgen05" and info["ctas"] == w.n_kv_heads


def test_bad_page_entry_sets_error_word_without_faulting(binding):
    w = wl.small_case("bf16", [100], [2], n_q_heads=4, n_kv_heads=2, head_dim=64,
                      tokens_per_fragment=16, seed=108)
    kp = w.k_pages.copy()
    kp[0, 2] = 10 ** 6          # names no fragment: the kernel must skip it and flag
    w2 = wl.Workload(**{**w.__dict__, "k_pages": kp})
    (_, _, _), err = gpu_run(binding, w2)
    assert err & binding.DEVERR_BAD_FRAGMENT


def test_bad_length_sets_error_word(binding):
    w = wl.small_case("bf16", [100], [2], n_q_heads=4, n_kv_heads=2, head_dim=64,
                      tokens_per_fragment=16, seed=109)
    lens = w.seq_lens.copy()
    lens[0] = 10 ** 6           # beyond the page-table capacity
    w2 = wl.Workload(**{**w.__dict__, "seq_lens": lens})
    (_, _, _), err = gpu_run(binding, w2)
    assert err & binding.DEVERR_BAD_LENGTH


# ---- the five full-size workloads, in the benchmark's launch configuration ----

# outputs the oracle checks of a workload too large for all of them: every
# head of these rows (the long query block: 64 of its 1024 rows, spread
# over all eight 128-row tiles, the first and last rows included)
SAMPLED_ROWS = {"prefill_block": sorted({0, 1023, *range(5, 1024, 16)})}


@pytest.mark.parametrize("name", wl.NAMES + wl.EXTRA_NAMES)
def test_full_size_workload(binding, name):
    # every (row, head) output of the workload against the oracle
    w = wl.BUILDERS[name]()
    (out, lse, info), err = gpu_run(binding, w)
    assert err == 0
    assert np.all(np.isfinite(out)) and np.all(np.isfinite(lse))
    rows = SAMPLED_ROWS.get(name)
    ref_out, ref_lse = oracle_all_outputs(to_problem(w), rows=rows)
    if rows is not None:
        out, lse, ref_out, ref_lse = out[rows], lse[rows], ref_out[rows], ref_lse[rows]
    assert_close(out, ref_out, w.dtype, what=name)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=lse_tol(w.dtype) * 4)


# ---- the tensor-core (tcgen05) partial pass --------------------------------------

def _rewrite_k(w, fn):
    """Rewrite every live K row of every sequence in place (test-side layout
    writer): row j of sequence s becomes fn(s, j, old_row_as_float32)."""
    from verify_attention_paged_b200.workloads import TORCH_DTYPES, ELEM_SIZE
    chunks = [c.copy() for c in w.chunks]
    T = w.tokens_per_fragment
    fpc = w.chunk_bytes // w.fragment_bytes
    row = w.n_kv_heads * w.head_dim * ELEM_SIZE[w.dtype]
    tdt = TORCH_DTYPES[w.dtype]
    for s in range(w.n_seqs):
        L = int(w.seq_lens[s])
        for j in range(L):
            c, off = divmod(int(w.k_pages[s, j // T]), fpc)
            b = off * w.fragment_bytes + (j % T) * row
            old = torch.from_numpy(chunks[c][b:b + row].copy()).view(tdt).float()
            new = fn(s, j, old).to(tdt).contiguous().view(torch.uint8).numpy()
            chunks[c][b:b + row] = new
    return wl.Workload(**{**w.__dict__, "chunks": chunks})


def check_kernel(b, w, kernel, two_pass=False):
    """One call through lse_attn_forward (the merge fused on tensor-core
    plans) against the oracle; with ``two_pass`` also lse_attn_run +
    lse_attn_merge (partials through the workspace) against the oracle."""
    (out, lse, info), err = gpu_run(b, w, kernel=kernel)
    assert info["kernel_name"] == kernel
    assert err == 0, f"device error word {err:#x}"
    ref_out, ref_lse = orc.attention(to_problem(w))
    assert_close(out, ref_out, w.dtype)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=lse_tol(w.dtype) * 4)
    if two_pass:
        call = b.DeviceCall(w, kernel=kernel)
        o2, l2 = call.run_two_pass()
        torch.cuda.synchronize()
        assert call.device_error() == 0
        o2 = o2[:w.total_rows].cpu().numpy()
        l2 = l2[:w.total_rows].cpu().numpy()
        call.close()
        assert_close(o2, ref_out, w.dtype, what="two-pass")
        np.testing.assert_allclose(l2, ref_lse, rtol=0, atol=lse_tol(w.dtype) * 4)
    return out


TC_DTYPES = ["bf16", "f16", "e4m3", "e5m2"]


@pytest.mark.parametrize("dtype", TC_DTYPES)
@pytest.mark.parametrize("tpf", [8, 16, 64, 128, 256, 512])
def test_tcgen05_fragment_sizes(binding, dtype, tpf):
    w = wl.small_case(dtype, [1, 127, 128, 129, 700, 2051], [1, 1, 2, 3, 4, 8],
                      n_q_heads=24, n_kv_heads=4, head_dim=128, tokens_per_fragment=tpf,
                      seed=200 + tpf)
    check_kernel(binding, w, "tcgen05")


@pytest.mark.parametrize("dtype", TC_DTYPES)
@pytest.mark.parametrize("heads,rows", [((24, 4), 8), ((32, 8), 12), ((8, 8), 1),
                                        ((16, 1), 3), ((12, 4), 16)])
def test_tcgen05_pairs_and_trees(binding, dtype, heads, rows):
    hq, hkv = heads
    lens = [300, 1000, rows, 4100, 64]
    w = wl.small_case(dtype, lens, [rows] * 5, n_q_heads=hq, n_kv_heads=hkv, head_dim=128,
                      tokens_per_fragment=64, tree=True, seed=210 + rows)
    check_kernel(binding, w, "tcgen05", two_pass=True)


@pytest.mark.parametrize("dtype", ["f16", "bf16", "e4m3"])
@pytest.mark.parametrize("heads,rows", [((24, 4), 16), ((32, 4), 12), ((16, 1), 8),
                                        ((24, 4), 9)])
def test_tcgen05_row_chunks(binding, dtype, heads, rows):
    # more (row, head) pairs per kv head than one score tile holds: the rows
    # are cut into chunks of floor(48 / G), each a segment of its own over
    # all of the sequence's keys (trees, ragged chunks, idle and short
    # sequences)
    hq, hkv = heads
    lens = [3000, rows, 700, 4100, 64, 1]
    rws = [rows, rows, max(1, rows // 2), rows, min(rows, 64), 1]
    w = wl.small_case(dtype, lens, rws, n_q_heads=hq, n_kv_heads=hkv, head_dim=128,
                      tokens_per_fragment=128, tree=True, seed=230 + rows + hq)
    (out, lse, info), err = gpu_run(binding, w, kernel="tcgen05")
    G = hq // hkv
    assert info["rows_per_chunk"] == (rows if G * rows <= 48 else 48 // G)
    assert err == 0
    ref_out, ref_lse = orc.attention(to_problem(w))
    assert_close(out, ref_out, w.dtype)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=lse_tol(w.dtype) * 4)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_tcgen05_many_segments_per_cta(binding, dtype):
    # 70 short sequences: CTAs cross many (sequence, kv head) segments, so the
    # Q ring, the two TMEM output slots and the piece numbering all rotate
    rng = np.random.default_rng(5)
    lens = [int(x) for x in rng.integers(1, 600, 70)]
    rows = [int(min(L, r)) for L, r in zip(lens, rng.integers(0, 7, 70))]
    w = wl.small_case(dtype, lens, rows, n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, tree=True, seed=220)
    out_tc = check_kernel(binding, w, "tcgen05", two_pass=True)
    out_cc = check_kernel(binding, w, "cuda_core")
    assert_close(out_tc, out_cc, dtype, what="tcgen05 vs cuda_core")


@pytest.mark.parametrize("dtype", ["f16", "e4m3"])
@pytest.mark.parametrize("n_sms", [3, 7, 16])
def test_tcgen05_segment_weighted_cut(binding, dtype, n_sms):
    # few working CTAs, so each takes at least 24 tiles and the cut charges
    # every segment 3 extra tiles: CTA ranges then start and end inside
    # short segments' overhead positions, and a segment's pieces are counted
    # by position in the pass (fused merge) and in the separate merge
    rng = np.random.default_rng(40 + n_sms)
    lens = [int(x) for x in rng.integers(1, 2500, 14)] + [130, 129, 1, 6000]
    rows = [int(min(L, r)) for L, r in zip(lens, rng.integers(0, 13, len(lens)))]
    w = wl.small_case(dtype, lens, rows, n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, tree=True, seed=240 + n_sms)
    props = torch.cuda.get_device_properties(0)
    limits = dict(n_sms=n_sms, smem_optin=props.shared_memory_per_block_optin, ctas_per_sm=0,
                  allow_tcgen05=1)
    ref_out, ref_lse = orc.attention(to_problem(w))
    call = binding.DeviceCall(w, plan_limits=limits)
    assert call.info["kernel_name"] == "tcgen05" and call.info["ctas"] == n_sms
    for label, fn in (("fused", call.run), ("two-pass", call.run_two_pass)):
        out, lse = fn()
        torch.cuda.synchronize()
        assert call.device_error() == 0, label
        assert_close(out[:w.total_rows].cpu().numpy(), ref_out, dtype, what=label)
        np.testing.assert_allclose(lse[:w.total_rows].cpu().numpy(), ref_lse, rtol=0,
                                   atol=lse_tol(dtype) * 4)
    call.close()


@pytest.mark.parametrize("dtype", ["f16", "e4m3"])
def test_tcgen05_more_sequences_than_the_cta_table(binding, dtype):
    # 130 sequences: more than the per-CTA sequence table holds, so the tile
    # iterator reads lengths from global memory (and numbers segments itself)
    rng = np.random.default_rng(6)
    lens = [int(x) for x in rng.integers(1, 900, 130)]
    rows = [int(min(L, r)) for L, r in zip(lens, rng.integers(0, 5, 130))]
    w = wl.small_case(dtype, lens, rows, n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, tree=True, seed=227)
    check_kernel(binding, w, "tcgen05", two_pass=True)


@pytest.mark.parametrize("dtype", ["f16", "e5m2"])
def test_tcgen05_fewer_tiles_than_ctas(binding, dtype):
    w = wl.small_case(dtype, [200], [2], n_q_heads=8, n_kv_heads=2, head_dim=128,
                      tokens_per_fragment=64, seed=221)
    check_kernel(binding, w, "tcgen05")


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_tcgen05_growing_scores_trigger_rescale(binding, dtype):
    # key rows grow with position, so the running maximum rises tile after
    # tile by more than the lazy threshold: the TMEM output must be rescaled
    w = wl.small_case(dtype, [3000, 900], [4, 1], n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=256, seed=222)
    w2 = _rewrite_k(w, lambda s, j, k: k * (0.25 + j / 150.0))
    check_kernel(binding, w2, "tcgen05")


@pytest.mark.parametrize("dtype", ["e4m3", "e5m2"])
@pytest.mark.parametrize("q_gain", [1e-3, 16.0])
def test_tcgen05_fp8_query_scale_range(binding, dtype, q_gain):
    # FP8 scores enter the tensor cores as scaled 8-bit terms of Q: tiny and
    # large query magnitudes (near-uniform and sharply peaked softmax, where
    # tiny probabilities must still count) stay within tolerance
    w = wl.small_case(dtype, [2000, 700], [3, 1], n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, seed=225)
    w2 = wl.Workload(**{**w.__dict__, "q": (w.q * q_gain).astype(np.float32)})
    check_kernel(binding, w2, "tcgen05")


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("smem", [232448, 200000, 185000, 160000])
def test_tcgen05_pipeline_configurations(binding, dtype, smem):
    # smaller shared-memory limits make the plan pick shallower K/V rings,
    # one Q slot and one P tile per softmax group: every configuration gives
    # the same results
    lens = [4000, 300, 2500, 129, 1]
    w = wl.small_case(dtype, lens, [3, 1, 2, 1, 1], n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, seed=226)
    props = torch.cuda.get_device_properties(0)
    limits = dict(n_sms=props.multi_processor_count, smem_optin=smem, ctas_per_sm=0,
                  allow_tcgen05=1)
    (out, lse, info), err = gpu_run(binding, w, plan_limits=limits)
    # where no tensor-core configuration fits, the plan falls back to the
    # CUDA-core kernel, which must give the same results
    assert info["kernel_name"] in ("tcgen05", "cuda_core")
    if smem >= 200000:
        assert info["kernel_name"] == "tcgen05"
    assert err == 0
    ref_out, ref_lse = orc.attention(to_problem(w))
    assert_close(out, ref_out, w.dtype, what=f"{info['kernel_name']} stages {info['stages']} "
                 f"q_slots {info['q_slots']} p_bufs {info['p_bufs']}")
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=lse_tol(w.dtype) * 4)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("frags_per_chunk", [5, 8])
def test_tcgen05_arena_of_many_chunks(binding, dtype, frags_per_chunk):
    # head_dim 128 on the tensor cores over an arena of 20-40 chunks (more
    # than 16 TMA descriptors), fragments shuffled across all of them
    w = wl.small_case(dtype, [3000, 700, 129, 2051], [4, 1, 2, 8], n_q_heads=24,
                      n_kv_heads=4, head_dim=128, tokens_per_fragment=64, tree=True,
                      frags_per_chunk=frags_per_chunk, seed=240 + frags_per_chunk)
    assert len(w.chunks) >= 17
    check_kernel(binding, w, "tcgen05", two_pass=True)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_tcgen05_capacity_far_above_live(binding, dtype):
    w = wl.small_case(dtype, [130, 5, 1000], [1, 1, 2], n_q_heads=24, n_kv_heads=4,
                      head_dim=128, tokens_per_fragment=128, max_pages=300, seed=223)
    check_kernel(binding, w, "tcgen05")


@pytest.mark.parametrize("dtype", ["bf16", "e5m2"])
def test_tcgen05_bad_page_sets_error_word(binding, dtype):
    w = wl.small_case(dtype, [600], [2], n_q_heads=8, n_kv_heads=2, head_dim=128,
                      tokens_per_fragment=128, seed=224)
    kp = w.k_pages.copy()
    kp[0, 1] = 10 ** 6
    w2 = wl.Workload(**{**w.__dict__, "k_pages": kp})
    (_, _, info), err = gpu_run(binding, w2, kernel="tcgen05")
    assert err & binding.DEVERR_BAD_FRAGMENT and not err & binding.DEVERR_TIMEOUT


def test_plan_picks_tensor_cores_for_the_16_bit_and_fp8_workloads(binding):
    for name, want in (("batched_decode", "tcgen05"), ("chain_verify", "tcgen05"),
                       ("long_fp8", "tcgen05"), ("tree_verify", "tcgen05"),
                       ("long_e5m2", "tcgen05"), ("long_fp8_scaled", "tcgen05"),
                       ("tiny_decode", "cuda_core"), ("prefill_block", "prefill")):
        w = wl.BUILDERS[name]()
        call = binding.DeviceCall(w)
        assert call.info["kernel_name"] == want, name
        call.close()
