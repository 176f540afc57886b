"""Long query blocks (more than 64 chained query rows per sequence) on the
rows-as-M tensor-core pass, against the float64 oracle on every output.

Source: LSE releases, v0.4.14 "Improvements" (paged attention over prefill
blocks, skipping key windows that no row of the block sees; the windows that
contribute keep their arithmetic).  Each row r of a block sees the context
and the positions up to its own; the kernel stops each 128-row tile's key
loop at the tile holding its last row's position."""
import numpy as np
import pytest
import torch

from verify_attention_paged_b200 import workloads as wl
from conftest import to_problem
from parity_util import assert_close, lse_tol, oracle_all_outputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def binding():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from verify_attention_paged_b200 import binding as b
    return b


def run(b, w):
    call = b.DeviceCall(w)
    out, lse = call.run()
    torch.cuda.synchronize()
    err = call.device_error()
    res = (out[:w.total_rows].cpu().numpy(), lse[:w.total_rows].cpu().numpy(), call.info)
    call.close()
    return res, err


def check(b, w):
    (out, lse, info), err = run(b, w)
    assert info["kernel_name"] == "prefill", info["kernel_name"]
    assert err == 0, f"device error word {err:#x}"
    ref_out, ref_lse = oracle_all_outputs(to_problem(w))
    assert_close(out, ref_out, w.dtype)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=lse_tol(w.dtype) * 4)
    return out, lse


@pytest.mark.parametrize("dtype", ["bf16", "f16", "e4m3", "e5m2"])
@pytest.mark.parametrize("lens,rows,tpf", [
    ([1100, 300, 129], [1000, 70, 129], 64),  # 1000 rows; a block with no context (L = R)
    ([5000, 700, 40], [150, 300, 5], 128),    # ragged row tiles; a verify-size block
    ([2048], [256], 256),                      # whole row tiles
])
def test_long_query_blocks(binding, dtype, lens, rows, tpf):
    w = wl.small_case(dtype, lens, rows, n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=tpf, kv_std=0.5 if dtype.startswith("e") else 1.0,
                      seed=400 + len(lens) + tpf)
    check(binding, w)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_long_context_segments_shared_by_ctas(binding, dtype):
    # 20K keys of context under 200 rows: each (row tile, head) segment is
    # cut across several CTAs and merged at the end of the launch
    w = wl.small_case(dtype, [20200], [200], n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, kv_std=0.5 if dtype == "e4m3" else 1.0,
                      seed=410)
    check(binding, w)


@pytest.mark.parametrize("dtype", ["f16", "e5m2"])
def test_many_segments_per_cta(binding, dtype):
    # short contexts, many sequences and heads: CTAs cross many segments, so
    # Q is restaged and the output accumulator reused within a CTA
    rng = np.random.default_rng(3)
    lens = [int(x) for x in rng.integers(70, 400, 9)]
    rows = [int(min(L, r)) for L, r in zip(lens, rng.integers(65, 300, 9))]
    w = wl.small_case(dtype, lens, rows, n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=16, kv_std=0.5 if dtype == "e5m2" else 1.0, seed=411)
    check(binding, w)


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
@pytest.mark.parametrize("q_gain", [1e-3, 8.0])
def test_query_scale_range(binding, dtype, q_gain):
    # near-uniform and sharply peaked softmaxes (tiny probabilities still count)
    w = wl.small_case(dtype, [900, 300], [300, 100], n_q_heads=8, n_kv_heads=2, head_dim=128,
                      tokens_per_fragment=64, kv_std=0.5 if dtype == "e4m3" else 1.0, seed=412)
    w2 = wl.Workload(**{**w.__dict__, "q": (w.q * q_gain).astype(np.float32)})
    check(binding, w2)


def test_fragment_placement_gives_identical_bits(binding):
    w = wl.small_case("bf16", [3000, 700], [300, 80], n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, seed=413)
    (o1, l1, i1), e1 = run(binding, w)
    (o2, l2, _), e2 = run(binding, wl.contiguous_copy(w))
    assert e1 == 0 and e2 == 0 and i1["kernel_name"] == "prefill"
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_bad_page_entry_sets_error_word(binding):
    w = wl.small_case("bf16", [700], [100], n_q_heads=8, n_kv_heads=2, head_dim=128,
                      tokens_per_fragment=128, seed=414)
    kp = w.k_pages.copy()
    kp[0, 2] = 10 ** 6
    (_, _, info), err = run(binding, wl.Workload(**{**w.__dict__, "k_pages": kp}))
    assert info["kernel_name"] == "prefill"
    assert err & binding.DEVERR_BAD_FRAGMENT and not err & binding.DEVERR_TIMEOUT


def test_two_pass_calls_refuse_a_long_block_plan(binding):
    w = wl.small_case("bf16", [300], [100], n_q_heads=8, n_kv_heads=2, head_dim=128,
                      tokens_per_fragment=128, seed=415)
    call = binding.DeviceCall(w)
    with pytest.raises(binding.LseError, match="lse_attn_forward"):
        call.run_partial()
    with pytest.raises(binding.LseError, match="lse_attn_forward"):
        call.run_merge()
    call.close()
