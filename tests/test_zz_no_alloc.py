"""The no-allocation entry point (lse_attn_forward_static) against the
regular entry points (lse_attn_run + lse_attn_merge on a caller workspace).

Callers that cannot allocate device memory when attention runs use the
static variant; it must give the same output as the regular path, call
after call, and refuse plans whose workspace exceeds its fixed scratch.
Collected last on purpose (file name) so a failure here leaves every other
test already run.
"""
import numpy as np
import pytest
import torch

from verify_attention_paged_b200 import workloads as wl
from parity_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def binding():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from verify_attention_paged_b200 import binding as b
    return b


def _static_call(b, call, out, lse):
    b.lse_attn_forward_static(call.plan, call.q, call.k_pages, call.v_pages, call.seq_lens,
                              call.row_offsets, call.row_masks, call.scale, out, lse,
                              call.stream)


@pytest.mark.parametrize("case", ["chain_bf16_tc", "tree_f16_tc", "tree_e4m3_cuda_core"])
def test_static_matches_regular_entry_points_twice(binding, case):
    if case == "chain_bf16_tc":
        w = wl.small_case("bf16", [700, 129, 3000], [8, 2, 4], n_q_heads=24, n_kv_heads=4,
                          head_dim=128, tokens_per_fragment=128, seed=301)
    elif case == "tree_f16_tc":
        w = wl.small_case("f16", [1500, 40, 260], [3, 5, 1], n_q_heads=24, n_kv_heads=4,
                          head_dim=128, tokens_per_fragment=64, tree=True, seed=302)
    else:
        w = wl.small_case("e4m3", [900, 77], [4, 2], n_q_heads=8, n_kv_heads=2, head_dim=128,
                          tokens_per_fragment=16, tree=True, seed=303)
    call = binding.DeviceCall(w)
    ref_out, ref_lse = call.run()
    torch.cuda.synchronize()
    assert call.device_error() == 0
    ref_out = ref_out[:w.total_rows].cpu().numpy()
    ref_lse = ref_lse[:w.total_rows].cpu().numpy()
    for _ in range(2):  # two calls in a row share the one scratch array
        out = torch.full_like(call.out, float("nan"))
        lse = torch.full_like(call.lse, float("nan"))
        _static_call(binding, call, out, lse)
        torch.cuda.synchronize()
        # the static call's device error word (bad page, bad length, timeout)
        assert binding.lse_attn_static_read_error(call.stream) == 0
        got = out[:w.total_rows].cpu().numpy()
        assert_close(got, ref_out, w.dtype, what=f"static {case}")
        np.testing.assert_allclose(lse[:w.total_rows].cpu().numpy(), ref_lse, rtol=0,
                                   atol=1e-5 if w.dtype == "f32" else 2e-3)
    call.close()


def test_static_refuses_plans_beyond_its_scratch(binding):
    # a capacity large enough that the workspace passes the static limit
    w = wl.small_case("bf16", [300], [4], n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, seed=304)
    call = binding.DeviceCall(w, max_total_rows=None)
    plan, ws = binding.lse_attn_plan(call.arena, 64, 64, 64 * 64, 24, 4096)
    assert ws > binding.STATIC_SCRATCH_BYTES
    with pytest.raises(binding.LseError, match="static scratch"):
        binding.lse_attn_forward_static(plan, call.q, call.k_pages, call.v_pages,
                                        call.seq_lens, call.row_offsets, None, call.scale,
                                        call.out, None, call.stream)
    binding.lse_attn_plan_destroy(plan)
    call.close()


def test_static_error_word_reports_a_bad_page(binding):
    # a page-table entry naming no fragment: the static call flags it in the
    # scratch's error word, which the static read-error call returns and
    # clears; the next clean call reads 0
    w = wl.small_case("bf16", [600], [2], n_q_heads=8, n_kv_heads=2, head_dim=128,
                      tokens_per_fragment=128, seed=305)
    kp = w.k_pages.copy()
    kp[0, 1] = 10 ** 6
    bad = wl.Workload(**{**w.__dict__, "k_pages": kp})
    for case, want in ((bad, binding.DEVERR_BAD_FRAGMENT), (w, 0)):
        call = binding.DeviceCall(case)
        _static_call(binding, call, call.out, call.lse)
        got = binding.lse_attn_static_read_error(call.stream)
        assert got == want, f"error word {got:#x}, expected {want:#x}"
        assert binding.lse_attn_static_read_error(call.stream) == 0  # cleared
        call.close()
