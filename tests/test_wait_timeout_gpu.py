"""The bounded waits of the tensor-core pass: when a tile never arrives
(each CTA skips loading one tile: a barrier that nothing completes), the
waits give up after about two seconds, the call reports LSE_DEVERR_TIMEOUT
through the device error word and leaves the GPU usable: the next call on
the same plan and workspace is correct.  No fault, trap or endless loop is
involved; the only failure is a flag that nothing sets."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from verify_attention_paged_b200 import workloads as wl
from conftest import to_problem
from parity_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def binding():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from verify_attention_paged_b200 import binding as b
    return b


@pytest.mark.parametrize("two_pass", [False, True])
def test_wait_that_runs_out_reports_timeout_and_the_next_call_is_clean(binding, two_pass):
    w = wl.small_case("bf16", [3000, 700, 129], [4, 1, 2], n_q_heads=24, n_kv_heads=4,
                      head_dim=128, tokens_per_fragment=128, seed=501)
    call = binding.DeviceCall(w)
    assert call.info["kernel_name"] == "tcgen05"
    binding.lse_attn_test_withhold_tile(call.plan, 0)
    (call.run_two_pass if two_pass else call.run)()
    torch.cuda.synchronize()
    err = call.device_error()      # also clears the fused pass's counters
    assert err & binding.DEVERR_TIMEOUT, f"error word {err:#x}"
    binding.lse_attn_test_withhold_tile(call.plan, -1)
    out, lse = (call.run_two_pass if two_pass else call.run)()
    torch.cuda.synchronize()
    assert call.device_error() == 0
    ref, _ = orc.attention(to_problem(w))
    assert_close(out[:w.total_rows].cpu().numpy(), ref, w.dtype)
    call.close()
