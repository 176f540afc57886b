"""GPU parity of per-vector FP32 K/V scales (the README's fp8/bf8 "with
scales" storage) against the float64 oracle, through the C ABI: both 8-bit
formats, the tensor-core kernel at every pair bucket and fragment size, the
CUDA-core kernel (head dims 64 and 256), scales spanning a wide range
(the vectors they give back of ordinary size), vectors of varying size, and
zero or tiny V scales."""
import numpy as np
import pytest
import torch

from verify_attention_paged_b200 import workloads as wl
from test_parity_gpu import binding, check_full  # noqa: F401  (fixture)

pytestmark = pytest.mark.gpu

FP8 = ["e4m3", "e5m2"]


@pytest.mark.parametrize("dtype", FP8)
@pytest.mark.parametrize("tree", [False, True])
@pytest.mark.parametrize("tpf", [16, 128, 512])
def test_scaled_tensor_core_path(binding, dtype, tree, tpf):
    w = wl.small_case(dtype, [1, 7, 33, 300, 517, 129], [1, 1, 3, 8, 4, 5], n_q_heads=24,
                      n_kv_heads=4, head_dim=128, tokens_per_fragment=tpf, tree=tree, seed=141,
                      kv_std=0.5, scaled=True, scale_spread=5.0)
    info = check_full(binding, w)
    assert info["kernel_name"] == "tcgen05" and info["scaled"] == 1


@pytest.mark.parametrize("dtype", FP8)
@pytest.mark.parametrize("rows", [1, 2, 4, 5, 8])
def test_scaled_pair_buckets(binding, dtype, rows):
    # G = 6: pairs 6, 12, 24, 30, 48 -> buckets 8, 16, 24, 32, 48
    w = wl.small_case(dtype, [700, 260], [rows, rows], n_q_heads=24, n_kv_heads=4,
                      head_dim=128, tokens_per_fragment=128, seed=142 + rows, kv_std=0.5,
                      scaled=True, scale_spread=3.0)
    info = check_full(binding, w)
    assert info["kernel_name"] == "tcgen05"


@pytest.mark.parametrize("dtype", FP8)
@pytest.mark.parametrize("head_dim", [64, 256])
def test_scaled_cuda_core_path(binding, dtype, head_dim):
    w = wl.small_case(dtype, [5, 90, 333], [1, 3, 2], n_q_heads=8, n_kv_heads=2,
                      head_dim=head_dim, tokens_per_fragment=16, tree=True, seed=150,
                      kv_std=0.5, scaled=True, scale_spread=5.0)
    info = check_full(binding, w)
    assert info["kernel_name"] == "cuda_core"


@pytest.mark.parametrize("dtype", FP8)
@pytest.mark.parametrize("kernel", ["tcgen05", "cuda_core"])
def test_zero_and_tiny_v_scales(binding, dtype, kernel):
    # V scales of 0 and 1e-30 on a fifth of the vectors: those keys still
    # weigh in the softmax denominator
    w = wl.small_case(dtype, [400, 129], [2, 3], n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, seed=151, kv_std=0.5, scaled=True)
    rng = np.random.default_rng(7)
    s = w.scales.copy()
    live = np.flatnonzero(~np.isnan(s))
    pick = rng.choice(live, len(live) // 5, replace=False)
    s[pick[: len(pick) // 2]] = 0.0
    s[pick[len(pick) // 2:]] = 1e-30
    w2 = wl.Workload(**{**w.__dict__, "scales": s})
    info = check_full(binding, w2, kernel=kernel)
    assert info["kernel_name"] == kernel


@pytest.mark.parametrize("dtype", FP8)
def test_scaled_vectors_of_varying_size(binding, dtype):
    # vector sizes vary by 2^(+-1) (their scales with them).  FP8 P carries
    # 11 bits, so the output error grows with the size of the V vectors it
    # weighs; at these sizes it stays within the stated tolerance.
    w = wl.small_case(dtype, [900, 333], [4, 1], n_q_heads=24, n_kv_heads=4, head_dim=128,
                      tokens_per_fragment=128, seed=153, kv_std=0.5, scaled=True,
                      magnitude_spread=1.0)
    check_full(binding, w)


def test_scaled_contiguous_cache_gives_identical_bits(binding):
    from test_parity_gpu import gpu_run
    w = wl.small_case("e4m3", [3000, 1500, 77], [1, 4, 2], n_q_heads=24, n_kv_heads=4,
                      head_dim=128, tokens_per_fragment=128, seed=152, kv_std=0.5, scaled=True,
                      scale_spread=2.0)
    (out1, lse1, info), e1 = gpu_run(binding, w)
    (out2, lse2, _), e2 = gpu_run(binding, wl.contiguous_copy(w))
    assert e1 == 0 and e2 == 0 and info["scaled"] == 1
    assert np.array_equal(out1, out2) and np.array_equal(lse1, lse2)
