"""GPU parity of the K/V append (lse_kv_append) against the oracle's append,
byte for byte, and append-then-attend against the oracle's attention."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from verify_attention_paged_b200 import workloads as wl
from conftest import to_problem
from parity_util import assert_close, lse_tol

pytestmark = pytest.mark.gpu

DTYPES = ["f32", "f16", "bf16", "e4m3", "e5m2"]


@pytest.fixture(scope="module")
def binding():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from verify_attention_paged_b200 import binding as b
    return b


def erase_tail(w, n_new):
    """w's arena with each sequence's last n_new keys (K and V) set to 0xFF
    (and their scales, if any, to NaN), and the append arguments that
    rewrite them."""
    chunks = [c.copy() for c in w.chunks]
    scales = None if w.scales is None else w.scales.copy()
    T = w.tokens_per_fragment
    fpc = w.chunk_bytes // w.fragment_bytes
    row = w.n_kv_heads * w.head_dim * wl.ELEM_SIZE[w.dtype]
    before, offs = [], [0]
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
                if scales is not None:
                    scales[f * w.n_kv_heads * T + np.arange(w.n_kv_heads) * T + j % T] = np.nan
    return (wl.Workload(**{**w.__dict__, "chunks": chunks, "scales": scales}),
            np.array(before, np.int32), np.array(offs, np.int32))


def device_append(b, call, w, before, offs, k_new, v_new):
    dev = call.q.device
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dt)).to(dev)  # noqa: E731
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    b.lse_kv_append(call.arena, w.n_seqs, w.k_pages.shape[1], t(k_new, np.float32),
                    t(v_new, np.float32), call.k_pages, call.v_pages, t(before, np.int32),
                    t(offs, np.int32), int(offs[-1]), err, call.stream)
    torch.cuda.synchronize()
    return int(err.item()) & 0xffffffff


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("head_dim", [64, 128, 256])
def test_append_matches_oracle_bytes(binding, dtype, head_dim):
    # random FP32 values (rounding exercised), some beyond the formats' range
    # (FP8 saturation, F16 overflow), written across fragment boundaries
    w = wl.small_case(dtype, [70, 9, 1, 33, 20], [1, 2, 1, 3, 1], n_q_heads=4, n_kv_heads=2,
                      head_dim=head_dim, tokens_per_fragment=8, seed=300 + head_dim)
    w2, before, offs = erase_tail(w, 12)
    n = int(offs[-1])
    rng = np.random.default_rng(head_dim)
    k_new = (rng.standard_normal((n, 2, head_dim)) * np.exp(rng.uniform(-6, 6, (n, 2, 1))))
    v_new = (rng.standard_normal((n, 2, head_dim)) * 3.0)
    k_new[0, 0, :4] = [1e6, -1e6, 70000.0, 460.0]
    k_new, v_new = k_new.astype(np.float32), v_new.astype(np.float32)
    want = [c.copy() for c in w2.chunks]
    st = orc.kv_append(want, w2.chunk_bytes, w2.fragment_bytes, dtype, 2, head_dim, w2.k_pages,
                       w2.v_pages, before, offs, k_new, v_new)
    assert st == 0
    call = binding.DeviceCall(w2)
    err = device_append(binding, call, w2, before, offs, k_new, v_new)
    assert err == 0
    for dc, hc in zip(call.chunks, want):
        assert np.array_equal(dc.cpu().numpy(), hc)
    call.close()


@pytest.mark.parametrize("dtype", ["bf16", "e4m3"])
def test_append_then_attend(binding, dtype):
    # erase the last keys (the verify step's drafts and more), append them
    # back from their values, then attend: the oracle's attention over the
    # generator's arena
    w = wl.small_case(dtype, [900, 300, 129], [4, 1, 2], n_q_heads=24, n_kv_heads=4,
                      head_dim=128, tokens_per_fragment=128, tree=True, seed=310)
    w2, before, offs = erase_tail(w, 10)
    k_new = np.concatenate([w.logical_k[s][int(before[s]):int(w.seq_lens[s])]
                            .to(torch.float32).numpy() for s in range(w.n_seqs)])
    v_new = np.concatenate([w.logical_v[s][int(before[s]):int(w.seq_lens[s])]
                            .to(torch.float32).numpy() for s in range(w.n_seqs)])
    call = binding.DeviceCall(w2)
    assert device_append(binding, call, w2, before, offs, k_new, v_new) == 0
    out, lse = call.run()
    torch.cuda.synchronize()
    assert call.device_error() == 0
    ref_out, ref_lse = orc.attention(to_problem(w))
    assert_close(out[:w.total_rows].cpu().numpy(), ref_out, dtype)
    np.testing.assert_allclose(lse[:w.total_rows].cpu().numpy(), ref_lse, rtol=0,
                               atol=lse_tol(dtype) * 4)
    call.close()


def test_append_past_the_page_table_sets_error_and_skips(binding):
    w = wl.small_case("bf16", [16, 8], [1, 1], n_q_heads=2, n_kv_heads=1, head_dim=64,
                      tokens_per_fragment=8, seed=320)
    call = binding.DeviceCall(w)
    before = np.array([15, 8], np.int32)
    offs = np.array([0, 3, 3], np.int32)  # keys 15, 16, 17 of sequence 0: table has 2 pages
    k_new = np.ones((3, 1, 64), np.float32)
    want = [c.copy() for c in w.chunks]
    st = orc.kv_append(want, w.chunk_bytes, w.fragment_bytes, "bf16", 1, 64, w.k_pages,
                       w.v_pages, before, offs, k_new, 2 * k_new)
    assert st == 2
    err = device_append(binding, call, w, before, offs, k_new, 2 * k_new)
    assert err & binding.DEVERR_BAD_FRAGMENT
    for dc, hc in zip(call.chunks, want):
        assert np.array_equal(dc.cpu().numpy(), hc)  # key 15 written, 16 and 17 not
    call.close()


@pytest.mark.parametrize("dtype", ["e4m3", "e5m2"])
@pytest.mark.parametrize("head_dim", [64, 128, 256])
def test_scaled_append_matches_oracle_bytes_and_scales(binding, dtype, head_dim):
    # an arena with per-vector scales: each new vector's scale and stored
    # codes, bit for bit (vectors of sizes spread over 2^(+-12), a zero vector)
    w = wl.small_case(dtype, [70, 9, 1, 33, 20], [1, 2, 1, 3, 1], n_q_heads=4, n_kv_heads=2,
                      head_dim=head_dim, tokens_per_fragment=8, seed=330 + head_dim,
                      scaled=True)
    w2, before, offs = erase_tail(w, 12)
    n = int(offs[-1])
    rng = np.random.default_rng(head_dim + 1)
    k_new = rng.standard_normal((n, 2, head_dim)) * np.exp2(rng.uniform(-12, 12, (n, 2, 1)))
    v_new = rng.standard_normal((n, 2, head_dim)) * 3.0
    k_new[1, 1] = 0.0
    k_new, v_new = k_new.astype(np.float32), v_new.astype(np.float32)
    want = [c.copy() for c in w2.chunks]
    want_sc = w2.scales.copy()
    st = orc.kv_append(want, w2.chunk_bytes, w2.fragment_bytes, dtype, 2, head_dim, w2.k_pages,
                       w2.v_pages, before, offs, k_new, v_new, scales=want_sc)
    assert st == 0
    call = binding.DeviceCall(w2)
    assert call.scales is not None
    err = device_append(binding, call, w2, before, offs, k_new, v_new)
    assert err == 0
    for dc, hc in zip(call.chunks, want):
        assert np.array_equal(dc.cpu().numpy(), hc)
    got_sc = call.scales.cpu().numpy()
    live = ~np.isnan(want_sc)
    assert live.sum() > np.isnan(w2.scales[~np.isnan(w.scales)]).sum() > 0  # erased, rewritten
    assert np.array_equal(got_sc[live].view(np.uint32), want_sc[live].view(np.uint32))
    call.close()


def test_scaled_append_then_attend(binding):
    # a scaled FP8 arena: erase the last keys, append them back from their
    # FP32 vectors (the library picks the scales), attend, compare with the
    # oracle's attention over the generator's arena
    w = wl.small_case("e4m3", [900, 300, 129], [4, 1, 2], n_q_heads=24, n_kv_heads=4,
                      head_dim=128, tokens_per_fragment=128, tree=True, seed=340, kv_std=0.5,
                      scaled=True, magnitude_spread=1.0)
    w2, before, offs = erase_tail(w, 10)
    k_new = np.concatenate([w.logical_k_src[s][int(before[s]):int(w.seq_lens[s])].numpy()
                            for s in range(w.n_seqs)])
    v_new = np.concatenate([w.logical_v_src[s][int(before[s]):int(w.seq_lens[s])].numpy()
                            for s in range(w.n_seqs)])
    call = binding.DeviceCall(w2)
    assert device_append(binding, call, w2, before, offs, k_new, v_new) == 0
    out, lse = call.run()
    torch.cuda.synchronize()
    assert call.device_error() == 0
    ref_out, ref_lse = orc.attention(to_problem(w))
    assert_close(out[:w.total_rows].cpu().numpy(), ref_out, "e4m3")
    np.testing.assert_allclose(lse[:w.total_rows].cpu().numpy(), ref_lse, rtol=0,
                               atol=lse_tol("e4m3") * 4)
    call.close()
