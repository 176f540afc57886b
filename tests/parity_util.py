"""Shared parity helpers: tolerances, comparison against the oracle, and
the oracle over every output of a large problem on all host cores."""
import os
import threading

import numpy as np

# Per-element tolerance, written out: FP32 K/V -> max |gpu - oracle| <= 1e-5;
# 16-bit and FP8 K/V -> |err| <= 2e-3, or |err| <= 2e-3 * |oracle|.
FP32_ABS = 1e-5
LOWP_TOL = 2e-3


def assert_close(got, want, dtype, what="out"):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite GPU values"
    err = np.abs(got - want)
    if dtype == "f32":
        worst = float(err.max(initial=0.0))
        assert worst <= FP32_ABS, f"{what}: max abs error {worst:.3e} > {FP32_ABS}"
    else:
        ok = (err <= LOWP_TOL) | (err <= LOWP_TOL * np.abs(want))
        if not ok.all():
            i = np.unravel_index(np.argmax(np.where(ok, 0, err)), err.shape)
            raise AssertionError(f"{what}: {int((~ok).sum())} elements out of tolerance, "
                                 f"worst at {i}: gpu {got[i]:.6g} oracle {want[i]:.6g}")
    return float(err.max(initial=0.0))


def lse_tol(dtype):
    return FP32_ABS if dtype == "f32" else LOWP_TOL


def oracle_all_outputs(pb, threads=None, rows=None):
    """Every (row, head) output of a problem from the float64 oracle, one
    output per call on one thread per host core (the ctypes calls release
    the GIL).  Same result as oracle.attention(pb), computed in parallel.
    ``rows`` (call row indices) restricts it to those rows; the other
    entries stay 0."""
    from oracle import oracle as orc
    m = orc.marshal(pb)
    ro = np.asarray(pb.row_offsets)
    n_rows = int(ro[-1])
    hq, d = pb.n_q_heads, pb.head_dim
    out = np.zeros((n_rows, hq, d), np.float64)
    lse = np.zeros((n_rows, hq), np.float64)
    keep = None if rows is None else set(int(x) for x in rows)
    items = [(s, r, h) for s in range(len(ro) - 1) for r in range(int(ro[s + 1] - ro[s]))
             for h in range(hq) if keep is None or int(ro[s]) + r in keep]
    # the longest sequences first, so the threads finish together
    lens = np.asarray(pb.seq_lens)
    items.sort(key=lambda t: -int(lens[t[0]]))
    lock = threading.Lock()
    state = {"next": 0, "error": None}

    def worker():
        while True:
            with lock:
                if state["next"] >= len(items) or state["error"] is not None:
                    return
                s, r, h = items[state["next"]]
                state["next"] += 1
            try:
                o, l = orc.attention_one(pb, s, r, h, marshalled=m)
            except Exception as e:  # surfaced below, on the caller's thread
                with lock:
                    state["error"] = e
                return
            out[ro[s] + r, h] = o
            lse[ro[s] + r, h] = l

    n = threads or os.cpu_count() or 1
    pool = [threading.Thread(target=worker) for _ in range(n)]
    for t in pool:
        t.start()
    for t in pool:
        t.join()
    if state["error"] is not None:
        raise state["error"]
    return out, lse
