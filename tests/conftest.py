import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    # temporary files (the oracle variants the tests compile) stay inside
    # the repository, in a git-ignored folder
    if not config.option.basetemp:
        config.option.basetemp = os.path.join(ROOT, ".pytest_tmp")


def to_problem(w, q=None, row_masks="keep", chunks=None, k_pages=None, v_pages=None):
    """Workload -> oracle Problem (same host arrays)."""
    from oracle import oracle as orc
    return orc.Problem(
        chunks=w.chunks if chunks is None else chunks,
        chunk_bytes=w.chunk_bytes, fragment_bytes=w.fragment_bytes, dtype=w.dtype,
        n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, n_q_heads=w.n_q_heads,
        k_pages=w.k_pages if k_pages is None else k_pages,
        v_pages=w.v_pages if v_pages is None else v_pages,
        seq_lens=w.seq_lens, row_offsets=w.row_offsets,
        row_masks=w.row_masks if isinstance(row_masks, str) else row_masks,
        q=w.q if q is None else q, scale=w.scale, scales=w.scales)


@pytest.fixture
def problem_of():
    return to_problem
