"""The oracle built with the undefined-behaviour sanitizer (CPU): the pins'
calls over every format, trees, long chains, scales and the encoder's edge
values run without a single sanitizer report.  The sanitized library runs in
a child process (a report aborts it)."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "lse_oracle.c")

SCRIPT = r"""
import ctypes, sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
from oracle import oracle as orc
from verify_attention_paged_b200 import workloads as wl
from conftest import to_problem
real = orc._load()
m = ctypes.CDLL({lib!r})
for fn in ("orc_attention", "orc_attention_one", "orc_attention_split", "orc_decode",
           "orc_kv_bytes_per_token", "orc_encode", "orc_kv_append"):
    f = getattr(m, fn); f.argtypes = getattr(real, fn).argtypes; f.restype = getattr(real, fn).restype
orc._lib = m
for dtype in ["f32", "f16", "bf16", "e4m3", "e5m2"]:
    w = wl.small_case(dtype, [70, 33, 8, 1], [2, 4, 1, 1], n_q_heads=6, n_kv_heads=3,
                      head_dim=16, tokens_per_fragment=8, tree=True, seed=4)
    orc.attention(to_problem(w)); orc.attention_split(to_problem(w), 7)
    for c in range(256): orc.decode(dtype, c)
    for x in [0.0, -0.0, 1e-40, 3.3e38, float("inf"), float("nan"), 65520.0, 448.0, 464.0]:
        orc.encode(dtype, x)
w = wl.small_case("e4m3", [300, 90], [150, 70], n_q_heads=4, n_kv_heads=2, head_dim=16,
                  tokens_per_fragment=16, seed=21)
orc.attention(to_problem(w))
w = wl.small_case("e5m2", [40, 9], [1, 2], n_q_heads=4, n_kv_heads=2, head_dim=16,
                  tokens_per_fragment=8, seed=44, scaled=True, magnitude_spread=4.0)
orc.attention(to_problem(w))
import numpy as np
sc = w.scales.copy()
st = orc.kv_append([c.copy() for c in w.chunks], w.chunk_bytes, w.fragment_bytes, "e5m2", 2, 16,
                   w.k_pages, w.v_pages, np.array([30, 5], np.int32), np.array([0, 3, 5], np.int32),
                   np.ones((5, 2, 16), np.float32), np.zeros((5, 2, 16), np.float32), scales=sc)
assert st == 0
print("clean")
"""


def test_oracle_has_no_undefined_behaviour(tmp_path):
    lib = str(tmp_path / "liblse_oracle_ubsan.so")
    subprocess.check_call(["gcc", "-std=c99", "-O1", "-fPIC", "-shared", "-fsanitize=undefined",
                           "-fno-sanitize-recover=all", "-static-libubsan", "-o", lib, SRC, "-lm"])
    script = SCRIPT.format(root=ROOT, tests=os.path.join(ROOT, "tests"), lib=lib)
    r = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "runtime error" not in r.stderr, r.stderr[-2000:]
    assert r.stdout.strip().endswith("clean")
