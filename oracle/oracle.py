"""Python face of the float64 CPU oracle (``lse_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
benchmark's CPU-baseline leg are the only callers.  The oracle shares no code
with the CUDA library and never imports it; it takes host numpy arrays (the
same arena bytes and page tables the GPU reads) and returns float64 results.

What each entry point follows is stated in ``lse_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lse_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liblse_oracle.so")

DTYPE_CODES = {"f32": 0, "f16": 1, "bf16": 2, "e4m3": 3, "e5m2": 4}
ELEM_SIZE = {"f32": 4, "f16": 2, "bf16": 2, "e4m3": 1, "e5m2": 1}

STATUS = {0: "ok", 1: "bad shape", 2: "bad page", 3: "bad mask", 4: "bad dtype"}


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C99, -O2, no fast-math)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    os.makedirs(_LIB_DIR, exist_ok=True)
    tmp = _LIB + f".{os.getpid()}.tmp"
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-fno-fast-math",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("chunks", ctypes.POINTER(ctypes.c_void_p)),
        ("n_chunks", ctypes.c_int),
        ("chunk_bytes", ctypes.c_int64),
        ("fragment_bytes", ctypes.c_int64),
        ("dtype", ctypes.c_int),
        ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("n_q_heads", ctypes.c_int),
        ("n_seqs", ctypes.c_int),
        ("max_pages", ctypes.c_int),
        ("k_pages", ctypes.c_void_p),
        ("v_pages", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("row_offsets", ctypes.c_void_p),
        ("row_masks", ctypes.c_void_p),
        ("q", ctypes.c_void_p),
        ("scale", ctypes.c_double),
        ("scales", ctypes.c_void_p),
        ("n_scales", ctypes.c_int64),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER(_Problem)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.orc_attention.argtypes = [P, dp, dp]
        lib.orc_attention_one.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, dp]
        lib.orc_attention_split.argtypes = [P, ctypes.c_int64, dp, dp, dp]
        lib.orc_decode.argtypes = [ctypes.c_int, ctypes.c_uint32]
        lib.orc_decode.restype = ctypes.c_double
        lib.orc_kv_bytes_per_token.argtypes = [ctypes.c_int] * 5
        lib.orc_kv_bytes_per_token.restype = ctypes.c_int64
        lib.orc_encode.argtypes = [ctypes.c_int, ctypes.c_double]
        lib.orc_encode.restype = ctypes.c_uint32
        vp = ctypes.c_void_p
        lib.orc_kv_append.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int,
                                      ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      vp, vp, vp, vp, vp, vp, vp, ctypes.c_int64]
        lib.orc_kv_append.restype = ctypes.c_int
        for f in (lib.orc_attention, lib.orc_attention_one, lib.orc_attention_split):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


@dataclass
class Problem:
    """Host-side description of one attention call (numpy arrays)."""
    chunks: list            # list of uint8 arrays, each chunk_bytes long
    chunk_bytes: int
    fragment_bytes: int
    dtype: str              # "f32" | "f16" | "bf16" | "e4m3" | "e5m2"
    n_kv_heads: int
    head_dim: int
    n_q_heads: int
    k_pages: np.ndarray     # int32 [S, max_pages]
    v_pages: np.ndarray     # int32 [S, max_pages]
    seq_lens: np.ndarray    # int32 [S]
    row_offsets: np.ndarray  # int32 [S + 1]
    row_masks: np.ndarray | None  # uint64 [total_rows] or None (chain)
    q: np.ndarray           # float32 [total_rows, Hq, D]
    scale: float
    # per-vector scales: float32, a block of T * Hkv per fragment id,
    # [kv_head][token] inside it; None means every scale is 1
    scales: np.ndarray | None = None


def _as(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


class _Marshalled:
    """Keeps the contiguous copies alive while the C struct points at them."""

    def __init__(self, pb: Problem):
        self.chunks = [np.ascontiguousarray(c, dtype=np.uint8) for c in pb.chunks]
        self.k_pages = _as(pb.k_pages, np.int32)
        self.v_pages = _as(pb.v_pages, np.int32)
        self.seq_lens = _as(pb.seq_lens, np.int32)
        self.row_offsets = _as(pb.row_offsets, np.int32)
        self.row_masks = None if pb.row_masks is None else _as(pb.row_masks, np.uint64)
        self.q = _as(pb.q, np.float32)
        self.scales = None if pb.scales is None else _as(pb.scales, np.float32).reshape(-1)
        self.chunk_ptrs = (ctypes.c_void_p * max(1, len(self.chunks)))(
            *[c.ctypes.data for c in self.chunks])
        ptr = lambda a: None if a is None else a.ctypes.data  # noqa: E731
        self.s = _Problem(
            ctypes.cast(self.chunk_ptrs, ctypes.POINTER(ctypes.c_void_p)), len(self.chunks),
            pb.chunk_bytes, pb.fragment_bytes, DTYPE_CODES[pb.dtype], pb.n_kv_heads,
            pb.head_dim, pb.n_q_heads, len(self.seq_lens), self.k_pages.shape[1],
            ptr(self.k_pages), ptr(self.v_pages), ptr(self.seq_lens), ptr(self.row_offsets),
            ptr(self.row_masks), ptr(self.q), float(pb.scale), ptr(self.scales),
            0 if self.scales is None else self.scales.size)


def _check(st):
    if st != 0:
        raise OracleError(f"oracle rejected the problem: {STATUS.get(st, st)}")


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def attention(pb: Problem):
    """All outputs: (out float64 [total_rows, Hq, D], lse float64 [total_rows, Hq])."""
    m = _Marshalled(pb)
    rows = int(m.row_offsets[-1])
    out = np.zeros((rows, pb.n_q_heads, pb.head_dim), np.float64)
    lse = np.zeros((rows, pb.n_q_heads), np.float64)
    _check(_load().orc_attention(ctypes.byref(m.s), _dp(out), _dp(lse)))
    return out, lse


def attention_one(pb: Problem, seq: int, row: int, head: int, marshalled=None):
    """One output (seq, row within seq, query head): (out [D], lse)."""
    m = marshalled or _Marshalled(pb)
    out = np.zeros(pb.head_dim, np.float64)
    lse = np.zeros(1, np.float64)
    _check(_load().orc_attention_one(ctypes.byref(m.s), seq, row, head, _dp(out), _dp(lse)))
    return out, float(lse[0])


def marshal(pb: Problem):
    """Marshal once for many attention_one calls."""
    return _Marshalled(pb)


def attention_split(pb: Problem, keys_per_part: int):
    """Split-then-merge evaluation with partitions of keys_per_part keys."""
    m = _Marshalled(pb)
    rows = int(m.row_offsets[-1])
    out = np.zeros((rows, pb.n_q_heads, pb.head_dim), np.float64)
    lse = np.zeros((rows, pb.n_q_heads), np.float64)
    scratch = np.zeros(pb.head_dim, np.float64)
    _check(_load().orc_attention_split(ctypes.byref(m.s), int(keys_per_part), _dp(out),
                                       _dp(lse), _dp(scratch)))
    return out, lse


def decode(dtype: str, bits: int) -> float:
    """Decode one stored element (its bit pattern) to a Python float."""
    return _load().orc_decode(DTYPE_CODES[dtype], int(bits))


def kv_bytes_per_token(dtype: str, n_layers: int, n_kv_heads: int, head_dim: int,
                       with_scales: bool) -> int:
    return int(_load().orc_kv_bytes_per_token(DTYPE_CODES[dtype], n_layers, n_kv_heads,
                                              head_dim, int(with_scales)))


def encode(dtype: str, x: float) -> int:
    """The stored bits of x in a format: nearest value, ties to even (FP8
    saturates at its largest finite value, F16/BF16 overflow to infinity)."""
    return int(_load().orc_encode(DTYPE_CODES[dtype], float(x)))


def kv_append(chunks, chunk_bytes, fragment_bytes, dtype, n_kv_heads, head_dim, k_pages,
              v_pages, seq_lens_before, new_offsets, k_new, v_new, scales=None):
    """Write new tokens' K/V into host copies of the arena chunks (modified in
    place): token i of sequence s (new_offsets[s] <= i < new_offsets[s+1])
    goes to key position seq_lens_before[s] + i - new_offsets[s].  With
    ``scales`` (a float32 per-vector scale array, 8-bit formats; modified in
    place) each vector is stored divided by its new scale.  Returns the
    oracle status (0, or 2 when some position has no fragment; the others
    are written)."""
    if scales is not None:
        assert scales.dtype == np.float32 and scales.flags["C_CONTIGUOUS"]
    for c in chunks:
        assert c.dtype == np.uint8 and c.flags["C_CONTIGUOUS"]
    kp, vp_ = _as(k_pages, np.int32), _as(v_pages, np.int32)
    sl, no = _as(seq_lens_before, np.int32), _as(new_offsets, np.int32)
    kn, vn = _as(k_new, np.float32), _as(v_new, np.float32)
    ptrs = (ctypes.c_void_p * max(1, len(chunks)))(*[c.ctypes.data for c in chunks])
    return int(_load().orc_kv_append(
        ctypes.cast(ptrs, ctypes.POINTER(ctypes.c_void_p)), len(chunks), int(chunk_bytes),
        int(fragment_bytes), DTYPE_CODES[dtype], int(n_kv_heads), int(head_dim), len(sl),
        kp.shape[1], kp.ctypes.data, vp_.ctypes.data, sl.ctypes.data, no.ctypes.data,
        kn.ctypes.data, vn.ctypes.data, None if scales is None else scales.ctypes.data,
        0 if scales is None else scales.size))
