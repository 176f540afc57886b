"""Thin ctypes binding of liblse_attn.so (declared in include/lse_attn.h).

Every function here has the name of the C entry point it wraps and only
marshals arguments: device pointers may be given as ints or as torch tensors
(their ``data_ptr()``), streams as ints or ``torch.cuda.Stream``.  All
attention arithmetic runs in the library's CUDA kernels.  Importing this
module loads the library and raises ImportError when it is missing; there is
no fallback.

``DeviceCall`` below uploads one host-side problem (arena bytes, page
tables, rows, Q) to the current CUDA device and calls run + merge; it is the
convenience path the tests, the smoke check and the benchmark share.
"""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblse_attn.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "lse_attn.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m verify_attention_paged_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

LSE_OK = 0
KV_DTYPES = {"f32": 0, "f16": 1, "bf16": 2, "e4m3": 3, "e5m2": 4}
KERNELS = {0: "cuda_core", 1: "tcgen05", 2: "prefill"}
DEVERR_BAD_FRAGMENT = 0x1
DEVERR_BAD_LENGTH = 0x2
DEVERR_TIMEOUT = 0x4

_vp = ctypes.c_void_p
_i = ctypes.c_int
_i32p = ctypes.POINTER(ctypes.c_int32)
_errp = ctypes.POINTER(ctypes.c_char_p)


class ArenaInfo(ctypes.Structure):
    _fields_ = [("tokens_per_fragment", ctypes.c_int32), ("n_fragments", ctypes.c_int32),
                ("n_free", ctypes.c_int32), ("n_chunks", ctypes.c_int32),
                ("n_empty_chunks", ctypes.c_int32)]


class PlanInfo(ctypes.Structure):
    _fields_ = [("n_splits", ctypes.c_int32), ("keys_per_split", ctypes.c_int32),
                ("kernel", ctypes.c_int32), ("key_tile", ctypes.c_int32),
                ("pairs", ctypes.c_int32), ("smem_bytes", ctypes.c_int32),
                ("ctas", ctypes.c_int32), ("workspace_bytes", ctypes.c_int64),
                ("stages", ctypes.c_int32), ("q_slots", ctypes.c_int32),
                ("p_bufs", ctypes.c_int32), ("rows_per_chunk", ctypes.c_int32),
                ("scaled", ctypes.c_int32), ("v_stages", ctypes.c_int32),
                ("merge_in_pass", ctypes.c_int32)]


class DeviceLimits(ctypes.Structure):
    _fields_ = [("n_sms", ctypes.c_int32), ("smem_optin", ctypes.c_int32),
                ("ctas_per_sm", ctypes.c_int32), ("allow_tcgen05", ctypes.c_int32)]


def _sig(name, res, *args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


_sig("lse_status_string", ctypes.c_char_p, _i)
_sig("lse_free", None, _vp)
_sig("lse_kv_arena_create", _i, ctypes.POINTER(_vp), _i, ctypes.c_size_t, ctypes.c_size_t, _i,
     _i, _i, ctypes.POINTER(_vp), _errp)
_sig("lse_kv_arena_add_chunk", _i, _vp, _vp, _i32p, _errp)
_sig("lse_kv_arena_alloc", _i, _vp, _i, _i32p, _errp)
_sig("lse_kv_arena_free", _i, _vp, _i, _i32p, _errp)
_sig("lse_kv_arena_query", _i, _vp, ctypes.POINTER(ArenaInfo))
_sig("lse_kv_arena_destroy", None, _vp)
_sig("lse_kv_arena_set_scales", _i, _vp, _vp, ctypes.c_int64, _errp)
_sig("lse_attn_plan", _i, _vp, _i, _i, _i, _i, _i, ctypes.POINTER(_vp),
     ctypes.POINTER(ctypes.c_size_t), _errp)
_sig("lse_attn_plan_ex", _i, _vp, _i, _i, _i, _i, _i, ctypes.POINTER(DeviceLimits),
     ctypes.POINTER(_vp), ctypes.POINTER(ctypes.c_size_t), _errp)
_sig("lse_attn_plan_query", _i, _vp, ctypes.POINTER(PlanInfo))
_sig("lse_attn_split_rule", _i, ctypes.c_int64, _i, _i, _i, _i, _i32p)
_sig("lse_attn_workspace_init", _i, _vp, _vp, _vp, _errp)
_sig("lse_attn_plan_destroy", None, _vp)
_sig("lse_attn_run", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _vp, _errp)
_sig("lse_attn_merge", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _errp)
_sig("lse_attn_forward", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _vp, _vp,
     _vp, _errp)
_sig("lse_attn_validate", _i, _vp, _i32p, _i32p, _i32p, _i32p,
     ctypes.POINTER(ctypes.c_uint64), _errp)
_sig("lse_attn_read_error", _i, _vp, _vp, _vp, ctypes.POINTER(ctypes.c_uint32), _errp)
_sig("lse_attn_forward_static", _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _vp, _vp,
     _vp, _errp)
_sig("lse_kv_append", _i, _vp, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _errp)
_sig("lse_attn_static_read_error", _i, _vp, ctypes.POINTER(ctypes.c_uint32), _errp)
_sig("lse_attn_test_withhold_tile", _i, _vp, _i)
STATIC_SCRATCH_BYTES = 32 << 20


class LseError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"[{lse_status_string(status)}] {message}")


def declared_symbols() -> list[str]:
    """Entry points declared in include/lse_attn.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^LSE_API\s+[\w\s\*]*?\b(lse_\w+)\(", text, flags=re.M)))


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "cuda_stream"):
        return x.cuda_stream
    raise TypeError(f"cannot take a pointer of {type(x)}")


def _call(fn, *args):
    err = ctypes.c_char_p()
    st = fn(*args, ctypes.byref(err))
    if st != LSE_OK:
        msg = err.value.decode() if err.value else ""
        if err.value:
            _lib.lse_free(ctypes.cast(err, _vp))
        raise LseError(st, msg)


def _i32(a):
    a = np.ascontiguousarray(a, dtype=np.int32)
    return a, a.ctypes.data_as(_i32p)


def lse_status_string(status: int) -> str:
    return _lib.lse_status_string(status).decode()


def lse_free(p) -> None:
    """Release a string the library returned (the binding does this itself)."""
    _lib.lse_free(p)


# ---- arena -------------------------------------------------------------------

def lse_kv_arena_create(chunk_bases, chunk_bytes: int, fragment_bytes: int, kv_dtype,
                        n_kv_heads: int, head_dim: int):
    bases = (_vp * len(chunk_bases))(*[_ptr(b) for b in chunk_bases])
    out = _vp()
    dt = KV_DTYPES[kv_dtype] if isinstance(kv_dtype, str) else int(kv_dtype)
    _call(_lib.lse_kv_arena_create, bases, len(chunk_bases), chunk_bytes, fragment_bytes, dt,
          n_kv_heads, head_dim, ctypes.byref(out))
    return out


def lse_kv_arena_add_chunk(arena, chunk_base) -> int:
    first = ctypes.c_int32()
    _call(_lib.lse_kv_arena_add_chunk, arena, _ptr(chunk_base), ctypes.byref(first))
    return first.value


def lse_kv_arena_alloc(arena, n: int) -> np.ndarray:
    ids = np.zeros(max(n, 1), np.int32)
    _call(_lib.lse_kv_arena_alloc, arena, n, ids.ctypes.data_as(_i32p))
    return ids[:n]


def lse_kv_arena_free(arena, ids) -> None:
    a, p = _i32(ids)
    _call(_lib.lse_kv_arena_free, arena, len(a), p)


def lse_kv_arena_query(arena) -> dict:
    info = ArenaInfo()
    st = _lib.lse_kv_arena_query(arena, ctypes.byref(info))
    if st:
        raise LseError(st, "lse_kv_arena_query")
    return {k: getattr(info, k) for k, _ in ArenaInfo._fields_}


def lse_kv_arena_destroy(arena) -> None:
    _lib.lse_kv_arena_destroy(arena)


def lse_kv_arena_set_scales(arena, scales, n_floats: int | None = None) -> None:
    """Attach a device FP32 per-vector scale array (None removes it)."""
    if scales is None:
        _call(_lib.lse_kv_arena_set_scales, arena, None, 0)
        return
    n = int(n_floats if n_floats is not None else scales.numel())
    _call(_lib.lse_kv_arena_set_scales, arena, _ptr(scales), n)


# ---- plan --------------------------------------------------------------------

def lse_attn_plan(arena, n_seqs, max_rows_per_seq, max_total_rows, n_q_heads,
                  max_pages_per_seq):
    out, ws = _vp(), ctypes.c_size_t()
    _call(_lib.lse_attn_plan, arena, n_seqs, max_rows_per_seq, max_total_rows, n_q_heads,
          max_pages_per_seq, ctypes.byref(out), ctypes.byref(ws))
    return out, ws.value


def lse_attn_plan_ex(arena, n_seqs, max_rows_per_seq, max_total_rows, n_q_heads,
                     max_pages_per_seq, n_sms, smem_optin, ctas_per_sm=0, allow_tcgen05=1):
    lim = DeviceLimits(n_sms, smem_optin, ctas_per_sm, allow_tcgen05)
    out, ws = _vp(), ctypes.c_size_t()
    _call(_lib.lse_attn_plan_ex, arena, n_seqs, max_rows_per_seq, max_total_rows, n_q_heads,
          max_pages_per_seq, ctypes.byref(lim), ctypes.byref(out), ctypes.byref(ws))
    return out, ws.value


def lse_attn_plan_query(plan) -> dict:
    info = PlanInfo()
    st = _lib.lse_attn_plan_query(plan, ctypes.byref(info))
    if st:
        raise LseError(st, "lse_attn_plan_query")
    d = {k: getattr(info, k) for k, _ in PlanInfo._fields_}
    d["kernel_name"] = KERNELS.get(d["kernel"], "?")
    return d


def lse_attn_split_rule(capacity_keys, units, n_sms, ctas_per_sm, key_tile):
    kp = ctypes.c_int32()
    n = _lib.lse_attn_split_rule(capacity_keys, units, n_sms, ctas_per_sm, key_tile,
                                 ctypes.byref(kp))
    return n, kp.value


def lse_attn_workspace_init(plan, workspace, stream=0) -> None:
    _call(_lib.lse_attn_workspace_init, plan, _ptr(workspace), _ptr(stream))


def lse_attn_plan_destroy(plan) -> None:
    _lib.lse_attn_plan_destroy(plan)


# ---- run / merge / checks ---------------------------------------------------------

def lse_kv_append(arena, n_seqs, max_pages, k_new, v_new, k_pages, v_pages, seq_lens_before,
                  new_offsets, total_new, err_word=None, stream=0) -> None:
    """Write new tokens' FP32 K/V into their fragments, cast to the arena's
    format (device tensors; see include/lse_attn.h)."""
    _call(_lib.lse_kv_append, arena, int(n_seqs), int(max_pages), _ptr(k_new), _ptr(v_new),
          _ptr(k_pages), _ptr(v_pages), _ptr(seq_lens_before), _ptr(new_offsets),
          int(total_new), _ptr(err_word), _ptr(stream))


def lse_attn_run(plan, q, k_pages, v_pages, seq_lens, row_offsets, row_masks, softmax_scale,
                 workspace, stream=0) -> None:
    _call(_lib.lse_attn_run, plan, _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(seq_lens),
          _ptr(row_offsets), _ptr(row_masks), float(softmax_scale), _ptr(workspace),
          _ptr(stream))


def lse_attn_merge(plan, seq_lens, row_offsets, workspace, out, lse_out=None, stream=0) -> None:
    _call(_lib.lse_attn_merge, plan, _ptr(seq_lens), _ptr(row_offsets), _ptr(workspace),
          _ptr(out), _ptr(lse_out), _ptr(stream))


def lse_attn_forward(plan, q, k_pages, v_pages, seq_lens, row_offsets, row_masks, softmax_scale,
                     workspace, out, lse_out=None, stream=0) -> None:
    """Partial and merge passes in one call (one launch on tensor-core plans)."""
    _call(_lib.lse_attn_forward, plan, _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(seq_lens),
          _ptr(row_offsets), _ptr(row_masks), float(softmax_scale), _ptr(workspace), _ptr(out),
          _ptr(lse_out), _ptr(stream))


def lse_attn_validate(plan, k_pages, v_pages, seq_lens, row_offsets, row_masks=None) -> None:
    kp, kpp = _i32(k_pages)
    vp, vpp = _i32(v_pages)
    sl, slp = _i32(seq_lens)
    ro, rop = _i32(row_offsets)
    if row_masks is None:
        mp = None
    else:
        rm = np.ascontiguousarray(row_masks, dtype=np.uint64)
        mp = rm.ctypes.data_as(ctypes.POINTER(ctypes.c_uint64))
    _call(_lib.lse_attn_validate, plan, kpp, vpp, slp, rop, mp)


def lse_attn_forward_static(plan, q, k_pages, v_pages, seq_lens, row_offsets, row_masks,
                            softmax_scale, out, lse_out=None, stream=0) -> None:
    """Partial and merge passes on the library's static scratch (no
    device allocation; see include/lse_attn.h for the limits)."""
    _call(_lib.lse_attn_forward_static, plan, _ptr(q), _ptr(k_pages), _ptr(v_pages),
          _ptr(seq_lens), _ptr(row_offsets), _ptr(row_masks), float(softmax_scale), _ptr(out),
          _ptr(lse_out), _ptr(stream))


def lse_attn_test_withhold_tile(plan, tile: int) -> None:
    """Tests of the bounded waits: later launches skip loading each CTA's
    tile ``tile`` (-1 restores normal loading)."""
    st = _lib.lse_attn_test_withhold_tile(plan, int(tile))
    if st != LSE_OK:
        raise LseError(st, "lse_attn_test_withhold_tile")


def lse_attn_static_read_error(stream=0) -> int:
    """Read and clear the device error word of the static scratch (the
    latest lse_attn_forward_static call on the current device)."""
    v = ctypes.c_uint32()
    _call(_lib.lse_attn_static_read_error, _ptr(stream), ctypes.byref(v))
    return v.value


def lse_attn_read_error(plan, workspace, stream=0) -> int:
    v = ctypes.c_uint32()
    _call(_lib.lse_attn_read_error, plan, _ptr(workspace), _ptr(stream), ctypes.byref(v))
    return v.value


# ---- device-side convenience ------------------------------------------------------

class DeviceCall:
    """One problem resident on the current CUDA device, with its arena,
    plan, workspace and output; ``run()`` launches the partial and merge
    passes on ``stream``.

    ``problem`` is any object with the host fields of
    ``workloads.Workload`` (chunks, page tables, lengths, row offsets,
    masks, Q, shapes, scale).
    """

    def __init__(self, problem, max_total_rows=None, stream=None, plan_limits=None,
                 kernel="auto"):
        import torch
        self.torch = torch
        dev = torch.device("cuda", torch.cuda.current_device())
        if kernel != "auto" and plan_limits is None:
            props = torch.cuda.get_device_properties(dev)
            plan_limits = dict(n_sms=props.multi_processor_count,
                               smem_optin=getattr(props, "shared_memory_per_block_optin",
                                                  232448),
                               ctas_per_sm=0, allow_tcgen05=int(kernel == "tcgen05"))
        self.w = problem
        self.chunks = [torch.from_numpy(c).to(dev) for c in problem.chunks]
        # a step's inputs (Q, page tables, lengths, row offsets, masks) live in
        # one device buffer, mirrored by one pinned host buffer, so a step's
        # inputs go up in one copy (upload)
        host = [np.ascontiguousarray(problem.q, dtype=np.float32),
                np.ascontiguousarray(problem.k_pages, dtype=np.int32),
                np.ascontiguousarray(problem.v_pages, dtype=np.int32),
                np.ascontiguousarray(problem.seq_lens, dtype=np.int32),
                np.ascontiguousarray(problem.row_offsets, dtype=np.int32)]
        if problem.row_masks is not None:
            host.append(np.ascontiguousarray(problem.row_masks).view(np.int64))
        offs, total = [], 0
        for a in host:
            offs.append(total)
            total += (a.nbytes + 255) // 256 * 256
        packed = np.zeros(max(total, 256), np.uint8)
        for a, o in zip(host, offs):
            packed[o:o + a.nbytes] = a.reshape(-1).view(np.uint8)
        self.host_inputs = torch.from_numpy(packed).pin_memory()
        self.inputs = self.host_inputs.to(dev)
        views = [self.inputs[o:o + a.nbytes].view(torch.float32 if a.dtype == np.float32 else
                                                  torch.int64 if a.dtype == np.int64 else
                                                  torch.int32).view(a.shape)
                 for a, o in zip(host, offs)]
        self.q, self.k_pages, self.v_pages, self.seq_lens, self.row_offsets = views[:5]
        self.row_masks = views[5] if len(views) > 5 else None
        rows = int(problem.row_offsets[-1])
        self.total_rows = rows
        max_rows = max(1, int(np.max(np.diff(problem.row_offsets))))
        self.arena = lse_kv_arena_create(self.chunks, problem.chunk_bytes,
                                         problem.fragment_bytes, problem.dtype,
                                         problem.n_kv_heads, problem.head_dim)
        self.scales = None
        if getattr(problem, "scales", None) is not None:
            self.scales = torch.from_numpy(np.ascontiguousarray(problem.scales,
                                                                dtype=np.float32)).to(dev)
            lse_kv_arena_set_scales(self.arena, self.scales)
        mtr = max(1, max_total_rows or rows)
        if plan_limits is None:
            self.plan, ws = lse_attn_plan(self.arena, len(problem.seq_lens), max_rows, mtr,
                                          problem.n_q_heads, problem.k_pages.shape[1])
        else:
            self.plan, ws = lse_attn_plan_ex(self.arena, len(problem.seq_lens), max_rows, mtr,
                                             problem.n_q_heads, problem.k_pages.shape[1],
                                             **plan_limits)
        self.info = lse_attn_plan_query(self.plan)
        if kernel != "auto" and self.info["kernel_name"] != kernel:
            raise LseError(2, f"plan chose {self.info['kernel_name']}, not {kernel}")
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        lse_attn_workspace_init(self.plan, self.workspace, self.stream)
        # out and lse in one device buffer (one copy back: download)
        n_out = max(rows, 1) * problem.n_q_heads * problem.head_dim
        n_lse = max(rows, 1) * problem.n_q_heads
        self.outputs = torch.empty(n_out + (n_lse + 63) // 64 * 64, dtype=torch.float32,
                                   device=dev)
        self.out = self.outputs[:n_out].view(max(rows, 1), problem.n_q_heads, problem.head_dim)
        self.lse = self.outputs[n_out:n_out + n_lse].view(max(rows, 1), problem.n_q_heads)
        self.scale = float(problem.scale)

    def upload(self, host_inputs=None):
        """Copy a step's packed inputs (the layout of ``host_inputs``, a
        pinned uint8 tensor) to the device in one copy on ``stream``."""
        src = self.host_inputs if host_inputs is None else host_inputs
        with self.torch.cuda.stream(self._torch_stream()):
            self.inputs.copy_(src, non_blocking=True)

    def download(self, host_outputs):
        """Copy out and lse (packed, FP32) into a pinned host tensor of
        ``outputs.numel()`` floats in one copy on ``stream``."""
        with self.torch.cuda.stream(self._torch_stream()):
            host_outputs.copy_(self.outputs, non_blocking=True)

    def _torch_stream(self):
        s = self.stream
        if isinstance(s, self.torch.cuda.Stream):
            return s
        return self.torch.cuda.current_stream()

    def run_partial(self):
        lse_attn_run(self.plan, self.q, self.k_pages, self.v_pages, self.seq_lens,
                     self.row_offsets, self.row_masks, self.scale, self.workspace, self.stream)

    def run_merge(self):
        lse_attn_merge(self.plan, self.seq_lens, self.row_offsets, self.workspace, self.out,
                       self.lse, self.stream)

    def run(self):
        """Both passes through lse_attn_forward (on tensor-core plans, one
        launch with the merge fused)."""
        lse_attn_forward(self.plan, self.q, self.k_pages, self.v_pages, self.seq_lens,
                         self.row_offsets, self.row_masks, self.scale, self.workspace, self.out,
                         self.lse, self.stream)
        return self.out, self.lse

    def run_two_pass(self):
        """lse_attn_run then lse_attn_merge (partials through the workspace)."""
        self.run_partial()
        self.run_merge()
        return self.out, self.lse

    def device_error(self) -> int:
        return lse_attn_read_error(self.plan, self.workspace, self.stream)

    def close(self):
        if self.plan:
            lse_attn_plan_destroy(self.plan)
            self.plan = None
        if self.arena:
            lse_kv_arena_destroy(self.arena)
            self.arena = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
