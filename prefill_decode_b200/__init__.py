"""Python binding of the fused hybrid-batch attention C ABI (``include/pod_attn.h``).

Argument marshalling only: every step of the attention runs in the CUDA kernels
of ``libpod_attn.so``; the planner runs in its C++ host code.  Tensors may be
torch tensors (anything with ``data_ptr()``) or raw integer addresses.  There is
no fallback: if the library is missing, importing the binding's entry points
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpod_attn.so")

POD_OK = 0
POD_ERR_INVALID_ARG = -1
POD_ERR_UNSUPPORTED = -2
POD_ERR_WORKSPACE = -3
POD_ERR_CUDA = -4
POD_ERR_BOUNDS = -5
POD_ERR_TIMEOUT = -6
POD_ERR_PLAN_MISMATCH = -7
POD_FLAG_SEQUENTIAL = 1
POD_FLAG_TRACE = 2
POD_FLAG_MERGE_KERNEL = 4
POD_FLAG_SELFTEST_TIMEOUT = 8
POD_FLAG_TWO_STREAMS = 16
POD_FLAG_SM_PARTITION = 32
POD_FLAG_DECODE_FOUR_WARPS = 64
POD_FLAG_PREFILL_SPLIT_UNLIMITED = 128

EXPORTED = [
    "pod_attn_plan", "pod_attn_plan_get_info", "pod_attn_plan_tables", "pod_attn_upload", "pod_attn_run",
    "pod_attn_plan_set_events", "pod_attn_event_create", "pod_attn_event_destroy", "pod_attn_event_elapsed_ms",
    "pod_attn_plan_destroy", "pod_attn_status_string", "pod_attn_last_cuda_error", "pod_attn_run_static",
    "pod_attn_plan_batched", "pod_attn_plan_prefill_requests", "pod_attn_plan_prefill_merges",
    "pod_attn_run_fp8kv",
]


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_q_heads", "num_kv_heads", "head_dim", "page_size", "num_sms", "ctas_per_sm",
        "ratio_prefill", "ratio_decode", "max_waves", "min_chunk_pages", "max_prefill_splits")] + [
            ("flags", ctypes.c_uint32)]


class PlanInfo(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "num_prefill_items", "num_decode_items", "num_merge_items", "num_partials", "ctas_per_sm",
        "ratio_prefill", "ratio_decode", "chunk_pages", "num_sms", "grid")] + [(n, ctypes.c_int64) for n in (
            "workspace_bytes", "error_offset", "prefill_flops", "decode_flops", "kv_bytes", "qo_bytes", "table_bytes")] + [
            (n, ctypes.c_int32) for n in ("num_prefill_requests", "num_prefill_rows", "num_prefill_partials",
                                          "num_prefill_merge_items")] + [("rescale_count_offset", ctypes.c_int64)]


class PodError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libpod_attn.so (build it first with prefill_decode_b200.build.build())."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m prefill_decode_b200.build` "
                               "(or __graft_entry__.build()); there is no fallback path")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        L.pod_attn_plan.argtypes = [ctypes.POINTER(Config), i32, i32, i32, ctypes.POINTER(i32),
                                    ctypes.POINTER(vp), ctypes.POINTER(sz)]
        L.pod_attn_plan_batched.argtypes = [ctypes.POINTER(Config), i32, ctypes.POINTER(i32), ctypes.POINTER(i32),
                                            i32, ctypes.POINTER(i32), ctypes.POINTER(vp), ctypes.POINTER(sz)]
        L.pod_attn_plan_prefill_requests.argtypes = [vp, vp]
        L.pod_attn_plan_prefill_merges.argtypes = [vp, vp]
        L.pod_attn_plan_get_info.argtypes = [vp, ctypes.POINTER(PlanInfo)]
        L.pod_attn_plan_tables.argtypes = [vp, vp, vp, vp]
        L.pod_attn_upload.argtypes = [vp, vp, sz, vp]
        L.pod_attn_run.argtypes = [vp, vp, vp, vp, vp, i64, vp, i32, vp, ctypes.c_float, vp, vp, vp, sz, vp, vp]
        L.pod_attn_plan_set_events.argtypes = [vp, vp, vp]
        L.pod_attn_event_create.argtypes = [ctypes.POINTER(vp)]
        L.pod_attn_event_destroy.argtypes = [vp]
        L.pod_attn_event_elapsed_ms.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_float)]
        L.pod_attn_plan_destroy.argtypes = [vp]
        L.pod_attn_plan_destroy.restype = None
        L.pod_attn_status_string.argtypes = [ctypes.c_int]
        L.pod_attn_status_string.restype = ctypes.c_char_p
        L.pod_attn_last_cuda_error.argtypes = []
        L.pod_attn_run_static.argtypes = [vp, vp, vp, vp, vp, i64, vp, i32, vp, ctypes.c_float, vp, vp, vp]
        L.pod_attn_run_fp8kv.argtypes = [vp, vp, vp, vp, vp, i64, vp, vp, i64, vp, vp, vp, i32, vp, ctypes.c_float,
                                         vp, vp, vp, sz, vp, vp]
        for n in EXPORTED:
            if n not in ("pod_attn_plan_destroy", "pod_attn_status_string"):
                getattr(L, n).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().pod_attn_status_string(int(s)).decode()


def _check(s: int, what: str) -> None:
    if s != POD_OK:
        if s == POD_ERR_CUDA:
            raise PodError(s, f"{what} (cudaError {lib().pod_attn_last_cuda_error()})")
        raise PodError(s, what)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


class Plan:
    """Host-side schedule of one hybrid batch.  ``prefill_len`` / ``prefill_kv_len``
    are ints for one prefill request (``pod_attn_plan``: block-table row 0,
    decodes from row 1) or equal-length sequences for several
    (``pod_attn_plan_batched``: rows 0..NP-1, decodes from row NP)."""

    def __init__(self, num_q_heads: int, num_kv_heads: int, head_dim: int, prefill_len,
                 prefill_kv_len, decode_lens: Sequence[int], *, num_sms: int = 0,
                 ctas_per_sm: int = 0, ratio: Tuple[int, int] = (0, 0), max_waves: int = 0,
                 min_chunk_pages: int = 0, max_prefill_splits: int = 0, flags: int = 0, page_size: int = 16):
        L = lib()
        self.cfg = Config(num_q_heads, num_kv_heads, head_dim, page_size, num_sms, ctas_per_sm,
                          ratio[0], ratio[1], max_waves, min_chunk_pages, max_prefill_splits, flags)
        lens = np.ascontiguousarray(np.asarray(decode_lens, dtype=np.int32))
        self._lens = lens
        h = ctypes.c_void_p()
        ws = ctypes.c_size_t()
        lp = lens.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)) if lens.size else None
        if np.ndim(prefill_len) == 0:
            _check(L.pod_attn_plan(ctypes.byref(self.cfg), int(prefill_len), int(prefill_kv_len), int(lens.size),
                                   lp, ctypes.byref(h), ctypes.byref(ws)), "pod_attn_plan")
        else:
            qo = np.ascontiguousarray(np.asarray(prefill_len, dtype=np.int32))
            kv = np.ascontiguousarray(np.asarray(prefill_kv_len, dtype=np.int32))
            if qo.shape != kv.shape:
                raise ValueError("prefill_len and prefill_kv_len differ in length")
            self._pre = (qo, kv)
            qp = qo.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)) if qo.size else None
            kp = kv.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)) if kv.size else None
            _check(L.pod_attn_plan_batched(ctypes.byref(self.cfg), int(qo.size), qp, kp, int(lens.size), lp,
                                           ctypes.byref(h), ctypes.byref(ws)), "pod_attn_plan_batched")
        self._h = h
        self.workspace_bytes = int(ws.value)
        self.info = PlanInfo()
        _check(L.pod_attn_plan_get_info(self._h, ctypes.byref(self.info)), "pod_attn_plan_get_info")

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.pod_attn_plan_destroy(h)
            self._h = None

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def prefill_requests(self) -> np.ndarray:
        """int32 [NP, 4]: first row in q_prefill, P_i, C_i, 0."""
        out = np.zeros((self.info.num_prefill_requests, 4), dtype=np.int32)
        _check(lib().pod_attn_plan_prefill_requests(self._h, out.ctypes.data), "pod_attn_plan_prefill_requests")
        return out

    def prefill_merges(self) -> np.ndarray:
        """int32 [num_prefill_merge_items, 4]: first partial, pieces, 0, 0."""
        out = np.zeros((self.info.num_prefill_merge_items, 4), dtype=np.int32)
        _check(lib().pod_attn_plan_prefill_merges(self._h, out.ctypes.data), "pod_attn_plan_prefill_merges")
        return out

    def tables(self):
        """Host copies of the prefill items [n, 8], decode items [n, 8] and decode merge items [n, 4]."""
        i = self.info
        pre = np.zeros((i.num_prefill_items, 8), dtype=np.int32)
        dec = np.zeros((i.num_decode_items, 8), dtype=np.int32)
        mer = np.zeros((i.num_merge_items, 4), dtype=np.int32)
        _check(lib().pod_attn_plan_tables(self._h, pre.ctypes.data, dec.ctypes.data, mer.ctypes.data),
               "pod_attn_plan_tables")
        return pre, dec, mer

    def upload(self, workspace, stream=None) -> None:
        nbytes = workspace.numel() * workspace.element_size() if hasattr(workspace, "numel") else self.workspace_bytes
        _check(lib().pod_attn_upload(self._h, _ptr(workspace), nbytes, _stream(stream)), "pod_attn_upload")

    def run(self, q_prefill, q_decode, k_cache, v_cache, num_blocks: int, block_table, block_table_stride: int,
            kv_lens, scale: float, o_prefill, o_decode, workspace, trace=None, stream=None,
            workspace_bytes: Optional[int] = None) -> None:
        if workspace_bytes is None:
            workspace_bytes = (workspace.numel() * workspace.element_size()
                               if hasattr(workspace, "numel") else self.workspace_bytes)
        _check(lib().pod_attn_run(self._h, _ptr(q_prefill), _ptr(q_decode), _ptr(k_cache), _ptr(v_cache),
                                  int(num_blocks), _ptr(block_table), int(block_table_stride), _ptr(kv_lens),
                                  float(scale), _ptr(o_prefill), _ptr(o_decode), _ptr(workspace),
                                  int(workspace_bytes), _ptr(trace), _stream(stream)), "pod_attn_run")

    def run_fp8kv(self, q_prefill, q_decode, k_cache, v_cache, num_blocks: int, k_cache_fp8, v_cache_fp8,
                  num_blocks_fp8: int, k_scale, v_scale, block_table, block_table_stride: int, kv_lens,
                  scale: float, o_prefill, o_decode, workspace, trace=None, stream=None,
                  workspace_bytes: Optional[int] = None) -> None:
        """pod_attn_run_fp8kv: the decode requests read the e4m3 pools (uint8) with per-kv-head fp32
        scales; the prefill requests read the bf16 pools."""
        if workspace_bytes is None:
            workspace_bytes = (workspace.numel() * workspace.element_size()
                               if hasattr(workspace, "numel") else self.workspace_bytes)
        _check(lib().pod_attn_run_fp8kv(self._h, _ptr(q_prefill), _ptr(q_decode), _ptr(k_cache), _ptr(v_cache),
                                        int(num_blocks), _ptr(k_cache_fp8), _ptr(v_cache_fp8), int(num_blocks_fp8),
                                        _ptr(k_scale), _ptr(v_scale), _ptr(block_table), int(block_table_stride),
                                        _ptr(kv_lens), float(scale), _ptr(o_prefill), _ptr(o_decode),
                                        _ptr(workspace), int(workspace_bytes), _ptr(trace), _stream(stream)),
               "pod_attn_run_fp8kv")

    def set_events(self, ev_start: Optional[int], ev_stop: Optional[int]) -> None:
        _check(lib().pod_attn_plan_set_events(self._h, ev_start, ev_stop), "pod_attn_plan_set_events")


class Event:
    """A cudaEvent_t made by the library (for timing the main kernel)."""

    def __init__(self):
        h = ctypes.c_void_p()
        _check(lib().pod_attn_event_create(ctypes.byref(h)), "pod_attn_event_create")
        self.handle = h.value

    def __del__(self):
        if getattr(self, "handle", None) and _lib is not None:
            _lib.pod_attn_event_destroy(self.handle)
            self.handle = None

    def elapsed_ms(self, stop: "Event") -> float:
        ms = ctypes.c_float()
        _check(lib().pod_attn_event_elapsed_ms(self.handle, stop.handle, ctypes.byref(ms)), "event elapsed")
        return float(ms.value)
