"""GQA decode attention over a paged KV cache with dynamic split-KV scheduling, for
NVIDIA B200 (sm_100a).

This module is the Python face of ``libdecattn.so`` (C ABI in ``include/decattn.h``):
it only marshals torch tensors into pointers and sizes. Every step of the work --
planning, the split kernel, the combine -- runs in the library's CUDA kernels. If the
library is missing, every call raises; there is no fallback.

Typical use (one plan per decode step, reused by every layer)::

    pl = plan(seq_lens, n_kv_heads=8, tile_len=256, max_total_kv_tokens=total)
    out, lse = run(q, k_pages, v_pages, page_table, seq_lens, pl)
"""
from __future__ import annotations

import ctypes as C
import math
import os
import threading
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdecattn.so")

OK, EINVAL, ENOTSUP, ESMALL, ECUDA, ETIMEOUT, EDEVICE, EALIGN, ECAPACITY = 0, -1, -2, -3, -4, -5, -6, -7, -8
KV_BF16, KV_FP8E4M3, KV_FP8E4M3_MMA8 = 0, 1, 2
API = ("dec_attn_default_bins", "dec_attn_default_tile_len", "dec_attn_plan_bytes", "dec_attn_plan", "dec_attn_plan_export",
       "dec_attn_workspace_bytes", "dec_attn_run", "dec_attn_split", "dec_attn_combine", "dec_attn_run_noalloc",
       "dec_attn_read_status", "dec_attn_status_string", "dec_attn_append_rope", "dec_attn_append_rope_fp8", "dec_attn_prefill",
       "dec_attn_prefill_varlen", "dec_attn_prefill_fp8_workspace_bytes", "dec_attn_prefill_fp8",
       "dec_attn_plan_sparse_bytes",
       "dec_attn_plan_sparse", "dec_attn_last_error", "dec_attn_test_set_waits")
NOALLOC_SCRATCH_BYTES = 64 << 20


class DecAttnError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        msg = f"{what}: {status_string(code)} ({code})" if what else f"{status_string(code)} ({code})"
        if code == ECUDA:
            detail = last_error()
            if detail:
                msg += f" [{detail}]"
        super().__init__(msg)


class PlanT(C.Structure):
    _fields_ = [("buf", C.c_void_p), ("buf_bytes", C.c_size_t), ("batch", C.c_int32), ("n_kv_heads", C.c_int32),
                ("tile_len", C.c_int32), ("n_bins", C.c_int32), ("max_units", C.c_int64),
                ("sparse", C.c_int32), ("reserved_", C.c_int32)]


class ShapeT(C.Structure):
    _fields_ = [("batch", C.c_int32), ("n_q_heads", C.c_int32), ("n_kv_heads", C.c_int32), ("head_dim", C.c_int32),
                ("q_tokens", C.c_int32), ("page_size", C.c_int32), ("num_pages", C.c_int32),
                ("max_pages_per_seq", C.c_int32), ("kv_dtype", C.c_int32), ("sm_scale", C.c_float)]


_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH):
    """Loads libdecattn.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m paged_kv_decode_29_b200.build` "
                               "(or __graft_entry__.build()); there is no fallback path")
        lib = C.CDLL(path)
        vp, i32, i64, sz = C.c_void_p, C.c_int, C.c_int64, C.c_size_t
        lib.dec_attn_default_bins.argtypes = [i32]
        lib.dec_attn_default_bins.restype = i32
        lib.dec_attn_default_tile_len.argtypes = [i32, i32, i64, i32, i32, i32, i32, i32]
        lib.dec_attn_default_tile_len.restype = i32
        lib.dec_attn_plan_bytes.argtypes = [i32, i32, i32, i64, i32]
        lib.dec_attn_plan_bytes.restype = sz
        lib.dec_attn_plan.argtypes = [vp, i32, i32, i32, i64, i32, vp, sz, C.POINTER(PlanT), vp]
        lib.dec_attn_plan.restype = i32
        lib.dec_attn_plan_export.argtypes = [C.POINTER(PlanT), vp, vp, vp, i64, vp, vp]
        lib.dec_attn_plan_export.restype = i32
        lib.dec_attn_workspace_bytes.argtypes = [C.POINTER(ShapeT), C.POINTER(PlanT)]
        lib.dec_attn_workspace_bytes.restype = sz
        for name in ("dec_attn_run", "dec_attn_split", "dec_attn_combine"):
            f = getattr(lib, name)
            f.argtypes = [C.POINTER(ShapeT), vp, vp, vp, vp, vp, vp, C.POINTER(PlanT), vp, sz, vp, vp, vp]
            f.restype = i32
        lib.dec_attn_run_noalloc.argtypes = [C.POINTER(ShapeT), vp, vp, vp, vp, vp, vp, C.POINTER(PlanT), vp, vp, vp]
        lib.dec_attn_run_noalloc.restype = i32
        lib.dec_attn_read_status.argtypes = [C.POINTER(PlanT), vp, vp]
        lib.dec_attn_read_status.restype = i32
        lib.dec_attn_status_string.argtypes = [i32]
        lib.dec_attn_status_string.restype = C.c_char_p
        lib.dec_attn_last_error.argtypes = [C.c_char_p, sz]
        lib.dec_attn_last_error.restype = sz
        lib.dec_attn_append_rope.argtypes = [C.POINTER(ShapeT), vp, vp, vp, vp, vp, C.c_float, vp, vp, vp, vp, vp]
        lib.dec_attn_plan_sparse_bytes.argtypes = [i32, i32, i32, i64, i32]
        lib.dec_attn_plan_sparse_bytes.restype = sz
        lib.dec_attn_plan_sparse.argtypes = [vp, vp, i32, i32, i32, i32, i64, i32, vp, sz, C.POINTER(PlanT), vp]
        lib.dec_attn_plan_sparse.restype = i32
        lib.dec_attn_append_rope.restype = i32
        lib.dec_attn_prefill.argtypes = [C.POINTER(ShapeT), vp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.dec_attn_prefill.restype = i32
        lib.dec_attn_append_rope_fp8.argtypes = [C.POINTER(ShapeT), vp, vp, vp, vp, vp, C.c_float, vp, vp, vp, vp,
                                                 vp, vp]
        lib.dec_attn_append_rope_fp8.restype = i32
        lib.dec_attn_prefill_varlen.argtypes = [C.POINTER(ShapeT), vp, vp, vp, vp, vp, vp, i64, vp, vp, vp, vp]
        lib.dec_attn_prefill_varlen.restype = i32
        lib.dec_attn_prefill_fp8_workspace_bytes.argtypes = [C.POINTER(ShapeT)]
        lib.dec_attn_prefill_fp8_workspace_bytes.restype = i64
        lib.dec_attn_prefill_fp8.argtypes = [C.POINTER(ShapeT), vp, vp, vp, vp, vp, vp, vp, i64, vp, i64, vp, vp, vp,
                                             vp]
        lib.dec_attn_prefill_fp8.restype = i32
        lib.dec_attn_test_set_waits.argtypes = [C.c_uint64, C.c_int32]
        lib.dec_attn_test_set_waits.restype = i32
        _lib = lib
        return lib


def status_string(code: int) -> str:
    return load_library().dec_attn_status_string(int(code)).decode()


def last_error() -> str:
    """dec_attn_last_error: the failing step and CUDA error behind this thread's last ECUDA ('' if none)."""
    lib = load_library()
    n = int(lib.dec_attn_last_error(None, 0))
    if n == 0:
        return ""
    buf = C.create_string_buffer(n + 1)
    lib.dec_attn_last_error(buf, n + 1)
    return buf.value.decode(errors="replace")


def _stream_handle(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    h = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return h or None


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


@dataclass
class Plan:
    """A plan: the device buffer holding the work list and its host handle."""
    buf: torch.Tensor
    handle: PlanT

    @property
    def n_bins(self) -> int:
        return int(self.handle.n_bins)

    @property
    def tile_len(self) -> int:
        return int(self.handle.tile_len)


def default_bins(device: int | None = None) -> int:
    dev = torch.cuda.current_device() if device is None else int(device)
    n = load_library().dec_attn_default_bins(dev)
    if n <= 0:
        raise DecAttnError(ECUDA, "dec_attn_default_bins")
    return n


def default_tile_len(batch: int, n_kv_heads: int, total_kv_tokens: int, page_size: int, head_dim: int,
                     rows_per_kv_head: int, kv_dtype: int = KV_BF16, n_bins: int | None = None) -> int:
    """dec_attn_default_tile_len: the tile length that minimises the library's estimate of the
    busiest CTA's bytes (host only when ``n_bins`` is given; else the current device's bins)."""
    nb = default_bins() if n_bins is None else int(n_bins)
    tl = load_library().dec_attn_default_tile_len(batch, n_kv_heads, int(total_kv_tokens), page_size, head_dim,
                                                  rows_per_kv_head, kv_dtype, nb)
    if tl <= 0:
        raise DecAttnError(tl, "dec_attn_default_tile_len")
    return int(tl)


def plan_bytes(batch: int, n_kv_heads: int, tile_len: int, max_total_kv_tokens: int, n_bins: int = 0) -> int:
    return int(load_library().dec_attn_plan_bytes(batch, n_kv_heads, tile_len, int(max_total_kv_tokens), n_bins))


def plan(seq_lens: torch.Tensor, n_kv_heads: int, tile_len: int, max_total_kv_tokens: int | None = None,
         n_bins: int = 0, buf: torch.Tensor | None = None, stream=None) -> Plan:
    """Enqueues the planner (one single-block kernel) on ``stream``.

    ``seq_lens``: int32 CUDA tensor [B]. ``max_total_kv_tokens`` bounds sum(seq_lens) and sizes the
    plan buffer (None: read it from ``seq_lens``, which synchronises)."""
    lib = load_library()
    assert seq_lens.is_cuda and seq_lens.dtype == torch.int32 and seq_lens.is_contiguous()
    B = int(seq_lens.numel())
    if max_total_kv_tokens is None:
        max_total_kv_tokens = int(seq_lens.sum().item()) if B else 0
    nbytes = lib.dec_attn_plan_bytes(B, n_kv_heads, tile_len, int(max_total_kv_tokens), n_bins)
    if nbytes == 0:
        raise DecAttnError(ENOTSUP, "dec_attn_plan_bytes")
    if buf is None:
        buf = torch.empty(nbytes, dtype=torch.uint8, device=seq_lens.device)
    h = PlanT()
    rc = lib.dec_attn_plan(_ptr(seq_lens), B, n_kv_heads, tile_len, int(max_total_kv_tokens), n_bins,
                           buf.data_ptr(), buf.numel(), C.byref(h), _stream_handle(stream))
    if rc != OK:
        raise DecAttnError(rc, "dec_attn_plan")
    return Plan(buf=buf, handle=h)


def plan_sparse(seq_lens: torch.Tensor, tile_mask: torch.Tensor, n_kv_heads: int, tile_len: int,
                max_total_kv_tokens: int | None = None, n_bins: int = 0, buf: torch.Tensor | None = None,
                stream=None) -> Plan:
    """Enqueues the block-sparse planner: only the tiles whose bit is set in ``tile_mask`` (int32 or
    uint32-valued CUDA tensor [B][n_kv_heads][words], bit i of (b, h) keeps tile i) enter the work
    list. The plan is then used with ``run`` like a dense one."""
    lib = load_library()
    assert seq_lens.is_cuda and seq_lens.dtype == torch.int32 and seq_lens.is_contiguous()
    assert tile_mask.is_cuda and tile_mask.dtype == torch.int32 and tile_mask.is_contiguous()
    B = int(seq_lens.numel())
    assert tile_mask.dim() == 3 and tile_mask.shape[0] == B and tile_mask.shape[1] == n_kv_heads
    if max_total_kv_tokens is None:
        max_total_kv_tokens = int(seq_lens.sum().item()) if B else 0
    nbytes = lib.dec_attn_plan_sparse_bytes(B, n_kv_heads, tile_len, int(max_total_kv_tokens), n_bins)
    if nbytes == 0:
        raise DecAttnError(ENOTSUP, "dec_attn_plan_sparse_bytes")
    if buf is None:
        buf = torch.empty(nbytes, dtype=torch.uint8, device=seq_lens.device)
    h = PlanT()
    rc = lib.dec_attn_plan_sparse(_ptr(seq_lens), _ptr(tile_mask), int(tile_mask.shape[2]), B, n_kv_heads, tile_len,
                                  int(max_total_kv_tokens), n_bins, buf.data_ptr(), buf.numel(), C.byref(h),
                                  _stream_handle(stream))
    if rc != OK:
        raise DecAttnError(rc, "dec_attn_plan_sparse")
    return Plan(buf=buf, handle=h)


def make_shape(q: torch.Tensor, k_pages: torch.Tensor, page_table: torch.Tensor, kv_dtype: int,
               sm_scale: float = 0.0) -> ShapeT:
    B, T, Hq, d = q.shape
    num_pages, Hkv, P, d2 = k_pages.shape
    assert d == d2
    return ShapeT(B, Hq, Hkv, d, T, P, num_pages, int(page_table.shape[1]), kv_dtype, float(sm_scale))


def kv_dtype_of(k_pages: torch.Tensor) -> int:
    if k_pages.dtype == torch.bfloat16:
        return KV_BF16
    if k_pages.dtype in (torch.uint8, torch.float8_e4m3fn):
        return KV_FP8E4M3
    raise TypeError(f"KV pool dtype {k_pages.dtype} is not bf16 / e4m3")


def workspace_bytes(shape: ShapeT, pl: Plan) -> int:
    n = load_library().dec_attn_workspace_bytes(C.byref(shape), C.byref(pl.handle))
    if n == 0:
        raise DecAttnError(ENOTSUP, "dec_attn_workspace_bytes")
    return int(n)


def run(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, page_table: torch.Tensor,
        seq_lens: torch.Tensor, pl: Plan, *, kv_scales: torch.Tensor | None = None, sm_scale: float = 0.0,
        workspace: torch.Tensor | None = None, out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
        stream=None, stage: str = "run", mma8: bool = False):
    """Enqueues split + combine on ``stream``; returns (out fp32 [B][T][Hq][d], lse fp32 [B][T][Hq]).

    q: bf16 [B][T][Hq][d]; k_pages / v_pages: [num_pages][Hkv][P][d] bf16, or uint8 / float8_e4m3fn
    E4M3 codes with ``kv_scales`` fp32 [2][num_pages][Hkv]; page_table: int32 [B][max_pages_per_seq];
    seq_lens: int32 [B] (the values the plan was made from). ``stage``: "run" (split + combine), or
    "split" / "combine" alone (the combine reads the partials the split left in ``workspace``).
    ``mma8``: E4M3 pages with both products on E4M3 tensor cores (KV_FP8E4M3_MMA8: q and P rounded
    to E4M3; head_dim 128, G*T <= 16)."""
    lib = load_library()
    kvt = kv_dtype_of(k_pages)
    if mma8:
        if kvt != KV_FP8E4M3:
            raise ValueError("mma8 needs E4M3 pages")
        kvt = KV_FP8E4M3_MMA8
    shape = make_shape(q, k_pages, page_table, kvt, sm_scale)
    B, T, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, T, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, T, Hq), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(workspace_bytes(shape, pl), dtype=torch.uint8, device=q.device)
    fn = {"run": lib.dec_attn_run, "split": lib.dec_attn_split, "combine": lib.dec_attn_combine}[stage]
    rc = fn(C.byref(shape), _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table), _ptr(seq_lens),
            _ptr(kv_scales), C.byref(pl.handle), _ptr(workspace), workspace.numel(), _ptr(out), _ptr(lse),
            _stream_handle(stream))
    if rc != OK:
        raise DecAttnError(rc, f"dec_attn_{stage}")
    return out, lse


def run_noalloc(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, page_table: torch.Tensor,
                seq_lens: torch.Tensor, pl: Plan, out: torch.Tensor, lse: torch.Tensor, *,
                kv_scales: torch.Tensor | None = None, sm_scale: float = 0.0, stream=None):
    """dec_attn_run_noalloc: split + combine using the library's fixed 64 MiB device scratch instead
    of a caller workspace, for callers that cannot allocate device memory. ``out`` and ``lse`` are
    caller-provided (this wrapper allocates nothing either). Calls overlapping on the GPU race on the
    shared scratch."""
    lib = load_library()
    shape = make_shape(q, k_pages, page_table, kv_dtype_of(k_pages), sm_scale)
    rc = lib.dec_attn_run_noalloc(C.byref(shape), _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table),
                                  _ptr(seq_lens), _ptr(kv_scales), C.byref(pl.handle), _ptr(out), _ptr(lse),
                                  _stream_handle(stream))
    if rc != OK:
        raise DecAttnError(rc, "dec_attn_run_noalloc")
    return out, lse


def append_rope(q_new: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, page_table: torch.Tensor,
                seq_lens: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, *,
                q_out: torch.Tensor | None = None, rope_base: float = 10000.0,
                status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """dec_attn_append_rope: rotary embedding of the step's new q / k rows and the append of the
    new K/V rows into their pages (bf16 pools, updated in place); returns the rotated q.

    q_new: bf16 [B][T][Hq][d]; k_new / v_new: bf16 [B][T][Hkv][d]; seq_lens: int32 [B], counting the
    T new tokens (token t of request b sits at position Lb - T + t); ``status``: optional int32
    device scalar that receives DECATTN_EDEVICE for a bad page id."""
    lib = load_library()
    shape = make_shape(q_new, k_pages, page_table, kv_dtype_of(k_pages))
    if q_out is None:
        q_out = torch.empty_like(q_new)
    rc = lib.dec_attn_append_rope(C.byref(shape), _ptr(q_new), _ptr(k_new), _ptr(v_new), _ptr(page_table),
                                  _ptr(seq_lens), float(rope_base), _ptr(q_out), _ptr(k_pages), _ptr(v_pages),
                                  _ptr(status), _stream_handle(stream))
    if rc != OK:
        raise DecAttnError(rc, "dec_attn_append_rope")
    return q_out


def append_rope_fp8(q_new: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, page_table: torch.Tensor,
                    seq_lens: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, kv_scales: torch.Tensor,
                    *, rope_base: float = 10000.0, q_out: torch.Tensor | None = None,
                    status: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """dec_attn_append_rope_fp8: the fused pre-processing over an E4M3 cache (k_pages / v_pages uint8
    or float8_e4m3fn codes [num_pages][Hkv][P][d], kv_scales fp32 [2][num_pages][Hkv], all updated in
    place); returns the rotated q."""
    lib = load_library()
    B, T, Hq, d = q_new.shape
    num_pages, Hkv, P, d2 = k_pages.shape
    shape = ShapeT(B, Hq, Hkv, d, T, P, num_pages, int(page_table.shape[1]), KV_FP8E4M3, 0.0)
    if q_out is None:
        q_out = torch.empty_like(q_new)
    rc = lib.dec_attn_append_rope_fp8(C.byref(shape), _ptr(q_new), _ptr(k_new), _ptr(v_new), _ptr(page_table),
                                      _ptr(seq_lens), float(rope_base), _ptr(q_out), _ptr(k_pages), _ptr(v_pages),
                                      _ptr(kv_scales), _ptr(status), _stream_handle(stream))
    if rc != OK:
        raise DecAttnError(rc, "dec_attn_append_rope_fp8")
    return q_out


def prefill(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, page_table: torch.Tensor,
            seq_lens: torch.Tensor, *, sm_scale: float = 0.0, out: torch.Tensor | None = None,
            lse: torch.Tensor | None = None, status: torch.Tensor | None = None, stream=None):
    """dec_attn_prefill: causal attention of the T query rows of each request (its last T
    positions, already in the bf16 pages) over its paged KV; returns (out fp32 [B][T][Hq][128],
    lse fp32 [B][T][Hq]). ``status``: optional int32 device scalar (DECATTN_EDEVICE /
    DECATTN_ETIMEOUT)."""
    lib = load_library()
    shape = make_shape(q, k_pages, page_table, kv_dtype_of(k_pages), sm_scale)
    B, T, Hq, d = q.shape
    if out is None:
        out = torch.empty((B, T, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, T, Hq), dtype=torch.float32, device=q.device)
    rc = lib.dec_attn_prefill(C.byref(shape), _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table),
                              _ptr(seq_lens), _ptr(out), _ptr(lse), _ptr(status), _stream_handle(stream))
    if rc != OK:
        raise DecAttnError(rc, "dec_attn_prefill")
    return out, lse


def prefill_varlen(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, page_table: torch.Tensor,
                   seq_lens: torch.Tensor, cu_q_lens: torch.Tensor, max_q_rows: int, *, sm_scale: float = 0.0,
                   out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                   status: torch.Tensor | None = None, stream=None):
    """dec_attn_prefill_varlen: request b's rows are the packed rows cu_q_lens[b] .. cu_q_lens[b+1]-1
    of q [total][Hq][128] (its last Tb positions); ``max_q_rows`` bounds every Tb. Returns (out fp32
    [total][Hq][128], lse fp32 [total][Hq])."""
    lib = load_library()
    total, Hq, d = q.shape
    B = page_table.shape[0]
    shape = ShapeT(B, Hq, k_pages.shape[1], d, int(max_q_rows), k_pages.shape[2], k_pages.shape[0],
                   page_table.shape[1], kv_dtype_of(k_pages), float(sm_scale))
    if out is None:
        out = torch.empty((total, Hq, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((total, Hq), dtype=torch.float32, device=q.device)
    rc = lib.dec_attn_prefill_varlen(C.byref(shape), _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(page_table),
                                     _ptr(seq_lens), _ptr(cu_q_lens), int(total), _ptr(out), _ptr(lse), _ptr(status),
                                     _stream_handle(stream))
    if rc != OK:
        raise DecAttnError(rc, "dec_attn_prefill_varlen")
    return out, lse


def prefill_fp8(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor, kv_scales: torch.Tensor,
                page_table: torch.Tensor, seq_lens: torch.Tensor, *, cu_q_lens: torch.Tensor | None = None,
                max_q_rows: int = 0, sm_scale: float = 0.0, workspace: torch.Tensor | None = None,
                out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                status: torch.Tensor | None = None, stream=None):
    """dec_attn_prefill_fp8: prefill over E4M3 pages (uint8 [num_pages][Hkv][P][128]) with fp32
    kv_scales [2][num_pages][Hkv]. q is [B][T][Hq][128] (cu_q_lens None) or packed
    [total][Hq][128] with cu_q_lens [B + 1] and ``max_q_rows`` bounding every request's rows.
    ``workspace``: uint8 device buffer of at least prefill_fp8_workspace_bytes (allocated here if
    None). Returns (out fp32, lse fp32) shaped like q's rows."""
    lib = load_library()
    if cu_q_lens is None:
        B, T, Hq, d = q.shape
        total = B * T
        out_shape = (B, T, Hq, d)
    else:
        total, Hq, d = q.shape
        B, T = page_table.shape[0], int(max_q_rows)
        out_shape = (total, Hq, d)
    shape = ShapeT(B, Hq, k_pages.shape[1], d, T, k_pages.shape[2], k_pages.shape[0], page_table.shape[1],
                   KV_FP8E4M3, float(sm_scale))
    need = int(lib.dec_attn_prefill_fp8_workspace_bytes(C.byref(shape)))
    if need < 0:
        raise DecAttnError(need, "dec_attn_prefill_fp8_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty(out_shape, dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty(out_shape[:-1], dtype=torch.float32, device=q.device)
    rc = lib.dec_attn_prefill_fp8(C.byref(shape), _ptr(q), _ptr(k_pages), _ptr(v_pages), _ptr(kv_scales),
                                  _ptr(page_table), _ptr(seq_lens), _ptr(cu_q_lens), int(total), _ptr(workspace),
                                  int(workspace.numel() * workspace.element_size()), _ptr(out), _ptr(lse),
                                  _ptr(status), _stream_handle(stream))
    if rc != OK:
        raise DecAttnError(rc, "dec_attn_prefill_fp8")
    return out, lse


def prefill_fp8_workspace_bytes(q_shape, k_pages: torch.Tensor, page_table: torch.Tensor, max_q_rows: int = 0) -> int:
    """dec_attn_prefill_fp8_workspace_bytes for these pools (the workspace does not depend on q)."""
    Hq, d = int(q_shape[-2]), int(q_shape[-1])
    shape = ShapeT(page_table.shape[0], Hq, k_pages.shape[1], d, max(int(max_q_rows), 1), k_pages.shape[2],
                   k_pages.shape[0], page_table.shape[1], KV_FP8E4M3, 0.0)
    n = int(load_library().dec_attn_prefill_fp8_workspace_bytes(C.byref(shape)))
    if n < 0:
        raise DecAttnError(n, "dec_attn_prefill_fp8_workspace_bytes")
    return n


def test_set_waits(limit_ns: int = 0, skip_fill: int = -1) -> None:
    """dec_attn_test_set_waits: the wait limit (0: the default 2 s) and a pipeline fill of CTA 0 to
    leave out (-1: none) for the launches that follow; for tests of the bounded waits only."""
    rc = load_library().dec_attn_test_set_waits(int(limit_ns), int(skip_fill))
    if rc != OK:
        raise DecAttnError(rc, "dec_attn_test_set_waits")


def read_status(pl: Plan | None = None, workspace: torch.Tensor | None = None, stream=None) -> int:
    """Synchronises the stream and returns the first device-side status (0 = ok)."""
    lib = load_library()
    return int(lib.dec_attn_read_status(None if pl is None else C.byref(pl.handle), _ptr(workspace),
                                        _stream_handle(stream)))


def plan_contents(pl: Plan, seq_lens: torch.Tensor, stream=None) -> dict:
    """The plan's explicit work list (dec_attn_plan_export), copied to the host: status, n_units,
    bin_off [n_bins + 1] and units [n_units][8] = (b, h, tok_begin, tok_end, seq_len, slot, tile, 0)."""
    import numpy as np
    lib = load_library()
    dev = pl.buf.device
    cap = int(pl.handle.max_units)
    bin_off = torch.empty(pl.n_bins + 1, dtype=torch.int32, device=dev)
    units = torch.empty((max(cap, 1), 8), dtype=torch.int32, device=dev)
    n = torch.empty(1, dtype=torch.int32, device=dev)
    rc = lib.dec_attn_plan_export(C.byref(pl.handle), _ptr(seq_lens), _ptr(bin_off), _ptr(units), cap, _ptr(n),
                                  _stream_handle(stream))
    if rc != OK:
        raise DecAttnError(rc, "dec_attn_plan_export")
    hdr = pl.buf[:128].cpu().numpy().view(np.int32)
    n_units = int(n.item())
    return dict(magic=int(hdr[0]), status=int(hdr[1]), run_status=int(hdr[2]), n_bins=int(hdr[3]),
                n_units=n_units, bin_off=bin_off.cpu().numpy(),
                units=units[:max(n_units, 0)].cpu().numpy())


def sm_scale_default(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)
