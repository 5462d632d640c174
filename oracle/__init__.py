"""CPU oracle for paged-KV GQA decode attention with split-KV scheduling.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import this module; the product path
(``paged_kv_decode_29_b200``) never does. It shares no code with the CUDA
path; both only read inputs drawn by ``workloads``.

Everything is computed in fp64 by ``oracle.c``:

* ``decode`` / ``decode_rows`` / ``attend``: scaled-dot-product attention of
  each query row over the paged KV cache, with an explicit full softmax and the
  bottom-right causal mask of speculative multi-token queries ("PaddlePaddle/
  HALOps" README, Highlights, GQA attention item); ``decode_varlen``: the same
  with a different number of query rows per request (each request on its own).
* ``plan``: the greedy bin-packing of uniform KV tiles onto CTAs ("HPC-Ops:
  Tencent's CUDA Kernel Library for LLM Inference Hot Paths", "How the kernels
  are organized around specific workload shapes"), as a literal sequential
  greedy over the tiles sorted by cost.
* ``e4m3_value``: the OCP E4M3 "fn" code table; ``e4m3_round`` / ``round_q_e4m3_rows``: the q
  rounding of the FP8-products mode, from the format's definition (nearest value, ties to even).

Parity pins for each function live in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into oracle/_build/liboracle.so (gcc, -O2, OpenMP)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(C.Structure):
    _fields_ = [
        ("batch", C.c_int32), ("q_tokens", C.c_int32), ("n_q_heads", C.c_int32), ("n_kv_heads", C.c_int32),
        ("head_dim", C.c_int32), ("page_size", C.c_int32), ("num_pages", C.c_int32),
        ("max_pages_per_seq", C.c_int32), ("kv_fp8", C.c_int32), ("pad_", C.c_int32),
        ("sm_scale", C.c_double),
        ("q", C.c_void_p), ("k_pages", C.c_void_p), ("v_pages", C.c_void_p), ("kv_scales", C.c_void_p),
        ("page_table", C.c_void_p), ("seq_lens", C.c_void_p),
        ("tile_mask", C.c_void_p), ("mask_words", C.c_int32), ("tile_len", C.c_int32),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            P = C.POINTER(_Problem)
            lib.oracle_decode.argtypes = [P, C.c_void_p, C.c_void_p, C.c_int]
            lib.oracle_decode_rows.argtypes = [P, C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p, C.c_int]
            lib.oracle_attend.argtypes = [P, C.c_int, C.c_int, C.c_int, C.c_int64, C.c_int64,
                                          C.c_void_p, C.c_void_p, C.c_void_p]
            lib.oracle_attend.restype = C.c_int64
            lib.oracle_plan.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int64,
                                        C.c_void_p, C.c_void_p, C.c_void_p]
            lib.oracle_plan.restype = C.c_int64
            lib.oracle_plan_masked.argtypes = [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                               C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p]
            lib.oracle_plan_masked.restype = C.c_int64
            lib.oracle_e4m3_value.argtypes = [C.c_uint8]
            lib.oracle_e4m3_value.restype = C.c_double
            lib.oracle_max_threads.restype = C.c_int
            lib.oracle_rope_row.argtypes = [C.c_void_p, C.c_int, C.c_double, C.c_double, C.c_void_p]
            lib.oracle_bf16_bits.argtypes = [C.c_double]
            lib.oracle_bf16_bits.restype = C.c_uint16
            lib.oracle_append_rope.argtypes = [C.c_void_p] * 5 + [C.c_int] * 8 + [C.c_double] + [C.c_void_p] * 3
            lib.oracle_append_rope.restype = C.c_int64
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


class _Bound:
    """Keeps the numpy arrays alive while the C struct points at them."""

    def __init__(self, pr):
        self.arrs = dict(
            q=np.ascontiguousarray(pr.q, dtype=np.uint16),
            k=np.ascontiguousarray(pr.k_pages),
            v=np.ascontiguousarray(pr.v_pages),
            s=None if pr.kv_scales is None else np.ascontiguousarray(pr.kv_scales, dtype=np.float32),
            t=np.ascontiguousarray(pr.page_table, dtype=np.int32),
            L=np.ascontiguousarray(pr.seq_lens, dtype=np.int32),
            m=None if getattr(pr, "tile_mask", None) is None else np.ascontiguousarray(pr.tile_mask, dtype=np.uint32),
        )
        a = self.arrs
        fp8 = pr.kv_dtype == "fp8e4m3"
        if fp8 and a["s"] is None:
            raise ValueError("FP8 KV needs kv_scales")
        self.s = _Problem(pr.batch, pr.q_tokens, pr.n_q_heads, pr.n_kv_heads, pr.head_dim, pr.page_size,
                          int(a["k"].shape[0]), int(a["t"].shape[1]), int(fp8), 0, float(pr.sm_scale),
                          _ptr(a["q"]), _ptr(a["k"]), _ptr(a["v"]), _ptr(a["s"]), _ptr(a["t"]), _ptr(a["L"]),
                          _ptr(a["m"]), 0 if a["m"] is None else int(a["m"].shape[-1]), int(pr.tile_len))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def decode(pr, nthreads: int = 0):
    """All rows. Returns out float64 [B][T][Hq][d] and lse float64 [B][T][Hq] (natural log)."""
    lib = _load()
    bd = _Bound(pr)
    out = np.zeros((pr.batch, pr.q_tokens, pr.n_q_heads, pr.head_dim), dtype=np.float64)
    lse = np.zeros((pr.batch, pr.q_tokens, pr.n_q_heads), dtype=np.float64)
    lib.oracle_decode(C.byref(bd.s), out.ctypes.data, lse.ctypes.data, int(nthreads))
    return out, lse


def decode_rows(pr, rows, nthreads: int = 0):
    """Selected rows, ``rows`` an int array [n][3] of (b, t, qh)."""
    lib = _load()
    bd = _Bound(pr)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
    n = rows.shape[0]
    out = np.zeros((n, pr.head_dim), dtype=np.float64)
    lse = np.zeros((n,), dtype=np.float64)
    lib.oracle_decode_rows(C.byref(bd.s), rows.ctypes.data, n, out.ctypes.data, lse.ctypes.data, int(nthreads))
    return out, lse


def decode_varlen(pr):
    """Variable-length query rows (``pr.cu_q`` set, q packed [total][Hq][d]): request b's
    Tb = cu_q[b+1] - cu_q[b] rows are its last Tb positions, with the bottom-right causal rule
    ("PaddlePaddle/HALOps" README, Highlights, GQA attention item: variable-length prefill). By
    definition each request is computed alone, as a decode of that one request with T = Tb.
    Returns out float64 [total][Hq][d] and lse float64 [total][Hq]."""
    import copy
    cu = np.asarray(pr.cu_q, dtype=np.int64)
    total = int(cu[-1])
    out = np.zeros((total, pr.n_q_heads, pr.head_dim), dtype=np.float64)
    lse = np.zeros((total, pr.n_q_heads), dtype=np.float64)
    for b in range(pr.batch):
        lo, hi = int(cu[b]), int(cu[b + 1])
        if hi == lo:
            continue
        one = copy.copy(pr)
        one.batch, one.q_tokens, one.cu_q, one.tile_mask = 1, hi - lo, None, None
        one.q = np.ascontiguousarray(pr.q[lo:hi][None])
        one.seq_lens = np.ascontiguousarray(pr.seq_lens[b:b + 1])
        one.page_table = np.ascontiguousarray(pr.page_table[b:b + 1])
        o, l = decode(one)
        out[lo:hi] = o[0]
        lse[lo:hi] = l[0]
    return out, lse


def attend(pr, b, t, qh, j_lo=0, j_hi=None, weights=False):
    """One row over keys [j_lo, j_hi) (clipped to the causal limit).

    Returns (out[d], lse, n_visible[, weights[n_visible]])."""
    lib = _load()
    bd = _Bound(pr)
    if j_hi is None:
        j_hi = int(pr.seq_lens[b])
    out = np.zeros(pr.head_dim, dtype=np.float64)
    lse = np.zeros(1, dtype=np.float64)
    w = np.zeros(max(1, int(j_hi) - int(j_lo)), dtype=np.float64) if weights else None
    n = lib.oracle_attend(C.byref(bd.s), int(b), int(t), int(qh), int(j_lo), int(j_hi),
                          out.ctypes.data, lse.ctypes.data, _ptr(w))
    if weights:
        return out, float(lse[0]), int(n), w[:n]
    return out, float(lse[0]), int(n)


UNIT_FIELDS = ("b", "h", "tok_begin", "tok_end", "seq_len", "slot", "tile", "zero")


def plan(seq_lens, n_kv_heads: int, tile_len: int, n_bins: int, capacity: int | None = None, tile_mask=None):
    """Greedy bin-packing of uniform KV tiles. Returns dict(n_units, bin_off, units[U][8], pair_off)
    or None when the tile count exceeds ``capacity``. ``tile_mask`` (uint32 [B][Hkv][words]): only
    the tiles whose bit is set enter the work list (block-sparse decode)."""
    lib = _load()
    L = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    B = L.shape[0]
    U_max = int(n_kv_heads * ((L.astype(np.int64) + tile_len - 1) // tile_len).sum())
    cap = U_max if capacity is None else int(capacity)
    bin_off = np.zeros(n_bins + 1, dtype=np.int32)
    units = np.zeros((max(U_max, 1), 8), dtype=np.int32)
    pair_off = np.zeros(B * n_kv_heads + 1, dtype=np.int32)
    if tile_mask is None:
        U = lib.oracle_plan(L.ctypes.data, B, int(n_kv_heads), int(tile_len), int(n_bins), cap,
                            bin_off.ctypes.data, units.ctypes.data, pair_off.ctypes.data)
    else:
        m = np.ascontiguousarray(tile_mask, dtype=np.uint32)
        assert m.shape[:2] == (B, n_kv_heads)
        U = lib.oracle_plan_masked(L.ctypes.data, m.ctypes.data, int(m.shape[2]), B, int(n_kv_heads), int(tile_len),
                                   int(n_bins), cap, bin_off.ctypes.data, units.ctypes.data, pair_off.ctypes.data)
    if U < 0:
        return None
    return dict(n_units=int(U), bin_off=bin_off, units=units[:U], pair_off=pair_off)


def e4m3_value(code: int) -> float:
    return float(_load().oracle_e4m3_value(int(code) & 0xFF))


def e4m3_table() -> np.ndarray:
    return np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


# ---- FP8 products mode: q rounded to one E4M3 part per row

def e4m3_round(x) -> np.ndarray:
    """The E4M3 value nearest to each x (fp64 array), ties to the even code, saturating at +-448:
    round-to-nearest-even onto the finite set of the OCP E4M3 "fn" format."""
    x = np.asarray(x, dtype=np.float64)
    tab = e4m3_table()
    codes = np.arange(128)  # non-negative codes 0x00 .. 0x7F (0x7F is NaN)
    vals = tab[:127]        # 0 .. 448, increasing with the code
    a = np.minimum(np.abs(x), 448.0)
    hi = np.clip(np.searchsorted(vals, a, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    dlo, dhi = a - vals[lo], vals[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (codes[hi] % 2 == 0))
    r = np.where(pick_hi, vals[hi], vals[lo])
    return np.copysign(r, x)


def round_q_e4m3_rows(q_bits) -> np.ndarray:
    """q of the FP8-products mode (KV_FP8E4M3_MMA8): each query row (the last axis) is scaled by
    2^E, E = 7 - floor(log2 max|q_row|) (E = 7 for a zero row, clamped to [-100, 100]), rounded to
    the nearest E4M3 value (ties to even) and scaled back. Input and output: bf16 bit patterns
    (every such value is a bf16 number). The oracle then runs on these rows."""
    qb = np.asarray(q_bits, dtype=np.uint16)
    v = (qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    amax = np.max(np.abs(v), axis=-1, keepdims=True)
    _, e = np.frexp(np.where(amax > 0, amax, 1.0))  # amax = m 2^e, m in [0.5, 1)
    E = np.where(amax > 0, 7 - (e - 1), 7)
    E = np.clip(E, -100, 100)
    r = e4m3_round(np.ldexp(v, E))
    out = np.ldexp(r, -E)
    return bf16_bits(out)


# ---- fused pre-processing of a decode step: rotary embedding + KV append (oracle.c)

def rope_rows(x, positions, base: float = 10000.0):
    """fp64 rotate-half rotary embedding of the rows x[n][d] at positions[n] (no rounding)."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    n, d = x.shape
    pos = np.asarray(positions, dtype=np.float64).reshape(n)
    y = np.empty_like(x)
    for i in range(n):
        lib.oracle_rope_row(x[i].ctypes.data, int(d), float(pos[i]), float(base), y[i].ctypes.data)
    return y


def bf16_bits(values):
    """bf16 bit patterns nearest to the fp64 values (ties to even)."""
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    return np.array([lib.oracle_bf16_bits(float(x)) for x in v.reshape(-1)], dtype=np.uint16).reshape(v.shape)


def append_rope(q_new, k_new, v_new, page_table, seq_lens, k_pages, v_pages, base: float = 10000.0):
    """Rotary embedding of the T new q and k rows and their append to the paged cache.
    q_new [B][T][Hq][d], k_new / v_new [B][T][Hkv][d], k_pages / v_pages [num_pages][Hkv][P][d]:
    bf16 bit patterns (uint16). Returns (q_out, k_pages', v_pages', rows written), the pages
    copied, or rows written = -1 for a page id out of range."""
    lib = _load()
    qn = np.ascontiguousarray(q_new, dtype=np.uint16)
    kn = np.ascontiguousarray(k_new, dtype=np.uint16)
    vn = np.ascontiguousarray(v_new, dtype=np.uint16)
    tab = np.ascontiguousarray(page_table, dtype=np.int32)
    L = np.ascontiguousarray(seq_lens, dtype=np.int32)
    kp = np.array(k_pages, dtype=np.uint16, copy=True, order="C")
    vp = np.array(v_pages, dtype=np.uint16, copy=True, order="C")
    B, T, Hq, d = qn.shape
    Hkv = kn.shape[2]
    num_pages, _, P, _ = kp.shape
    q_out = np.empty_like(qn)
    n = lib.oracle_append_rope(qn.ctypes.data, kn.ctypes.data, vn.ctypes.data, tab.ctypes.data, L.ctypes.data,
                               B, T, Hq, Hkv, d, P, num_pages, int(tab.shape[1]), float(base), q_out.ctypes.data,
                               kp.ctypes.data, vp.ctypes.data)
    return q_out, kp, vp, int(n)


# ---- the same pre-processing over an FP8 E4M3 cache: appending rows to a page with one scale

def e4m3_codes(values) -> np.ndarray:
    """The E4M3 code (uint8) of each value, which must be an E4M3 number (e.g. from e4m3_round)."""
    v = np.asarray(values, dtype=np.float64)
    tab = e4m3_table()
    mag = np.abs(v)
    idx = np.searchsorted(tab[:127], mag)        # codes 0x00 .. 0x7E hold 0 .. 448, increasing
    assert np.all(tab[np.minimum(idx, 126)] == mag), "not an E4M3 value"
    return (idx | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def append_rope_fp8(q_new, k_new, v_new, page_table, seq_lens, k_codes, v_codes, kv_scales, base: float = 10000.0):
    """Rotary embedding of the T new q and k rows and their append to an E4M3 paged cache with one
    fp32 scale per (page, KV head) for K and for V (the reading for FP8 pages; "PaddlePaddle/HALOps"
    README, Highlights, GQA attention item: fused pre/post-processing, BF16 / FP8 KV cache).

    The scale of a page and head covers its valid rows: |row value| <= 448 * scale (the encoding
    reading of the pages' FP8 scales). Appending new rows keeps that and never re-rounds old rows
    it does not have to:
      * x: the new rows' values (k rotated exactly, in fp64; v as given), A = max |x| over the
        page's new rows, rounded to fp32;
      * the page's old rows are its slots before the first new one; with old rows the scale
        becomes s' = max(s, A / 448), else s' = A / 448 (1 when A = 0), the divisions in fp32;
      * if s' > s, each old code is re-rounded: E4M3(fp32(value(code) * fp32(s / s')));
      * new rows: E4M3(fp32(fp32(x) / s'));
    E4M3(.) rounds to the nearest E4M3 value, ties to even, saturating at 448: every rounding
    decision is taken on the same fp32 numbers a single-precision implementation forms. q is
    rotated and rounded to bf16 as in append_rope; rows at positions < 0 have no slot.
    Inputs: q_new [B][T][Hq][d], k_new / v_new [B][T][Hkv][d] bf16 bits; k_codes / v_codes uint8
    [num_pages][Hkv][P][d]; kv_scales float32 [2][num_pages][Hkv]. Returns (q_out, k_codes',
    v_codes', kv_scales'), copies."""
    qn = np.asarray(q_new, dtype=np.uint16)
    kn = np.asarray(k_new, dtype=np.uint16)
    vn = np.asarray(v_new, dtype=np.uint16)
    tab = np.asarray(page_table, dtype=np.int64)
    L = np.asarray(seq_lens, dtype=np.int64)
    kc = np.array(k_codes, dtype=np.uint8, copy=True)
    vc = np.array(v_codes, dtype=np.uint8, copy=True)
    sc = np.array(kv_scales, dtype=np.float32, copy=True)
    B, T, Hq, d = qn.shape
    Hkv = kn.shape[2]
    P = kc.shape[2]
    f32 = np.float32
    val = e4m3_table()

    def to64(bits):
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    # q: the bf16 append's rotation
    pos_all = L[:, None] - T + np.arange(T)[None, :]                     # [B][T]
    q_out = np.empty_like(qn)
    for b in range(B):
        for t in range(T):
            pos = max(int(pos_all[b, t]), 0)
            q_out[b, t] = bf16_bits(rope_rows(to64(qn[b, t]), [pos] * Hq, base))
    for b in range(B):
        first = int(max(L[b] - T, 0))
        if L[b] <= first:
            continue
        for pg in range(first // P, (int(L[b]) - 1) // P + 1):
            lo, hi = max(first, pg * P), min(int(L[b]), pg * P + P)   # new positions in this page
            pid = int(tab[b, pg])
            ts = np.arange(lo, hi) - (int(L[b]) - T)                 # their token indices
            s_first = lo - pg * P
            for which, codes, new in ((0, kc, kn), (1, vc, vn)):
                for h in range(Hkv):
                    x = to64(new[b, ts, h])                            # [n][d]
                    if which == 0:
                        x = rope_rows(x, np.arange(lo, hi), base)
                    x32 = x.astype(f32)
                    A = f32(np.max(np.abs(x32)))
                    s_old = f32(sc[which, pid, h])
                    if s_first > 0:
                        s_new = max(s_old, f32(A / f32(448)))
                    else:
                        s_new = f32(A / f32(448)) if A > 0 else f32(1)
                    if s_first > 0 and s_new != s_old:
                        r = f32(s_old / s_new)
                        old = val[codes[pid, h, :s_first]].astype(f32)
                        codes[pid, h, :s_first] = e4m3_codes(e4m3_round((old * r).astype(np.float64)))
                    codes[pid, h, s_first:s_first + (hi - lo)] = e4m3_codes(e4m3_round((x32 / s_new).astype(np.float64)))
                    sc[which, pid, h] = s_new
    return q_out, kc, vc, sc
