"""Seeded synthetic inputs for paged-KV GQA decode attention.

This module only draws and lays out inputs. It computes no attention, no
softmax and no scheduling, so both the CPU oracle (``oracle/``) and the CUDA
path (``paged_kv_decode_29_b200``) can use it without sharing any of the
method's arithmetic.

Input recipe (one reading of the workloads the pages leave open):

* values: q, K and V are drawn fp32 N(0, 1) and rounded to bf16 with
  round-to-nearest-even; everything downstream uses those bf16 values exactly;
* the KV pools are ``[num_pages][n_kv_heads][page_size][head_dim]``; physical
  page ids are a seeded random permutation of the pool, handed to each request
  in logical order; the slots of a partial last page past ``seq_len`` are zero;
* the page table is ``int32 [batch][max_pages_per_seq]``, padded with -1;
* FP8 pools (OCP E4M3 "fn": bias 7, largest finite 448, no infinities) carry
  one fp32 scale per (page, KV head) for K and for V: ``absmax / 448`` over the
  valid tokens of that page and head (1 if the absmax is 0); codes are
  ``RNE(x / scale)`` saturated to +-448;
* "peaky" K rows: each K row (page, head, slot) is multiplied by 8 with an
  independent Bernoulli(frac) draw (x8 is exact in bf16).

Random streams: every (seed, stream, chunk) triple gets its own PCG64 generator
from ``SeedSequence(seed, spawn_key=(stream, chunk))``, so the draws do not
depend on thread count or on how the work is split.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_CHUNK = 1 << 22  # values per independent random chunk
_STREAM_LENS, _STREAM_PERM, _STREAM_Q, _STREAM_K, _STREAM_V, _STREAM_PEAKY = range(6)
_STREAM_NEW_Q, _STREAM_NEW_K, _STREAM_NEW_V, _STREAM_MASK = range(6, 10)

E4M3_MAX = 448.0


def _gen(seed: int, stream: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(stream, chunk))))


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).copy()
    r = (u >> 16) & 1
    r += 0x7FFF
    u += r
    u >>= 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """fp32 -> OCP E4M3 "fn" codes, round-to-nearest-even, saturating at +-448.

    Finite codes: exponent field e in [1, 15] gives (1 + m/8) * 2^(e-7) (e = 15,
    m = 7 is NaN and never produced); e = 0 gives the subnormals m * 2^-9.
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.minimum(np.abs(x).astype(np.float64), E4M3_MAX)
    _, ex = np.frexp(a)                       # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)                # unbiased exponent, subnormals share -6
    step = np.ldexp(1.0, e - 3)               # spacing of the 3-bit mantissa grid
    n = np.rint(a / step)                     # ties to even -> even mantissa LSB
    qv = n * step
    _, ex2 = np.frexp(qv)
    e2 = np.maximum(ex2 - 1, -6)
    normal = qv >= 2.0 ** -6
    m = np.where(normal, qv / np.ldexp(1.0, e2 - 3) - 8, qv / 2.0 ** -9)
    code = np.where(normal, (e2 + 7) * 8 + m, m).astype(np.int64)
    code = np.where(a == 0, 0, code)
    sign = (np.signbit(x) & (code != 0)).astype(np.int64) << 7
    return (code | sign).astype(np.uint8)


@dataclass
class Problem:
    """One decode-attention problem with its inputs in host memory."""
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    page_size: int
    q_tokens: int
    kv_dtype: str            # "bf16" or "fp8e4m3"
    tile_len: int
    seq_lens: np.ndarray     # int32 [B]
    page_table: np.ndarray   # int32 [B][max_pages_per_seq], -1 padded
    q: np.ndarray            # uint16 bf16 bits [B][T][Hq][d]
    k_pages: np.ndarray      # uint16 bf16 bits or uint8 e4m3 codes [num_pages][Hkv][P][d]
    v_pages: np.ndarray
    kv_scales: np.ndarray | None = None  # float32 [2][num_pages][Hkv] (K then V), FP8 only
    sm_scale: float = 0.0
    tile_mask: np.ndarray | None = None  # uint32 [B][Hkv][words]: block-sparse decode, bit i keeps tile i
    # variable-length query rows (prefill): request b's rows are rows cu_q[b] .. cu_q[b+1]-1 of a
    # packed q [total][Hq][d]; q_tokens is then the largest per-request count
    cu_q: np.ndarray | None = None       # int32 [B+1]
    meta: dict = field(default_factory=dict)

    @property
    def num_pages(self) -> int:
        return int(self.k_pages.shape[0])

    @property
    def max_pages_per_seq(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def kv_elem_bytes(self) -> int:
        return 1 if self.kv_dtype == "fp8e4m3" else 2

    def algorithmic_bytes(self) -> int:
        """Bytes the method must move once: visible KV rows, q, out+lse, page-table rows, scales.
        With a block-sparse tile mask, only the kept tiles' KV rows (per KV head), and the pages
        some head keeps."""
        d, P, hkv = self.head_dim, self.page_size, self.n_kv_heads
        L = self.seq_lens.astype(np.int64)
        q = self.q.nbytes
        out = self.batch * self.q_tokens * self.n_q_heads * (d + 1) * 4
        if self.tile_mask is None:
            kv = int(L.sum()) * hkv * d * self.kv_elem_bytes() * 2
            pages = int(((L + P - 1) // P).sum())
            kv_pages = pages * hkv
        else:
            tl = self.tile_len
            kv = pages = kv_pages = 0
            for b in range(self.batch):
                nb = int((L[b] + tl - 1) // tl)
                i = np.arange(nb)
                kept = ((self.tile_mask[b][:, i // 32] >> (i % 32).astype(np.uint32)) & 1).astype(bool)  # [Hkv][nb]
                toks = np.minimum((i + 1) * tl, L[b]) - i * tl
                kv += int((kept * toks[None, :]).sum()) * d * self.kv_elem_bytes() * 2
                pg = -(-toks // P)  # pages per tile
                pages += int((kept.any(axis=0) * pg).sum())
                kv_pages += int((kept * pg[None, :]).sum())
        table = pages * 4 + self.batch * 4
        scales = kv_pages * 2 * 4 if self.kv_scales is not None else 0
        return kv + q + out + table + scales


def _fill_normal_bf16(seed: int, stream: int, n: int, scale_rows=None) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    nchunks = (n + _CHUNK - 1) // _CHUNK

    def work(c):
        lo, hi = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        x = _gen(seed, stream, c).standard_normal(hi - lo, dtype=np.float32)
        out[lo:hi] = bf16_bits_from_f32(x)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, range(nchunks)))
    return out


def _fill_normal_f32(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    nchunks = (n + _CHUNK - 1) // _CHUNK

    def work(c):
        lo, hi = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        out[lo:hi] = _gen(seed, stream, c).standard_normal(hi - lo, dtype=np.float32)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, range(nchunks)))
    return out


def make_problem(*, name="custom", batch, n_q_heads, n_kv_heads, head_dim, seq_lens, page_size,
                 q_tokens=1, kv_dtype="bf16", tile_len=256, seed=0, pool_pages=None,
                 peaky_frac=0.0, peaky_mult=8.0, sm_scale=None) -> Problem:
    """Build a seeded problem. ``seq_lens`` is a list/array of KV lengths (tokens)."""
    assert n_q_heads % n_kv_heads == 0
    L = np.asarray(seq_lens, dtype=np.int64).reshape(batch)
    P, d, hkv = page_size, head_dim, n_kv_heads
    npg = (L + P - 1) // P
    need = int(npg.sum())
    num_pages = int(pool_pages) if pool_pages is not None else max(need, 1)
    assert num_pages >= need, "page pool too small"
    perm = _gen(seed, _STREAM_PERM, 0).permutation(num_pages).astype(np.int32)
    mpps = max(int(npg.max()) if batch else 0, 1)
    table = np.full((batch, mpps), -1, dtype=np.int32)
    cur = 0
    for b in range(batch):
        table[b, : npg[b]] = perm[cur: cur + npg[b]]
        cur += int(npg[b])

    q = _fill_normal_bf16(seed, _STREAM_Q, batch * q_tokens * n_q_heads * d).reshape(batch, q_tokens, n_q_heads, d)

    # valid[page, slot]: whether pool slot (page, slot) holds a token of some request
    valid = np.zeros((num_pages, P), dtype=bool)
    for b in range(batch):
        for p in range(int(npg[b])):
            n_here = min(P, int(L[b]) - p * P)
            valid[table[b, p], :n_here] = True

    shape = (num_pages, hkv, P, d)
    nval = num_pages * hkv * P * d
    inv_pages, inv_slots = np.nonzero(~valid)
    scales = None
    if kv_dtype == "bf16":
        k = _fill_normal_bf16(seed, _STREAM_K, nval).reshape(shape)
        v = _fill_normal_bf16(seed, _STREAM_V, nval).reshape(shape)
        if peaky_frac > 0:
            rows = _gen(seed, _STREAM_PEAKY, 0).random((num_pages, hkv, P)) < peaky_frac
            kf = bf16_bits_to_f32(k[rows])
            k[rows] = bf16_bits_from_f32(kf * np.float32(peaky_mult))
        k[inv_pages, :, inv_slots, :] = 0
        v[inv_pages, :, inv_slots, :] = 0
    elif kv_dtype == "fp8e4m3":
        assert peaky_frac == 0
        scales = np.empty((2, num_pages, hkv), dtype=np.float32)
        codes = []
        for i, stream in enumerate((_STREAM_K, _STREAM_V)):
            xf = _fill_normal_f32(seed, stream, nval).reshape(shape)
            xf[inv_pages, :, inv_slots, :] = 0
            out = np.empty(shape, dtype=np.uint8)
            step = 1024

            def work(p0, xf=xf, out=out, i=i):
                blk = xf[p0:p0 + step]
                amax = np.abs(blk).max(axis=(2, 3))
                sc = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
                scales[i, p0:p0 + step] = sc
                out[p0:p0 + step] = e4m3_encode(blk / sc[:, :, None, None])

            with ThreadPoolExecutor(_threads()) as ex:
                list(ex.map(work, range(0, num_pages, step)))
            codes.append(out)
            del xf
        k, v = codes
    else:
        raise ValueError(kv_dtype)

    return Problem(name=name, batch=batch, n_q_heads=n_q_heads, n_kv_heads=hkv, head_dim=d,
                   page_size=P, q_tokens=q_tokens, kv_dtype=kv_dtype, tile_len=tile_len,
                   seq_lens=L.astype(np.int32), page_table=table, q=q, k_pages=k, v_pages=v,
                   kv_scales=scales,
                   sm_scale=float(sm_scale) if sm_scale is not None else 1.0 / math.sqrt(d),
                   meta=dict(seed=seed, peaky_frac=peaky_frac, pool_pages=num_pages))


def config_seq_lens(name: str) -> list[int]:
    """KV lengths of the named workload (seeded)."""
    if name == "tiny":
        return [17, 300]
    if name == "uniform":
        return [4096] * 32
    if name == "mixed":
        u = _gen(2, _STREAM_LENS, 0).random(64)
        L = np.floor(np.exp(math.log(128) + u * (math.log(65536) - math.log(128))))
        return [int(x) for x in np.clip(L, 128, 65536)]
    if name == "long_b1":
        return [131072]
    if name == "long_b4":
        return [131072] * 4
    if name == "fp8_spec":
        return [int(x) for x in _gen(4, _STREAM_LENS, 0).integers(1024, 32768, size=16, endpoint=True)]
    if name == "prefill":
        return [2048] * 4
    raise KeyError(name)


# name -> (shape, tile length) of the five workloads; the tile lengths the configs do not fix
# (uniform, long_b1, long_b4, fp8_spec) are those the library's rule, dec_attn_default_tile_len,
# gives on 592 bins (148 SMs x 4).
CONFIGS = {
    "tiny": dict(batch=2, n_q_heads=4, n_kv_heads=1, head_dim=64, page_size=16, q_tokens=1,
                 kv_dtype="bf16", tile_len=64, seed=0, pool_pages=64),
    "uniform": dict(batch=32, n_q_heads=32, n_kv_heads=8, head_dim=128, page_size=16, q_tokens=1,
                    kv_dtype="bf16", tile_len=256, seed=1),
    "mixed": dict(batch=64, n_q_heads=32, n_kv_heads=8, head_dim=128, page_size=16, q_tokens=1,
                  kv_dtype="bf16", tile_len=256, seed=2, peaky_frac=0.01, peaky_mult=8.0),
    "long_b1": dict(batch=1, n_q_heads=64, n_kv_heads=8, head_dim=128, page_size=64, q_tokens=1,
                    kv_dtype="bf16", tile_len=256, seed=3),
    "long_b4": dict(batch=4, n_q_heads=64, n_kv_heads=8, head_dim=128, page_size=64, q_tokens=1,
                    kv_dtype="bf16", tile_len=1024, seed=3),
    "fp8_spec": dict(batch=16, n_q_heads=32, n_kv_heads=8, head_dim=128, page_size=16, q_tokens=4,
                     kv_dtype="fp8e4m3", tile_len=4096, seed=4),
    # prefill (dec_attn_prefill): 4 prompts of 2048 tokens, every position a query row
    "prefill": dict(batch=4, n_q_heads=32, n_kv_heads=8, head_dim=128, page_size=16, q_tokens=2048,
                    kv_dtype="bf16", tile_len=256, seed=6),
}


def make_varlen_problem(*, name="varlen", q_lens, **kw) -> Problem:
    """A problem with a different number of query rows per request: ``q_lens[b]`` rows for request
    b (its last q_lens[b] positions), packed into q [sum q_lens][Hq][d] with offsets cu_q [B+1].
    The rows of request b are the first q_lens[b] rows of the same seeded draw that a problem with
    max(q_lens) query tokens would use. Other arguments as make_problem (q_tokens is set)."""
    ql = np.asarray(q_lens, dtype=np.int64)
    assert ql.ndim == 1 and np.all(ql >= 0)
    T = max(int(ql.max()) if ql.size else 0, 1)
    pr = make_problem(name=name, q_tokens=T, **kw)
    cu = np.zeros(ql.size + 1, dtype=np.int64)
    cu[1:] = np.cumsum(ql)
    assert cu[-1] < 2 ** 31
    pr.q = np.ascontiguousarray(np.concatenate([pr.q[b, : ql[b]] for b in range(ql.size)], axis=0)
                                if ql.size else np.zeros((0, pr.n_q_heads, pr.head_dim), dtype=np.uint16))
    pr.cu_q = cu.astype(np.int32)
    return pr


def make_config(name: str, **overrides) -> Problem:
    kw = dict(CONFIGS[name])
    kw.update(overrides)
    return make_problem(name=name, seq_lens=config_seq_lens(name), **kw)


def make_step_inputs(pr: Problem, seed: int | None = None):
    """The new rows of one decode step before the fused pre-processing: q_new bf16 bits
    [B][T][Hq][d], k_new and v_new bf16 bits [B][T][Hkv][d], all ~N(0,1) rounded to bf16.
    Seeded by (seed or the problem's seed) on streams of their own; no method arithmetic."""
    s = pr.meta["seed"] if seed is None else seed
    B, T, hq, hkv, d = pr.batch, pr.q_tokens, pr.n_q_heads, pr.n_kv_heads, pr.head_dim
    q = _fill_normal_bf16(s, _STREAM_NEW_Q, B * T * hq * d).reshape(B, T, hq, d)
    k = _fill_normal_bf16(s, _STREAM_NEW_K, B * T * hkv * d).reshape(B, T, hkv, d)
    v = _fill_normal_bf16(s, _STREAM_NEW_V, B * T * hkv * d).reshape(B, T, hkv, d)
    return q, k, v


def make_tile_mask(pr: Problem, density: float, seed: int | None = None, keep_last: bool = True) -> np.ndarray:
    """A block-sparse decode mask: uint32 [B][Hkv][words] with bit i of (b, h) set (tile i of the
    pair's tile_len-token tiles kept) independently with probability ``density``; with
    ``keep_last`` the tile holding each request's newest token is always kept (a local window).
    Bits past a request's last tile are 0. Seeded; no method arithmetic."""
    s = pr.meta["seed"] if seed is None else seed
    L = pr.seq_lens.astype(np.int64)
    nb = (L + pr.tile_len - 1) // pr.tile_len
    n_max = int(nb.max()) if pr.batch else 0
    words = max(1, (n_max + 31) // 32)
    keep = _gen(s, _STREAM_MASK, 0).random((pr.batch, pr.n_kv_heads, words * 32)) < density
    idx = np.arange(words * 32)
    keep &= idx[None, None, :] < nb[:, None, None]
    if keep_last:
        for b in range(pr.batch):
            if nb[b] > 0:
                keep[b, :, nb[b] - 1] = True
    bits = (keep.reshape(pr.batch, pr.n_kv_heads, words, 32).astype(np.uint64) << np.arange(32, dtype=np.uint64))
    return bits.sum(axis=-1).astype(np.uint32)
