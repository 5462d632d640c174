"""The C ABI without a GPU: the library loads, exports exactly what include/decattn.h
declares, and rejects bad arguments on the host before anything is enqueued."""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest

import paged_kv_decode_29_b200 as da
import workloads as W
from paged_kv_decode_29_b200 import build as dbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "decattn.h")


@pytest.fixture(scope="module")
def lib():
    dbuild.build()
    return da.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DECATTN_API\s+[\w\s\*]*?\b(dec_attn_\w+)\s*\(", text)))


def test_header_declares_the_binding_api():
    assert declared_symbols() == sorted(da.API)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", da.LIB_PATH]).decode()
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for sym in declared_symbols():
        assert sym in exported, sym
        assert getattr(lib, sym) is not None
    # nothing else leaks out of the library as a public function
    assert {s for s in exported if s.startswith("dec_attn")} == set(declared_symbols())


def test_status_strings(lib):
    for code in (da.OK, da.EINVAL, da.ENOTSUP, da.ESMALL, da.ECUDA, da.ETIMEOUT, da.EDEVICE, da.EALIGN,
                 da.ECAPACITY):
        s = da.status_string(code)
        assert s and s != "unknown status"
    assert da.status_string(12345) == "unknown status"


def test_plan_bytes_host_only(lib):
    n = lib.dec_attn_plan_bytes(32, 8, 256, 32 * 4096, 592)
    assert 0 < n < 64 * 1024
    # full tiles are stored in closed form: the plan does not grow with the KV length
    assert lib.dec_attn_plan_bytes(32, 8, 256, 32 * 4096 * 100, 592) == n
    assert lib.dec_attn_plan_bytes(64, 8, 256, 1000, 592) > n
    assert lib.dec_attn_plan_bytes(32, 8, 250, 1000, 592) == 0      # tile not a multiple of 16
    assert lib.dec_attn_plan_bytes(-1, 8, 256, 1000, 592) == 0
    assert lib.dec_attn_plan_bytes(4, 0, 256, 1000, 592) == 0
    assert lib.dec_attn_plan_bytes(4, 8, 256, 1000, 100000) == 0     # too many bins


def _shape(**kw):
    base = dict(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, q_tokens=1, page_size=16, num_pages=64,
                max_pages_per_seq=8, kv_dtype=da.KV_BF16, sm_scale=0.0)
    base.update(kw)
    return da.ShapeT(*[base[f] for f, _ in da.ShapeT._fields_])


def _plan(**kw):
    base = dict(buf=0x10000, buf_bytes=1 << 20, batch=2, n_kv_heads=2, tile_len=64, n_bins=8, max_units=64,
                sparse=0, reserved_=0)
    base.update(kw)
    return da.PlanT(*[base[f] for f, _ in da.PlanT._fields_])


FAKE = 0x7f0000000000  # never dereferenced: every case below fails a host check first


def _run(lib, shape, plan, q=FAKE, k=FAKE, v=FAKE, tab=FAKE, lens=FAKE, sc=None, ws=FAKE, ws_bytes=1 << 30,
         out=FAKE, lse=FAKE):
    return lib.dec_attn_run(C.byref(shape), q, k, v, tab, lens, sc, C.byref(plan), ws, ws_bytes, out, lse, None)


@pytest.mark.parametrize("shape_kw,plan_kw,code", [
    (dict(head_dim=96), {}, da.ENOTSUP),
    (dict(head_dim=256), {}, da.ENOTSUP),
    (dict(page_size=8), {}, da.ENOTSUP),
    (dict(page_size=48), dict(tile_len=64), da.ENOTSUP),       # tile not a multiple of the page
    (dict(n_q_heads=130, n_kv_heads=2, q_tokens=1), {}, da.ENOTSUP),  # G*T = 65
    (dict(q_tokens=9, n_q_heads=2, n_kv_heads=2), {}, da.ENOTSUP),    # T = 9
    (dict(q_tokens=5, n_q_heads=26, n_kv_heads=2), {}, da.ENOTSUP),   # G*T = 65
    (dict(q_tokens=5, n_q_heads=8, n_kv_heads=2, kv_dtype=da.KV_FP8E4M3_MMA8), {}, da.ENOTSUP),  # 20 > 16
    (dict(kv_dtype=7), {}, da.ENOTSUP),
    (dict(n_q_heads=6, n_kv_heads=4), dict(n_kv_heads=4), da.EINVAL),
    (dict(batch=3), {}, da.EINVAL),                             # plan made for another batch
    (dict(q_tokens=0), {}, da.EINVAL),
])
def test_run_rejects_bad_shapes(lib, shape_kw, plan_kw, code):
    assert _run(lib, _shape(**shape_kw), _plan(**plan_kw)) == code


@pytest.mark.parametrize("Hq,T,kv,ok", [
    (128, 1, da.KV_BF16, True), (16, 8, da.KV_BF16, True), (16, 8, da.KV_FP8E4M3, True),   # G*T = 64
    (130, 1, da.KV_BF16, False), (18, 8, da.KV_FP8E4M3, False), (2, 9, da.KV_BF16, False),
    (8, 4, da.KV_FP8E4M3_MMA8, True), (8, 5, da.KV_FP8E4M3_MMA8, False),                  # MMA8: G*T <= 16
])
def test_supported_query_rows_per_kv_head(lib, Hq, T, kv, ok):
    # host only: the workspace size is 0 exactly for the shapes dec_attn_run refuses
    s = _shape(n_q_heads=Hq, n_kv_heads=2, q_tokens=T, kv_dtype=kv)
    n = lib.dec_attn_workspace_bytes(C.byref(s), C.byref(_plan()))
    assert (n > 0) == ok
    if ok:  # partials [tiles][G*T][d + 1] fp32 among the rest
        assert n >= 64 * (Hq // 2) * T * 129 * 4


def test_run_rejects_null_and_misaligned(lib):
    s, p = _shape(), _plan()
    assert _run(lib, s, p, q=None) == da.EINVAL
    assert _run(lib, s, p, ws=None) == da.EINVAL
    assert _run(lib, _shape(kv_dtype=da.KV_FP8E4M3), p, sc=None) == da.EINVAL
    assert _run(lib, s, p, q=FAKE + 8) == da.EALIGN
    assert _run(lib, s, p, k=FAKE + 4) == da.EALIGN
    assert _run(lib, s, p, lse=FAKE + 2) == da.EALIGN


def test_run_rejects_small_workspace(lib):
    s, p = _shape(), _plan()
    need = lib.dec_attn_workspace_bytes(C.byref(s), C.byref(p))
    assert need > 0
    assert _run(lib, s, p, ws_bytes=need - 1) == da.ESMALL


def test_empty_batch_is_a_no_op(lib):
    assert _run(lib, _shape(batch=0), _plan(batch=0), q=None, k=None, v=None) == da.OK


def test_plan_rejects_bad_args(lib):
    h = da.PlanT()
    assert lib.dec_attn_plan(FAKE, 2, 2, 64, 1000, 8, None, 1 << 20, C.byref(h), None) == da.EINVAL
    assert lib.dec_attn_plan(FAKE, 2, 2, 64, 1000, 8, FAKE + 8, 1 << 20, C.byref(h), None) == da.EALIGN
    assert lib.dec_attn_plan(FAKE, 2, 2, 60, 1000, 8, FAKE, 1 << 20, C.byref(h), None) == da.ENOTSUP
    need = lib.dec_attn_plan_bytes(2, 2, 64, 1000, 8)
    assert lib.dec_attn_plan(FAKE, 2, 2, 64, 1000, 8, FAKE, need - 1, C.byref(h), None) == da.ESMALL


def _append(lib, s, base=10000.0, **ptrs):
    a = dict(qn=FAKE, kn=FAKE, vn=FAKE, tab=FAKE, lens=FAKE, qo=FAKE, kp=FAKE, vp=FAKE, st=None)
    a.update(ptrs)
    return lib.dec_attn_append_rope(C.byref(s), a["qn"], a["kn"], a["vn"], a["tab"], a["lens"], base, a["qo"],
                                    a["kp"], a["vp"], a["st"], None)


def test_append_rope_rejects_bad_args(lib):
    # every case fails a host check before a launch: the pointers are never dereferenced
    s = _shape()
    assert lib.dec_attn_append_rope(None, FAKE, FAKE, FAKE, FAKE, FAKE, 10000.0, FAKE, FAKE, FAKE, None,
                                    None) == da.EINVAL
    assert _append(lib, _shape(kv_dtype=da.KV_FP8E4M3)) == da.ENOTSUP  # FP8 pages: scale covers the page
    assert _append(lib, _shape(head_dim=96)) == da.ENOTSUP
    assert _append(lib, s, base=0.0) == da.EINVAL
    assert _append(lib, s, base=float("inf")) == da.EINVAL
    assert _append(lib, _shape(n_q_heads=6, n_kv_heads=4)) == da.EINVAL
    for name in ("qn", "kn", "vn", "tab", "lens", "qo", "kp", "vp"):
        assert _append(lib, s, **{name: None}) == da.EINVAL
    assert _append(lib, s, qo=FAKE + 2) == da.EALIGN       # d = 128: 4-byte lane accesses
    assert _append(lib, s, kp=FAKE + 2) == da.EALIGN
    assert _append(lib, _shape(batch=0), qn=None, kn=None, vn=None, tab=None, lens=None, qo=None, kp=None,
                   vp=None) == da.OK


def _prefill(lib, s, **ptrs):
    a = dict(q=FAKE, k=FAKE, v=FAKE, tab=FAKE, lens=FAKE, out=FAKE, lse=FAKE, st=None)
    a.update(ptrs)
    return lib.dec_attn_prefill(C.byref(s), a["q"], a["k"], a["v"], a["tab"], a["lens"], a["out"], a["lse"], a["st"],
                                None)


def test_prefill_rejects_bad_args(lib):
    # every case fails a host check before any tensor map is built or a kernel launched
    s = _shape(q_tokens=300)
    assert lib.dec_attn_prefill(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None) == da.EINVAL
    assert _prefill(lib, _shape(q_tokens=0)) == da.EINVAL
    assert _prefill(lib, _shape(batch=-1)) == da.EINVAL
    assert _prefill(lib, _shape(n_q_heads=6, n_kv_heads=4)) == da.EINVAL
    assert _prefill(lib, _shape(kv_dtype=da.KV_FP8E4M3)) == da.ENOTSUP   # bf16 pages only
    assert _prefill(lib, _shape(head_dim=64)) == da.ENOTSUP
    assert _prefill(lib, _shape(page_size=8)) == da.ENOTSUP
    for name in ("q", "k", "v", "tab", "lens", "out", "lse"):
        assert _prefill(lib, s, **{name: None}) == da.EINVAL
    assert _prefill(lib, s, q=FAKE + 8) == da.EALIGN
    assert _prefill(lib, s, out=FAKE + 4) == da.EALIGN
    assert _prefill(lib, s, lse=FAKE + 2) == da.EALIGN
    assert _prefill(lib, s, st=FAKE + 1) == da.EALIGN
    assert _prefill(lib, _shape(batch=0, q_tokens=300), q=None, k=None, v=None, tab=None, lens=None, out=None,
                    lse=None) == da.OK


def _no_usable_gpu():
    import torch

    return not torch.cuda.is_available()


@pytest.mark.skipif(not _no_usable_gpu(), reason="makes a CUDA call fail, which needs a host without a usable GPU")
def test_last_error_names_the_failing_step(lib):
    import threading

    # no device: the stream synchronisation fails and the step is recorded with CUDA's message
    assert lib.dec_attn_read_status(None, None, None) == da.ECUDA
    msg = da.last_error()
    assert msg.startswith("cudaStreamSynchronize: ") and len(msg) > len("cudaStreamSynchronize: ")
    # truncation: len counts the terminating zero; the full length is returned
    buf = C.create_string_buffer(8)
    assert lib.dec_attn_last_error(buf, 8) == len(msg)
    assert buf.value.decode() == msg[:7]
    assert lib.dec_attn_last_error(None, 0) == len(msg)
    # the binding's exception carries the detail
    assert "[cudaStreamSynchronize: " in str(da.DecAttnError(da.ECUDA, "dec_attn_read_status"))
    # per host thread: a fresh thread has no error recorded
    seen = []
    t = threading.Thread(target=lambda: seen.append(da.last_error()))
    t.start()
    t.join()
    assert seen == [""]


def test_test_set_waits_checks_its_range(lib):
    assert lib.dec_attn_test_set_waits(10, -1) == da.EINVAL             # below 0.1 ms
    assert lib.dec_attn_test_set_waits(3_000_000_000, -1) == da.EINVAL  # above the default 2 s
    assert lib.dec_attn_test_set_waits(1_000_000, -2) == da.EINVAL
    assert lib.dec_attn_test_set_waits(1_000_000, 3) == da.OK
    assert lib.dec_attn_test_set_waits(0, -1) == da.OK                  # back to the defaults


def test_default_tile_len_rule(lib):
    # host only; the rule's estimate (include/decattn.h) reproduces the hand-made choices where the
    # trade-off is clear, and never returns a length that is not a multiple of the page
    f = lib.dec_attn_default_tile_len
    assert f(32, 8, 32 * 4096, 16, 128, 4, da.KV_BF16, 592) == 256         # uniform
    assert f(1, 8, 131072, 64, 128, 8, da.KV_BF16, 592) == 256             # long context, one request
    assert f(4, 8, 4 * 131072, 64, 128, 8, da.KV_BF16, 592) == 1024        # long context, four requests
    assert f(2, 1, 317, 16, 64, 4, da.KV_BF16, 592) == 16                  # too small to fill the bins
    # every workload whose tile length the configs leave open uses the rule's length
    for name in ("uniform", "long_b1", "long_b4", "fp8_spec"):
        c = W.CONFIGS[name]
        L = np.asarray(W.config_seq_lens(name), dtype=np.int64)
        kv = da.KV_BF16 if c["kv_dtype"] == "bf16" else da.KV_FP8E4M3
        rows = c["n_q_heads"] // c["n_kv_heads"] * c["q_tokens"]
        assert f(len(L), c["n_kv_heads"], int(L.sum()), c["page_size"], c["head_dim"], rows, kv, 592) == c["tile_len"], name
    for P in (16, 32, 48, 64, 256):
        tl = f(8, 8, 100000, P, 128, 8, da.KV_BF16, 592)
        assert tl > 0 and tl % P == 0 and tl % 16 == 0
    # more query rows per KV head -> more partial bytes per tile -> tiles no shorter
    a = f(16, 8, 270000, 16, 128, 4, da.KV_FP8E4M3, 592)
    b = f(16, 8, 270000, 16, 128, 64, da.KV_FP8E4M3, 592)
    assert b >= a
    assert f(0, 8, 100, 16, 128, 4, da.KV_BF16, 592) == da.EINVAL
    assert f(4, 8, 100, 24, 128, 4, da.KV_BF16, 592) == da.EINVAL           # page not a multiple of 16
    assert f(4, 8, 100, 16, 128, 4, da.KV_BF16, 0) == da.EINVAL


def test_append_rope_fp8_rejects_bad_args(lib):
    def call(s, **kw):
        args = dict(q=FAKE, k=FAKE, v=FAKE, tab=FAKE, lens=FAKE, qo=FAKE, kp=FAKE, vp=FAKE, sc=FAKE)
        args.update(kw)
        return lib.dec_attn_append_rope_fp8(C.byref(s), args["q"], args["k"], args["v"], args["tab"], args["lens"],
                                            10000.0, args["qo"], args["kp"], args["vp"], args["sc"], None, None)
    assert call(_shape(kv_dtype=da.KV_BF16)) == da.ENOTSUP          # bf16 pages go through dec_attn_append_rope
    assert call(_shape(kv_dtype=da.KV_FP8E4M3, head_dim=96)) == da.ENOTSUP
    assert call(_shape(kv_dtype=da.KV_FP8E4M3), sc=None) == da.EINVAL
    assert call(_shape(kv_dtype=da.KV_FP8E4M3), sc=FAKE + 2) == da.EALIGN
    assert call(_shape(kv_dtype=da.KV_FP8E4M3), q=FAKE + 2) == da.EALIGN


def test_prefill_fp8_workspace_and_host_checks(lib):
    # the widened pool: K and V bf16 [B * max_pages_per_seq][Hkv][P][128], then its page table
    s = _shape(kv_dtype=da.KV_FP8E4M3, q_tokens=300)
    B, mpps, Hkv, P, d = s.batch, s.max_pages_per_seq, s.n_kv_heads, s.page_size, s.head_dim
    kv = -(-(B * mpps * Hkv * P * d * 2) // 256) * 256
    need = lib.dec_attn_prefill_fp8_workspace_bytes(C.byref(s))
    assert need == 2 * kv + -(-(B * mpps * 4) // 256) * 256
    assert lib.dec_attn_prefill_fp8_workspace_bytes(None) == da.EINVAL

    def call(shape, ws_bytes=need, total=None, **kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, sc=FAKE, tab=FAKE, lens=FAKE, cu=None, ws=FAKE, out=FAKE, lse=FAKE)
        a.update(kw)
        total = shape.batch * shape.q_tokens if total is None else total
        return lib.dec_attn_prefill_fp8(C.byref(shape), a["q"], a["k"], a["v"], a["sc"], a["tab"], a["lens"], a["cu"],
                                        total, a["ws"], ws_bytes, a["out"], a["lse"], None, None)
    # every case fails a host check before any tensor map is built or a kernel launched
    assert lib.dec_attn_prefill_fp8(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, FAKE, need, FAKE, FAKE,
                                    None, None) == da.EINVAL
    assert call(_shape(kv_dtype=da.KV_BF16, q_tokens=300)) == da.ENOTSUP      # bf16 pools: dec_attn_prefill
    assert call(_shape(kv_dtype=da.KV_FP8E4M3_MMA8, q_tokens=300)) == da.ENOTSUP
    assert call(_shape(kv_dtype=da.KV_FP8E4M3, q_tokens=300, head_dim=64)) == da.ENOTSUP
    assert call(_shape(kv_dtype=da.KV_FP8E4M3, q_tokens=300, page_size=8)) == da.ENOTSUP
    assert call(_shape(kv_dtype=da.KV_FP8E4M3, q_tokens=0)) == da.EINVAL
    assert call(s, total=5) == da.EINVAL                  # no row offsets: batch * q_tokens rows
    for name in ("k", "v", "sc", "tab", "lens", "ws"):
        assert call(s, **{name: None}) == da.EINVAL
    assert call(s, k=FAKE + 8) == da.EALIGN
    assert call(s, ws=FAKE + 8) == da.EALIGN
    assert call(s, sc=FAKE + 2) == da.EALIGN
    assert call(s, ws_bytes=need - 1) == da.ESMALL
    assert call(_shape(kv_dtype=da.KV_FP8E4M3, batch=0, q_tokens=300), q=None, k=None, v=None, sc=None, tab=None,
                lens=None, ws=None, out=None, lse=None) == da.OK
