"""dec_attn_run_noalloc: split + combine for callers that cannot allocate device memory (an
engine that owns all device memory and gives plugins no allocation hook, or a fixed device
memory budget with no allocation while decoding). It takes its workspace from the library's
fixed device scratch, so it must match dec_attn_run with a caller workspace, call after call.

This file is collected last on purpose: the first no-alloc call on a device sets up the
scratch, and the test must pass both alone in a fresh process and after every other test."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_29_b200 as da
import workloads as W
from tests import _gpu as U


@pytest.mark.gpu
@pytest.mark.parametrize("kv", ["bf16", "fp8e4m3"])
def test_noalloc_matches_workspace_entry_point_twice(kv):
    pr = W.make_problem(name="noalloc", batch=5, n_q_heads=8, n_kv_heads=2, head_dim=128,
                        seq_lens=[1, 40, 300, 1500, 777], page_size=16, q_tokens=2, kv_dtype=kv, tile_len=64,
                        seed=21)
    dev = U.to_device(pr)
    total = int(pr.seq_lens.sum())
    pl = da.plan(dev["lens"], pr.n_kv_heads, pr.tile_len, max_total_kv_tokens=total)
    ref_out, ref_lse = da.run(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], pl, kv_scales=dev["sc"])
    ref_out, ref_lse = ref_out.cpu().numpy(), ref_lse.cpu().numpy()
    # outputs allocated up front: torch's own allocator must not move device memory in the loop
    out = torch.empty(pr.batch, pr.q_tokens, pr.n_q_heads, pr.head_dim, dtype=torch.float32, device="cuda")
    lse = torch.empty(pr.batch, pr.q_tokens, pr.n_q_heads, dtype=torch.float32, device="cuda")
    free_after_first = None
    for i in range(2):   # the second call reuses the scratch left by the first
        out.zero_()
        lse.zero_()
        da.run_noalloc(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], pl, out, lse, kv_scales=dev["sc"])
        assert da.read_status(pl) == da.OK
        torch.cuda.synchronize()
        if i == 0:
            free_after_first = torch.cuda.mem_get_info()[0]
        else:
            # once set up, a call takes no device memory at all
            assert torch.cuda.mem_get_info()[0] == free_after_first
        # same tolerance as every parity test, against the workspace entry point ...
        U.check_rows(out.cpu().numpy(), lse.cpu().numpy(), ref_out.astype(np.float64),
                     ref_lse.astype(np.float64), "noalloc vs run")
    # ... and the result is also right against the oracle
    o, l = oracle.decode(pr)
    U.check_rows(out.cpu().numpy(), lse.cpu().numpy(), o, l, "noalloc vs oracle")


@pytest.mark.gpu
def test_noalloc_rejects_plans_larger_than_the_scratch():
    # 131072 tokens x 64 requests of partials need far more than the 64 MiB scratch
    lens = torch.full((64,), 131072, dtype=torch.int32, device="cuda")
    pl = da.plan(lens, 8, 16, max_total_kv_tokens=64 * 131072)
    shape = da.ShapeT(64, 32, 8, 128, 1, 16, 8 * 64, 8192, da.KV_BF16, 0.0)
    assert da.load_library().dec_attn_workspace_bytes(C.byref(shape), C.byref(pl.handle)) > da.NOALLOC_SCRATCH_BYTES
    fake = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = fake.data_ptr()
    rc = da.load_library().dec_attn_run_noalloc(C.byref(shape), p, p, p, p, p, None, C.byref(pl.handle), p, p, None)
    assert rc == da.ESMALL


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(n for n in W.CONFIGS if n != "prefill"))
def test_noalloc_scratch_holds_every_decode_workload(name):
    # The scratch is sized for the decode workloads of this library: each one's workspace (partials
    # for every tile the plan can hold, combine counters and chunk states) fits in it.
    c = W.CONFIGS[name]
    lens_h = np.asarray(W.config_seq_lens(name), dtype=np.int32)
    lens = torch.from_numpy(lens_h).cuda()
    total = int(lens_h.astype(np.int64).sum())
    pl = da.plan(lens, c["n_kv_heads"], c["tile_len"], max_total_kv_tokens=total)
    P = c["page_size"]
    pages = int(((lens_h.astype(np.int64) + P - 1) // P).sum())
    kv = da.KV_BF16 if c["kv_dtype"] == "bf16" else da.KV_FP8E4M3
    shape = da.ShapeT(len(lens_h), c["n_q_heads"], c["n_kv_heads"], c["head_dim"], c["q_tokens"], P, pages,
                      int(((lens_h.max() + P - 1) // P)), kv, 0.0)
    need = da.load_library().dec_attn_workspace_bytes(C.byref(shape), C.byref(pl.handle))
    print(f"{name}: workspace {need} bytes ({need / 2**20:.1f} MiB) of {da.NOALLOC_SCRATCH_BYTES >> 20} MiB")
    assert 0 < need <= da.NOALLOC_SCRATCH_BYTES
