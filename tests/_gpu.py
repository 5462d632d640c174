"""Moves a workloads.Problem to the GPU and runs it through the C ABI binding."""
from __future__ import annotations

import numpy as np
import torch

import paged_kv_decode_29_b200 as da

OUT_ATOL = 2e-3   # max abs error of out against the fp64 oracle
LSE_ATOL = 1e-4   # max abs error of lse against the fp64 oracle


def to_device(pr, device="cuda"):
    q = torch.from_numpy(np.ascontiguousarray(pr.q).view(np.int16)).view(torch.bfloat16).to(device)
    if pr.kv_dtype == "bf16":
        k = torch.from_numpy(np.ascontiguousarray(pr.k_pages).view(np.int16)).view(torch.bfloat16).to(device)
        v = torch.from_numpy(np.ascontiguousarray(pr.v_pages).view(np.int16)).view(torch.bfloat16).to(device)
        sc = None
    else:
        k = torch.from_numpy(np.ascontiguousarray(pr.k_pages)).to(device)
        v = torch.from_numpy(np.ascontiguousarray(pr.v_pages)).to(device)
        sc = torch.from_numpy(np.ascontiguousarray(pr.kv_scales)).to(device)
    tab = torch.from_numpy(np.ascontiguousarray(pr.page_table)).to(device)
    lens = torch.from_numpy(np.ascontiguousarray(pr.seq_lens)).to(device)
    return dict(q=q, k=k, v=v, tab=tab, lens=lens, sc=sc)


GUARD = 256          # canary bytes after the plan buffer, the workspace, out and lse
CANARY = 0xA5


def _guarded(nbytes, device):
    """A device byte buffer of nbytes followed by GUARD canary bytes; returns (whole, head view)."""
    whole = torch.full((nbytes + GUARD,), CANARY, dtype=torch.uint8, device=device)
    return whole, whole[:nbytes]


def check_canaries(*wholes):
    for w in wholes:
        tail = w[-GUARD:]
        assert bool(torch.all(tail == CANARY)), "a kernel wrote past the end of its buffer"


def run_problem(pr, dev=None, tile_len=None, n_bins=0, sync=True):
    """Plan + split + combine through the C ABI. The plan buffer, the workspace, out and lse each
    end in GUARD canary bytes, checked unchanged after the run."""
    dev = dev or to_device(pr)
    tl = tile_len or pr.tile_len
    total = int(pr.seq_lens.astype(np.int64).sum())
    d = dev["q"].device
    pb_whole, pbuf = _guarded(da.plan_bytes(pr.batch, pr.n_kv_heads, tl, total, n_bins), d)
    pl = da.plan(dev["lens"], pr.n_kv_heads, tl, max_total_kv_tokens=total, n_bins=n_bins, buf=pbuf)
    shape = da.make_shape(dev["q"], dev["k"], dev["tab"], da.kv_dtype_of(dev["k"]), pr.sm_scale)
    ws_whole, ws = _guarded(da.workspace_bytes(shape, pl), d)
    B, T, Hq, D = dev["q"].shape
    o_whole, o_bytes = _guarded(B * T * Hq * D * 4, d)
    l_whole, l_bytes = _guarded(B * T * Hq * 4, d)
    out = o_bytes.view(torch.float32).view(B, T, Hq, D)
    lse = l_bytes.view(torch.float32).view(B, T, Hq)
    out, lse = da.run(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], pl, kv_scales=dev["sc"],
                      sm_scale=pr.sm_scale, workspace=ws, out=out, lse=lse)
    status = da.read_status(pl, ws) if sync else None
    if sync:
        check_canaries(pb_whole, ws_whole, o_whole, l_whole)
    return out, lse, pl, status


def check_rows(out, lse, ref_out, ref_lse, what=""):
    """out/lse: fp32 arrays; ref: fp64 oracle arrays of the same shape."""
    out = np.asarray(out, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    empty = np.isneginf(ref_lse)
    assert np.array_equal(np.isneginf(lse), empty), f"{what}: -inf lse pattern differs"
    assert np.all(out[empty] == 0), f"{what}: rows with no visible key must be 0"
    full = ~empty
    assert np.all(np.isfinite(out[full])) and np.all(np.isfinite(lse[full])), f"{what}: non-finite"
    e_out = float(np.max(np.abs(out[full] - ref_out[full]))) if full.any() else 0.0
    e_lse = float(np.max(np.abs(lse[full] - ref_lse[full]))) if full.any() else 0.0
    assert e_out <= OUT_ATOL, f"{what}: max |out - oracle| = {e_out:.3e}"
    assert e_lse <= LSE_ATOL, f"{what}: max |lse - oracle| = {e_lse:.3e}"
    return e_out, e_lse
