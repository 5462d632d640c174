"""Block-sparse decode on the GPU against the fp64 oracle, through the C ABI: the sparse planner's
work list byte-exact against the oracle's sequential greedy over the kept tiles, and attention
over the kept tiles within out 2e-3 / lse 1e-4."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_29_b200 as da
import workloads as W
from tests import _gpu as U

pytestmark = pytest.mark.gpu


def _mask_dev(mask):
    return torch.from_numpy(np.ascontiguousarray(mask).view(np.int32)).cuda()


def _random_mask(lens, hkv, tl, density, seed, words=None):
    rng = np.random.default_rng(seed)
    nb = (np.asarray(lens, dtype=np.int64) + tl - 1) // tl
    words = words or max(1, int((nb.max() + 31) // 32))
    keep = rng.random((len(lens), hkv, words * 32)) < density
    bits = keep.reshape(len(lens), hkv, words, 32).astype(np.uint64) << np.arange(32, dtype=np.uint64)
    m = bits.sum(axis=-1).astype(np.uint32)
    # stray bits past a request's last tile must be ignored
    return m


def gpu_plan_sparse(lens, mask, hkv, tl, n_bins, max_total=None):
    t = torch.tensor(np.asarray(lens, dtype=np.int32), device="cuda")
    total = int(np.asarray(lens, dtype=np.int64).clip(0).sum()) if max_total is None else max_total
    pl = da.plan_sparse(t, _mask_dev(mask), hkv, tl, max_total_kv_tokens=total, n_bins=n_bins)
    st = da.read_status(pl)
    return pl, st, da.plan_contents(pl, t)


@pytest.mark.parametrize("lens,hkv,tl,n_bins,density", [
    ([5, 300, 1000, 64], 2, 64, 7, 0.5),
    ([4096] * 32, 8, 256, 592, 0.3),
    ([17, 18, 1, 0, 999, 257], 3, 16, 11, 0.7),
    ([131072], 8, 256, 592, 0.1),
    ([700, 1, 33, 2000, 64, 65] * 20, 4, 64, 148, 0.5),
    ([40] * 3, 2, 16, 5, 0.0),
    ([300] * 200, 8, 256, 592, 0.5),      # many kept partial tiles of one cost
    ([5000 + 41 * i for i in range(64)], 8, 256, 592, 0.3),
])
def test_sparse_plan_matches_oracle(lens, hkv, tl, n_bins, density):
    mask = _random_mask(lens, hkv, tl, density, seed=len(lens) + hkv)
    pl, st, got = gpu_plan_sparse(lens, mask, hkv, tl, n_bins)
    assert st == da.OK, da.status_string(st)
    ref = oracle.plan(lens, hkv, tl, n_bins, tile_mask=mask)
    assert got["n_units"] == ref["n_units"]
    assert np.array_equal(got["bin_off"], ref["bin_off"])
    assert np.array_equal(got["units"], ref["units"]), "work lists differ"


def test_sparse_plan_all_ones_equals_dense_plan():
    lens, hkv, tl, n_bins = [5, 300, 1000, 64, 4096], 2, 64, 37
    mask = np.full((len(lens), hkv, 4), 0xFFFFFFFF, dtype=np.uint32)
    _, st, got = gpu_plan_sparse(lens, mask, hkv, tl, n_bins)
    assert st == da.OK
    t = torch.tensor(np.asarray(lens, dtype=np.int32), device="cuda")
    dense = da.plan_contents(da.plan(t, hkv, tl, max_total_kv_tokens=sum(lens), n_bins=n_bins), t)
    assert np.array_equal(got["units"], dense["units"]) and np.array_equal(got["bin_off"], dense["bin_off"])


def test_sparse_plan_capacity_and_bad_length():
    lens = [500, 600]
    mask = np.full((2, 2, 1), 0xFFFFFFFF, dtype=np.uint32)
    pl, st, got = gpu_plan_sparse(lens, mask, 2, 64, 9, max_total=100)
    assert st == da.ECAPACITY and got["n_units"] == -1
    pl, st, _ = gpu_plan_sparse([-5, 64], mask, 2, 64, 9, max_total=64)
    assert st == da.EDEVICE


def _sparse_problem(lens, *, Hq=8, Hkv=2, d=128, P=16, T=1, kv="bf16", tl=64, density=0.5, seed=9, mask=None):
    pr = W.make_problem(name="sparse", batch=len(lens), n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_lens=lens,
                        page_size=P, q_tokens=T, kv_dtype=kv, seed=seed, tile_len=tl)
    pr.tile_mask = W.make_tile_mask(pr, density, keep_last=False) if mask is None else mask
    return pr


def _run_sparse(pr, dev=None):
    dev = dev or U.to_device(pr)
    total = int(pr.seq_lens.astype(np.int64).sum())
    pl = da.plan_sparse(dev["lens"], _mask_dev(pr.tile_mask), pr.n_kv_heads, pr.tile_len, max_total_kv_tokens=total)
    out, lse = da.run(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], pl, kv_scales=dev["sc"],
                      sm_scale=pr.sm_scale)
    return out, lse, da.read_status(pl)


@pytest.mark.parametrize("kv", ["bf16", "fp8e4m3"])
@pytest.mark.parametrize("G,T,d", [(4, 1, 128), (8, 1, 128), (1, 1, 64), (4, 4, 128), (2, 3, 64)])
def test_sparse_decode_matches_oracle(kv, G, T, d):
    pr = _sparse_problem([1, 40, 300, 1000, 2049], Hq=2 * G, Hkv=2, d=d, T=T, kv=kv, density=0.5)
    out, lse, st = _run_sparse(pr)
    assert st == da.OK, da.status_string(st)
    ref_o, ref_l = oracle.decode(pr)
    U.check_rows(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, f"sparse {kv} G{G} T{T}")


def test_sparse_edge_pairs():
    # per pair: every tile masked; one tile kept (the split kernel writes the row); only the
    # partial tile kept; every tile kept; a tile mask wider than the request; an empty request
    lens = [300, 300, 300, 300, 300, 0]
    mask = np.zeros((6, 2, 2), dtype=np.uint32)
    mask[1, :, 0] = 1 << 2
    mask[2, :, 0] = 1 << 4                      # tile 4 = tokens 256..299, the partial tile
    mask[3, :, 0] = 0b11111
    mask[4, :, :] = 0xFFFFFFFF                  # stray bits past tile 4 are ignored
    mask[5, :, :] = 0xFFFFFFFF
    mask[0, 1, 0] = 0b10                        # request 0: head 0 fully masked, head 1 keeps tile 1
    pr = _sparse_problem(lens, Hq=8, Hkv=2, d=128, T=2, tl=64, mask=mask)
    out, lse, st = _run_sparse(pr)
    assert st == da.OK, da.status_string(st)
    ref_o, ref_l = oracle.decode(pr)
    U.check_rows(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, "sparse edges")


def test_all_ones_sparse_decode_is_the_dense_decode_bit_for_bit():
    pr = _sparse_problem([17, 300, 1000, 4096], Hq=16, Hkv=2, d=128, T=1, tl=64,
                         mask=np.full((4, 2, 2), 0xFFFFFFFF, dtype=np.uint32))
    dev = U.to_device(pr)
    out_s, lse_s, st = _run_sparse(pr, dev)
    assert st == da.OK
    out_d, lse_d, _, st_d = U.run_problem(pr, dev)
    assert st_d == da.OK
    assert torch.equal(out_s, out_d) and torch.equal(lse_s, lse_d)


def test_sparse_full_size_mixed_all_rows():
    pr = W.make_config("mixed")
    pr.tile_mask = W.make_tile_mask(pr, 0.3)
    out, lse, st = _run_sparse(pr)
    assert st == da.OK, da.status_string(st)
    ref_o, ref_l = oracle.decode(pr)
    U.check_rows(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, "mixed, 30% of tiles")


def test_sparse_plan_and_run_in_one_cuda_graph():
    pr = _sparse_problem([200, 513, 64, 1000], Hq=8, Hkv=2, d=128, T=1, tl=64, density=0.6)
    dev = U.to_device(pr)
    total = int(pr.seq_lens.sum())
    m = _mask_dev(pr.tile_mask)
    pl = da.plan_sparse(dev["lens"], m, 2, 64, max_total_kv_tokens=total)
    shape = da.make_shape(dev["q"], dev["k"], dev["tab"], da.KV_BF16)
    ws = torch.empty(da.workspace_bytes(shape, pl), dtype=torch.uint8, device="cuda")
    out = torch.empty(pr.batch, 1, pr.n_q_heads, pr.head_dim, device="cuda")
    lse = torch.empty(pr.batch, 1, pr.n_q_heads, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        da.plan_sparse(dev["lens"], m, 2, 64, max_total_kv_tokens=total, buf=pl.buf, stream=s)
        da.run(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], pl, sm_scale=pr.sm_scale, workspace=ws,
               out=out, lse=lse, stream=s)
    g.replay()
    torch.cuda.synchronize()
    ref_o, ref_l = oracle.decode(pr)
    U.check_rows(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, "graph: sparse plan + run")
