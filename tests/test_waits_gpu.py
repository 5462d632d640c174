"""Failure detection without a GPU fault: every pipeline wait of the split kernels (warp-MMA and
tcgen05) and of the prefill kernel is bounded. A test lowers the limit to 1 ms and leaves one
pipeline fill of CTA 0 out (dec_attn_test_set_waits), so that nothing ever completes the waits on
it: the run must end with DECATTN_ETIMEOUT in the status word, the CTA must leave in order (copies
already issued land, tensor memory is freed), and the context must stay usable -- the next run,
with the default limit and no fill left out, matches the oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_decode_29_b200 as da
import workloads as W
from tests import _gpu as U

pytestmark = pytest.mark.gpu

LIMIT_NS = 1_000_000


@pytest.fixture(autouse=True)
def _restore_waits():
    yield
    da.test_set_waits(0, -1)   # back to the defaults whatever happened


def _decode_problem(kv, G, T, d):
    # long enough that bin 0 holds several tiles of many 16-key blocks
    return W.make_problem(name="waits", batch=4, n_q_heads=2 * G, n_kv_heads=2, head_dim=d,
                          seq_lens=[3000, 2500, 4000, 1000], page_size=16, q_tokens=T, kv_dtype=kv, seed=31,
                          tile_len=512)


@pytest.mark.parametrize("kv,G,T,d,mma8,kernel", [
    ("bf16", 4, 1, 128, False, "split_kernel, 1 consumer warp"),
    ("bf16", 8, 4, 128, False, "split_kernel, 4 consumer warps"),
    ("fp8e4m3", 4, 2, 64, False, "split_kernel, FP8"),
    ("fp8e4m3", 4, 4, 128, False, "split_tc_kernel"),
    ("fp8e4m3", 4, 1, 128, True, "split_tc_kernel, FP8 products"),
])
def test_decode_wait_runs_out_then_the_context_is_usable(kv, G, T, d, mma8, kernel):
    pr = _decode_problem(kv, G, T, d)
    dev = U.to_device(pr)
    total = int(pr.seq_lens.sum())
    da.test_set_waits(LIMIT_NS, 2)
    pl = da.plan(dev["lens"], pr.n_kv_heads, pr.tile_len, max_total_kv_tokens=total)
    da.run(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], pl, kv_scales=dev["sc"], mma8=mma8)
    assert da.read_status(pl) == da.ETIMEOUT, kernel
    da.test_set_waits(0, -1)
    torch.cuda.synchronize()   # the context is still usable
    pl = da.plan(dev["lens"], pr.n_kv_heads, pr.tile_len, max_total_kv_tokens=total)
    out, lse = da.run(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], pl, kv_scales=dev["sc"], mma8=mma8)
    assert da.read_status(pl) == da.OK
    if not mma8:
        ref_o, ref_l = oracle.decode(pr)
        U.check_rows(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, kernel)


def test_prefill_wait_runs_out_then_the_context_is_usable():
    pr = W.make_problem(name="waits", batch=2, n_q_heads=4, n_kv_heads=2, head_dim=128, seq_lens=[1000, 700],
                        page_size=16, q_tokens=300, kv_dtype="bf16", seed=32, tile_len=64)
    dev = U.to_device(pr)
    st = torch.zeros((), dtype=torch.int32, device="cuda")
    da.test_set_waits(LIMIT_NS, 1)
    da.prefill(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == da.ETIMEOUT
    da.test_set_waits(0, -1)
    st.zero_()
    out, lse = da.prefill(dev["q"], dev["k"], dev["v"], dev["tab"], dev["lens"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == da.OK
    ref_o, ref_l = oracle.decode(pr)
    # the prefill tolerance (tests/test_prefill_gpu.py): lse 1e-4, out 2^-9 max|v| + 1e-5, here with
    # the largest |v| of the whole pool
    vmax = float(np.abs(W.bf16_bits_to_f32(pr.v_pages)).max())
    assert np.all(np.abs(lse.cpu().numpy() - ref_l) <= 1e-4)
    assert np.all(np.abs(out.cpu().numpy() - ref_o) <= 2.0 ** -9 * vmax + 1e-5)
