"""The allocation-free paged decode entry point, fa_decode_paged_noalloc.

It exists for callers that cannot allocate device memory (a plugin whose
host application owns every allocation, or a serving loop whose memory is
reserved up front and may not call cudaMalloc on its hot path): instead of a
caller-supplied workspace it uses a fixed scratch array inside the library.
This test calls it through the C ABI twice in a row, on two different
workloads, and checks each result against the workspace entry point
(fa_decode_paged) and against the fp64 oracle, within the parity
tolerances used everywhere else.  It
also checks that shapes needing more scratch than the library holds are
rejected before any launch.  The file is named to be collected last.
"""
import ctypes

import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check

pytestmark = pytest.mark.gpu


def noalloc_fn():
    lib = fa.load()
    fn = lib.fa_decode_paged_noalloc
    fn.argtypes = [ctypes.POINTER(fa.PagedParams), ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return lib, fn


def call_noalloc(fn, q, kc, vc, tb, sl, scale, num_splits=0):
    dv = vc.shape[3] // 34 * 32 if vc.dtype == torch.uint8 else vc.shape[3]  # q8_0 rows: 34 bytes per 32 values
    o = torch.full((q.shape[0], q.shape[1], dv), float("nan"), device="cuda")
    lse = torch.full((q.shape[0], q.shape[1]), float("nan"), device="cuda")
    p = fa.paged_params(q, kc, vc, tb, sl, o, lse, scale, num_splits, None)
    st = fn(ctypes.byref(p), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, o, lse


def test_noalloc_matches_workspace_entry_point_twice():
    lib, fn = noalloc_fn()
    cases = [W.PagedCase("noalloc_a", 16, 32, 8, 128, 128, 64, 1, 4000, seed=123),
             W.PagedCase("noalloc_b", 9, 16, 4, 128, 128, 64, 0, 2500, seed=124, lens=(0, 1, 64, 65, 700, 2500, 3, 128, 129))]
    for c in cases:  # two calls in a row; the second finds the first's leftovers in the scratch
        host = W.paged_inputs(c)
        q, kc, vc, tb, sl = [t.cuda() for t in host]
        ref_o, ref_l = fa.decode_paged(q, kc, vc, tb, sl, scale=c.scale)
        st, o, lse = call_noalloc(fn, q, kc, vc, tb, sl, c.scale)
        assert st == fa.FA_OK, lib.fa_last_error().decode()
        torch.cuda.synchronize()
        check(o, ref_o, lse, ref_l, what=c.name)
        qh, kh, vh, th, lh = host
        o64, l64 = oracle.decode_paged(W.bits(qh), W.bits(kh), W.bits(vh), th.numpy(), lh.numpy(), c.scale)
        check(o, o64, lse, l64, what=c.name + " vs the oracle")
    assert fa.device_error() == 0


def test_noalloc_q8_0_caches():
    # the in-kernel q8_0 prologue through the allocation-free entry point
    lib, fn = noalloc_fn()
    c = W.PagedCase("noalloc_q8", 7, 16, 4, 128, 128, 64, 0, 2000, seed=126, lens=(0, 1, 64, 65, 700, 2000, 129))
    q, _, _, tb, sl = W.paged_inputs(c)
    kq, vq = W.paged_q8_caches(c, int(tb.max()) + 1)
    q, kq, vq, tb, sl = q.cuda(), kq.cuda(), vq.cuda(), tb.cuda(), sl.cuda()
    ref_o, ref_l = fa.decode_paged(q, kq, vq, tb, sl, scale=c.scale)
    st, o, lse = call_noalloc(fn, q, kq, vq, tb, sl, c.scale)
    assert st == fa.FA_OK, lib.fa_last_error().decode()
    torch.cuda.synchronize()
    check(o, ref_o, lse, ref_l, what=c.name)
    assert fa.device_error() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib, fn = noalloc_fn()
    c = W.PagedCase("noalloc_big", 64, 32, 8, 128, 128, 64, 1, 64, seed=125)
    q, kc, vc, tb, sl = [t.cuda() for t in W.paged_inputs(c)]
    # 64 * 32 query rows * 128 splits of 516 bytes each is far above 8 MiB
    big_table = torch.zeros(c.B, 4096, dtype=torch.int32, device="cuda")
    st, _, _ = call_noalloc(fn, q, kc, vc, big_table, sl, c.scale, num_splits=128)
    assert st == fa.FA_ERR_WORKSPACE
    assert "fixed scratch" in lib.fa_last_error().decode()
