"""Errors the kernels find on the device, and the bounded-wait path.

The kernels never trap.  A bad index is latched in a device word
(fa_device_error) and replaced by a harmless one, and the rest of the batch
is still computed correctly:
  - a block-table entry outside [0, num_blocks) in fa_decode_paged (bf16 and
    q8_0 caches) is latched as FA_DEVERR_BAD_BLOCK (2) and block 0 is read in
    its place, so the output equals the oracle's on the table with that
    entry set to 0;
  - a sequence longer than its table (seq_len > max_blocks * 64) is latched
    the same way and read up to the table's end; the combine then reads only
    the splits the decode kernel wrote (checked with a workspace filled with
    NaN beforehand);
  - a gather index >= n_rows or < -1 in fa_decode_gather is latched as
    FA_DEVERR_BAD_ROW (3) and the slot is treated as empty.

Bounded waits: fa_debug_decode_paged_stall runs the paged decode with a short
wait limit and a barrier that nothing completes.  The wait runs out, the
kernel returns, FA_DEVERR_TIMEOUT (1) is latched, every row is O = 0 and
LSE = -inf, and the next ordinary call on the same context is correct."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check

pytestmark = pytest.mark.gpu

FA_DEVERR_TIMEOUT, FA_DEVERR_BAD_BLOCK, FA_DEVERR_BAD_ROW = 1, 2, 3


def plant_bad_blocks(table, lens, num_blocks):
    """Two out-of-range ids inside sequence 1's blocks and one in sequence 3's."""
    bad = table.clone()
    nb1 = (int(lens[1]) + 63) // 64
    nb3 = (int(lens[3]) + 63) // 64
    bad[1, 0] = num_blocks + 5
    bad[1, nb1 - 1] = -7
    bad[3, nb3 // 2] = 1 << 30
    fixed = bad.clone()
    fixed[(bad < 0) | (bad >= num_blocks)] = 0
    fixed[table < 0] = -1  # slots past a sequence's end stay unused
    return bad, fixed


def test_paged_bad_block_bf16():
    c = W.PagedCase("badblk", 5, 8, 2, 128, 128, 64, 0, 0, seed=301, lens=(200, 700, 64, 1000, 129))
    q, kc, vc, table, lens = W.paged_inputs(c)
    nbk = kc.shape[0]
    bad, fixed = plant_bad_blocks(table, lens, nbk)
    fa.device_error()  # start from a clear word
    o, lse = fa.decode_paged(q.cuda(), kc.cuda(), vc.cuda(), bad.cuda(), lens.cuda(), scale=c.scale)
    assert fa.device_error() == FA_DEVERR_BAD_BLOCK
    o_ref, l_ref = oracle.decode_paged(W.bits(q), W.bits(kc), W.bits(vc), fixed.numpy(), lens.numpy(), c.scale)
    check(o, o_ref, lse, l_ref, what="bad block ids read as block 0")
    assert fa.device_error() == 0  # cleared by the read above


def test_paged_bad_block_q8_0():
    c = W.PagedCase("badblk8", 5, 8, 2, 128, 128, 64, 0, 0, seed=302, lens=(300, 640, 1, 900, 65))
    q, _, _, table, lens = W.paged_inputs(c)
    nbk = int(table.max()) + 1
    kq, vq = W.paged_q8_caches(c, nbk)
    bad, fixed = plant_bad_blocks(table, lens, nbk)
    fa.device_error()
    o, lse = fa.decode_paged(q.cuda(), kq.cuda(), vq.cuda(), bad.cuda(), lens.cuda(), scale=c.scale)
    assert fa.device_error() == FA_DEVERR_BAD_BLOCK
    kb = oracle.dequant_rows(kq.numpy(), "q8_0", 128)
    vb = oracle.dequant_rows(vq.numpy(), "q8_0", 128)
    o_ref, l_ref = oracle.decode_paged(W.bits(q), kb, vb, fixed.numpy(), lens.numpy(), c.scale)
    check(o, o_ref, lse, l_ref, what="q8_0 bad block ids read as block 0")


@pytest.mark.parametrize("entry", ["workspace", "noalloc"])
def test_paged_sequence_longer_than_its_table(entry):
    # 9 table slots, 4 splits of 3 blocks: a sequence of 9 * 64 + 100 keys is
    # read up to its table's end (576 keys) and latched; split 3 of it holds
    # no block and writes no partial, so the combine must not read one.
    c = W.PagedCase("longseq", 3, 8, 2, 128, 128, 64, 0, 0, seed=303, lens=(576, 300, 576))
    q, kc, vc, table, lens = W.paged_inputs(c)
    assert table.shape[1] == 9
    long_lens = lens.clone()
    long_lens[0] = 9 * 64 + 100
    dq, dk, dv, dt, dl = q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), long_lens.cuda()
    fa.device_error()
    if entry == "workspace":
        n = fa.paged_workspace_bytes(dq, dk, dv, dt, dl, num_splits=4)
        ws = torch.full((n // 4 + 64,), float("nan"), device="cuda")  # poisoned partials
        o, lse = fa.decode_paged(dq, dk, dv, dt, dl, scale=c.scale, num_splits=4, workspace=ws)
    else:
        lib = fa.load()
        fn = lib.fa_decode_paged_noalloc
        fn.argtypes = [ctypes.POINTER(fa.PagedParams), ctypes.c_void_p]
        fn.restype = ctypes.c_int
        # first fill the fixed scratch with another call's partials (NaN-free
        # but unrelated), then run the long sequence
        o0 = torch.empty(3, 8, 128, device="cuda")
        l0 = torch.empty(3, 8, device="cuda")
        p0 = fa.paged_params(dq, dk, dv, dt, lens.cuda(), o0, l0, 7.5, 4, None)
        assert fn(ctypes.byref(p0), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == fa.FA_OK
        o = torch.empty(3, 8, 128, device="cuda")
        lse = torch.empty(3, 8, device="cuda")
        p = fa.paged_params(dq, dk, dv, dt, dl, o, lse, c.scale, 4, None)
        assert fn(ctypes.byref(p), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == fa.FA_OK
    assert fa.device_error() == FA_DEVERR_BAD_BLOCK
    o_ref, l_ref = oracle.decode_paged(W.bits(q), W.bits(kc), W.bits(vc), table.numpy(), lens.numpy(), c.scale)
    check(o, o_ref, lse, l_ref, what="sequence past its table (%s)" % entry)


def test_gather_bad_row():
    c = W.LatentCase("badrow", 3, 128, 3000, 300, seed=304, select_from_all=True, q_pos0=2500)
    q, rows, idx, qpos = W.latent_inputs(c)
    bad = idx.clone()
    bad[0, 5] = c.n_rows
    bad[0, 200] = c.n_rows + 1000
    bad[2, 17] = -5
    fixed = bad.clone()
    fixed[(bad < -1) | (bad >= c.n_rows)] = -1
    fa.device_error()
    o, lse = fa.decode_gather(q.cuda(), rows.cuda(), bad.cuda(), q_pos=qpos.cuda(), scale=c.scale)
    assert fa.device_error() == FA_DEVERR_BAD_ROW
    o_ref, l_ref = oracle.decode_latent(W.bits(q), W.bits(rows), fixed.numpy(), c.scale, c.dk, c.dv, c.v_offset,
                                        None, qpos.numpy())
    check(o, o_ref, lse, l_ref, what="bad rows treated as empty slots")


def stall_fn():
    fn = fa.load().fa_debug_decode_paged_stall
    fn.argtypes = [ctypes.POINTER(fa.PagedParams), ctypes.c_uint64, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    c = W.PagedCase("stall", 6, 8, 2, 128, 128, 64, 0, 0, seed=305, lens=(100, 2000, 64, 4000, 1, 700))
    q, kc, vc, table, lens = [t.cuda() for t in W.paged_inputs(c)]
    fn = stall_fn()
    n = fa.paged_workspace_bytes(q, kc, vc, table, lens)
    ws = torch.empty(max(n, 256), device="cuda", dtype=torch.uint8)
    o = torch.full((6, 8, 128), float("nan"), device="cuda")
    lse = torch.full((6, 8), float("nan"), device="cuda")
    p = fa.paged_params(q, kc, vc, table, lens, o, lse, c.scale, 0, ws)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert fn(ctypes.byref(p), ctypes.c_uint64(10), stream) == fa.FA_ERR_INVALID_ARG  # below 1 us
    assert fn(ctypes.byref(p), ctypes.c_uint64(3 * 10 ** 9), stream) == fa.FA_ERR_INVALID_ARG  # above 2 s
    fa.device_error()
    assert fn(ctypes.byref(p), ctypes.c_uint64(200_000), stream) == fa.FA_OK  # 200 us
    torch.cuda.synchronize()  # returns: the kernel gave up and left
    assert fa.device_error() == FA_DEVERR_TIMEOUT
    assert torch.all(o == 0) and torch.all(lse == -float("inf"))
    # the same context, an ordinary call: correct and clean
    o2, l2 = fa.decode_paged(q, kc, vc, table, lens, scale=c.scale)
    assert fa.device_error() == 0
    qh, kh, vh, th, lh = W.paged_inputs(c)
    o_ref, l_ref = oracle.decode_paged(W.bits(qh), W.bits(kh), W.bits(vh), th.numpy(), lh.numpy(), c.scale)
    check(o2, o_ref, l2, l_ref, what="after the timeout")


def test_bounded_wait_runs_out_with_converter_warps():
    # q8_0 caches: the CTA also runs converter warps between the raw and the
    # bf16 rings.  With the MMA warps stuck on the stall barrier, the
    # converters fill the bf16 ring and then wait for a stage that is never
    # released; the producer waits for raw stages.  Every one of those waits
    # is bounded and watches the abort flag, so the CTA leaves.
    c = W.PagedCase("stall_q8", 6, 8, 2, 128, 128, 64, 0, 0, seed=306, lens=(100, 2000, 64, 4000, 1, 700))
    q, _, _, table, lens = [t.cuda() for t in W.paged_inputs(c)]
    nbk = int(table.max()) + 1
    kq, vq = W.paged_q8_caches(c, nbk)
    kq, vq = kq.cuda(), vq.cuda()
    fn = stall_fn()
    n = fa.paged_workspace_bytes(q, kq, vq, table, lens)
    ws = torch.empty(max(n, 256), device="cuda", dtype=torch.uint8)
    o = torch.full((6, 8, 128), float("nan"), device="cuda")
    lse = torch.full((6, 8), float("nan"), device="cuda")
    p = fa.paged_params(q, kq, vq, table, lens, o, lse, c.scale, 0, ws)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    fa.device_error()
    assert fn(ctypes.byref(p), ctypes.c_uint64(200_000), stream) == fa.FA_OK  # 200 us
    torch.cuda.synchronize()  # returns: every role gave up and left
    assert fa.device_error() == FA_DEVERR_TIMEOUT
    assert torch.all(o == 0) and torch.all(lse == -float("inf"))
    # the same context, an ordinary call over the same caches
    o2, l2 = fa.decode_paged(q, kq, vq, table, lens, scale=c.scale)
    assert fa.device_error() == 0
    kb = oracle.dequant_rows(kq.cpu().numpy(), "q8_0", 128)
    vb = oracle.dequant_rows(vq.cpu().numpy(), "q8_0", 128)
    o_ref, l_ref = oracle.decode_paged(W.bits(q.cpu()), kb, vb, table.cpu().numpy(), lens.cpu().numpy(), c.scale)
    check(o2, o_ref, l2, l_ref, what="q8_0 after the timeout")
