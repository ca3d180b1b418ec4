"""Latent sparse decode parity: CUDA path (C ABI) vs the fp64 oracle, plus a
bit-exact row-gather probe."""
import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check

pytestmark = pytest.mark.gpu


def run(c, num_splits=0, key_pos=None, use_qpos=True, out_dtype=torch.float32, idx=None, tokens=None):
    q, rows, idx0, qpos = W.latent_inputs(c)
    if idx is not None:
        idx0 = idx
    kp = None if key_pos is None else key_pos.cuda()
    o, lse = fa.decode_gather(q.cuda(), rows.cuda(), idx0.cuda(), key_pos=kp,
                              q_pos=qpos.cuda() if use_qpos else None, scale=c.scale,
                              num_splits=num_splits, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o, lse = o.cpu(), lse.cpu()
    tk = list(range(c.T)) if tokens is None else tokens
    o_ref, l_ref = oracle.decode_latent(W.bits(q)[tk], W.bits(rows), idx0.numpy()[tk], c.scale, c.dk, c.dv,
                                        c.v_offset, None if key_pos is None else key_pos.numpy()[tk],
                                        qpos.numpy()[tk] if use_qpos else None)
    return o[tk], lse[tk], o_ref, l_ref


@pytest.mark.parametrize("topk", [1, 31, 32, 100, 257, 512])
def test_small_topk_masked(topk):
    c = W.LatentCase("t", 3, 128, 4000, topk, seed=topk, select_from_all=True, q_pos0=1500)
    o, lse, o_ref, l_ref = run(c)
    check(o, o_ref, lse, l_ref, what="topk %d" % topk)


@pytest.mark.parametrize("splits", [1, 2, 5, 16])
def test_explicit_splits(splits):
    c = W.LatentCase("t", 2, 128, 3000, 1024, seed=40 + splits, select_from_all=True, q_pos0=2000)
    o, lse, o_ref, l_ref = run(c, num_splits=splits)
    check(o, o_ref, lse, l_ref, what="splits %d" % splits)


def test_empty_slots_and_no_mask():
    c = W.LatentCase("t", 3, 128, 2000, 200, seed=51, select_from_all=True)
    q, rows, idx, qpos = W.latent_inputs(c)
    idx[0, :] = -1          # nothing selected: O = 0, LSE = -inf
    idx[1, ::3] = -1        # holes
    o, lse, o_ref, l_ref = run(c, idx=idx, use_qpos=False)
    check(o, o_ref, lse, l_ref, what="empty slots")
    assert torch.all(o[0] == 0) and torch.all(lse[0] == -float("inf"))


def test_explicit_key_positions():
    c = W.LatentCase("t", 2, 128, 2000, 300, seed=52, select_from_all=True, q_pos0=50)
    q, rows, idx, qpos = W.latent_inputs(c)
    kp = torch.randint(0, 100, idx.shape, generator=torch.Generator().manual_seed(3), dtype=torch.int32)
    o, lse, o_ref, l_ref = run(c, key_pos=kp)
    check(o, o_ref, lse, l_ref, what="key_pos")


def test_bf16_output():
    c = W.LatentCase("t", 2, 128, 2000, 256, seed=53, select_from_all=True, q_pos0=1999)
    o, lse, o_ref, l_ref = run(c, out_dtype=torch.bfloat16)
    check(o, o_ref, lse, l_ref, what="bf16 output")


def test_latent_config_sampled_tokens():
    """T=32, Hq=128, dk=576/dv=512, 65536-row cache, top-2048 -- the benchmark
    launch; tokens sampled for the oracle."""
    c = W.LATENT_SPARSE
    o, lse, o_ref, l_ref = run(c, tokens=[0, 1, 13, 31])
    check(o, o_ref, lse, l_ref, what=c.name)


def test_row_gather_bitexact():
    """For each token one selected row scores 128 nats above every other
    (exp underflows to exactly 0 in fp32), so every head's output must be that
    row's latent part bit for bit.  Rows encode their own index as exact bf16
    integers; token t's query and its target row share a private component
    (1 + t), so a target of one token is invisible to the others."""
    T, n_rows, topk = 4, 5000, 300
    c = W.LatentCase("t", T, 128, n_rows, topk, seed=61, select_from_all=True)
    q, rows, idx, qpos = W.latent_inputs(c)
    base = torch.zeros_like(rows)
    r = torch.arange(n_rows)
    base[:, 64] = (r % 256).to(torch.bfloat16)
    base[:, 65] = (r // 256).to(torch.bfloat16)
    base[:, 66] = 1.0
    qq = torch.zeros_like(q)
    for t in range(T):
        qq[t, :, 1 + t] = 96.0  # 96 * 32 / sqrt(576) = 128 nats
    for trial in range(3):
        rr = base.clone()
        want = []
        for t in range(T):
            j = [0, topk - 1, 137][trial]
            row = int(idx[t, j])
            rr[row, 1 + t] = 32.0
            want.append(row)
        for splits in (1, 4, 0):
            o, _ = fa.decode_gather(qq.cuda(), rr.cuda(), idx.cuda(), num_splits=splits)
            torch.cuda.synchronize()
            o = o.cpu()
            for t in range(T):
                ref = rr[want[t], 64:576].float()
                assert torch.equal(o[t], ref.expand(128, 512)), (trial, splits, t)



def test_decode_512_rows():
    # 512-wide rows that are both key and value (v_offset 0), selected rows, causal by row index
    T, topk, n_rows = 6, 300, 5000
    q = W.randn_bf16((T, 128, 512), 1301)
    rows = W.randn_bf16((n_rows, 512), 2301)
    g = torch.Generator().manual_seed(4301)
    idx = torch.stack([torch.randperm(n_rows, generator=g)[:topk] for _ in range(T)]).to(torch.int32)
    idx[1, 17] = -1
    qpos = torch.randint(0, n_rows, (T,), generator=g).to(torch.int32)
    o, lse = fa.decode_gather(q.cuda(), rows.cuda(), idx.cuda(), q_pos=qpos.cuda(), scale=1 / 24, dk=512)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o_ref, l_ref = oracle.decode_latent(W.bits(q), W.bits(rows), idx.numpy(), 1 / 24, 512, 512, 0, q_pos=qpos.numpy())
    check(o, o_ref, lse, l_ref, what="gather decode 512 rows")
