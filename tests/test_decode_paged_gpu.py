"""Paged split-KV decode parity: CUDA path (C ABI) vs the fp64 oracle, plus
bit-exact block-table indexing probes."""
import math

import numpy as np
import pytest
import torch

import oracle
from attention_attn_fwd_11_b200 import fa
from attention_attn_fwd_11_b200 import workloads as W
from parity import check

pytestmark = pytest.mark.gpu


def run(c, num_splits=0, out_dtype=torch.float32, sample=None):
    q, kc, vc, table, lens = W.paged_inputs(c)
    dev = [t.cuda() for t in (q, kc, vc, table, lens)]
    o, lse = fa.decode_paged(*dev, scale=c.scale, num_splits=num_splits, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.device_error() == 0
    o, lse = o.cpu(), lse.cpu()
    if sample is not None:
        rows = sample
        qb = W.bits(q)[rows]
        o_ref, l_ref = oracle.decode_paged(qb, W.bits(kc), W.bits(vc), table.numpy()[rows], lens.numpy()[rows], c.scale)
        return o[rows], lse[rows], o_ref, l_ref
    o_ref, l_ref = oracle.decode_paged(W.bits(q), W.bits(kc), W.bits(vc), table.numpy(), lens.numpy(), c.scale)
    return o, lse, o_ref, l_ref


@pytest.mark.parametrize("group", [1, 2, 4, 8])
def test_edge_lengths(group):
    lens = (0, 1, 63, 64, 65, 127, 128, 129, 1000, 3)
    c = W.PagedCase("t", len(lens), 2 * group, 2, 128, 128, 64, 0, 0, seed=group, lens=lens)
    o, lse, o_ref, l_ref = run(c)
    check(o, o_ref, lse, l_ref, what="group %d" % group)


@pytest.mark.parametrize("splits", [1, 2, 3, 7, 64])
def test_explicit_splits(splits):
    c = W.PagedCase("t", 6, 8, 2, 128, 128, 64, 1, 2000, seed=50 + splits)
    o, lse, o_ref, l_ref = run(c, num_splits=splits)
    check(o, o_ref, lse, l_ref, what="splits %d" % splits)


def test_bf16_output():
    c = W.PagedCase("t", 5, 8, 2, 128, 128, 64, 1, 700, seed=61)
    o, lse, o_ref, l_ref = run(c, out_dtype=torch.bfloat16)
    check(o, o_ref, lse, l_ref, what="bf16 output")


def test_paged_config_sampled():
    """B=64, Hq=32, Hkv=8, d=128, block 64, Sk ~ U[1024, 8192] -- the
    benchmark launch; sequences sampled for the oracle."""
    c = W.PAGED_GQA
    rows = [0, 1, 17, 31, 32, 47, 63]
    o, lse, o_ref, l_ref = run(c, sample=rows)
    check(o, o_ref, lse, l_ref, what=c.name)


def test_block_table_indexing_bitexact():
    """One key per query head scores ~360 above every other (exp underflows to
    exactly 0 in fp32), so the output must be that key's V row bit for bit.
    V rows encode (block id, slot, kv head) as exact bf16 integers; the target
    walks over block starts/ends, slots and split boundaries."""
    B, Hq, Hkv, bs = 8, 8, 2, 64
    lens = [1, 64, 65, 200, 640, 1000, 4097, 130]
    c = W.PagedCase("t", B, Hq, Hkv, 128, 128, bs, 0, 0, seed=77, lens=tuple(lens))
    _, kc, vc, table, lens_t = W.paged_inputs(c)
    nb = kc.shape[0]
    kc = torch.zeros_like(kc)
    vc = torch.zeros_like(vc)
    blk = torch.arange(nb).view(nb, 1, 1).expand(nb, Hkv, bs)
    slot = torch.arange(bs).view(1, 1, bs).expand(nb, Hkv, bs)
    head = torch.arange(Hkv).view(1, Hkv, 1).expand(nb, Hkv, bs)
    vc[..., 0] = (blk % 256).to(torch.bfloat16)
    vc[..., 1] = (blk // 256).to(torch.bfloat16)
    vc[..., 2] = slot.to(torch.bfloat16)
    vc[..., 3] = head.to(torch.bfloat16)
    q = torch.zeros(B, Hq, 128, dtype=torch.bfloat16)
    q[..., 0] = 64.0
    rng = np.random.default_rng(5)
    for trial in range(3):
        kk = kc.clone()
        targets = []
        for b in range(B):
            n = lens[b]
            j = [0, n - 1, int(rng.integers(0, n))][trial]
            targets.append(j)
            pb = int(table[b, j // bs])
            kk[pb, :, j % bs, 0] = 64.0
        for splits in (1, 3, 0):
            o, _ = fa.decode_paged(q.cuda(), kk.cuda(), vc.cuda(), table.cuda(), lens_t.cuda(), num_splits=splits)
            torch.cuda.synchronize()
            o = o.cpu()
            for b in range(B):
                j = targets[b]
                pb = int(table[b, j // bs])
                for h in range(Hq):
                    want = vc[pb, h // (Hq // Hkv), j % bs].float()
                    assert torch.equal(o[b, h], want), (trial, splits, b, h, j)
