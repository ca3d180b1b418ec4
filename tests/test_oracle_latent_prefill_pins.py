"""Pin for the latent (MLA) prefill the gather path serves with contiguous
rows: Sq new tokens x Hq heads against rows 0 .. Sk - 1, token t at position
Sk - Sq + t ("MLA Decode Attention Kernel API Reference": rows [k_pe |
kv_latent], key = the whole row, value = the latent part; causal mask from
positions).  It must equal dense multi-query attention -- one KV head, K the
full 576-wide rows, V their last 512 columns, bottom-right causal -- computed
by the oracle's separate dense routine."""
import numpy as np
import pytest

import oracle
from attention_attn_fwd_11_b200 import workloads as W


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(5, 9), (9, 9), (3, 40)])
def test_latent_prefill_equals_dense_mqa(causal, Sq, Sk):
    Hq, scale = 4, 1.0 / 24
    q = W.bits(W.randn_bf16((Sq, Hq, 576), 1 + Sq))
    rows = W.bits(W.randn_bf16((Sk, 576), 2 + Sk))
    idx = np.tile(np.arange(Sk, dtype=np.int32), (Sq, 1))
    q_pos = np.arange(Sk - Sq, Sk, dtype=np.int32) if causal else None
    o, lse = oracle.decode_latent(q, rows, idx, scale, 576, 512, 64, q_pos=q_pos)
    qd = np.ascontiguousarray(q.transpose(1, 0, 2))[None]           # [1, Hq, Sq, 576]
    k = rows[None, None]                                             # [1, 1, Sk, 576]
    v = np.ascontiguousarray(rows[:, 64:])[None, None]               # [1, 1, Sk, 512]
    od, ld = oracle.attention(qd, k, v, scale, causal)
    assert np.allclose(o, od[0].transpose(1, 0, 2), rtol=0, atol=1e-13)
    assert np.allclose(lse, ld[0].T, rtol=0, atol=1e-13)
