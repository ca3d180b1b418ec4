"""Shared parity checks for the GPU tests: the tolerances stated for this
path (bf16 inputs, fp32 accumulation): max |O - O_ref| <= 1e-2, cosine
(fp64, flattened) >= 0.99999, |LSE - LSE_ref| <= 1e-3 where a key is
visible, and -inf exactly where none is."""
import numpy as np
import torch

MAX_ABS = 1e-2
MIN_COS = 0.99999
LSE_ABS = 1e-3


def as_np(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def check(o, o_ref, lse=None, lse_ref=None, max_abs=MAX_ABS, min_cos=MIN_COS, lse_abs=LSE_ABS, what=""):
    o, o_ref = as_np(o), as_np(o_ref)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.isfinite(o).all(), what + ": non-finite output"
    err = np.abs(o - o_ref).max() if o.size else 0.0
    a, b = o.ravel(), o_ref.ravel()
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        cos = 1.0
    else:
        cos = float(a @ b / (na * nb)) if na > 0 and nb > 0 else 0.0
    assert err <= max_abs, "%s: max abs err %.3e > %.1e" % (what, err, max_abs)
    assert cos >= min_cos, "%s: cosine %.8f < %.5f" % (what, cos, min_cos)
    if lse is not None:
        lse, lse_ref = as_np(lse), as_np(lse_ref)
        fin = np.isfinite(lse_ref)
        assert np.array_equal(np.isfinite(lse), fin), what + ": LSE finiteness differs"
        assert np.all(lse[~fin] == -np.inf), what + ": empty rows must have LSE = -inf"
        if fin.any():
            le = np.abs(lse[fin] - lse_ref[fin]).max()
            assert le <= lse_abs, "%s: LSE err %.3e > %.1e" % (what, le, lse_abs)
    return err, cos
