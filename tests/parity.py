"""Shared parity checks for the GPU tests: the tolerances stated for this
path (bf16 inputs, fp32 accumulation): max |O - O_ref| <= 1e-2, cosine
(fp64, flattened) >= 0.99999, |LSE - LSE_ref| <= 1e-3 where a key is
visible, and -inf exactly where none is.

bf16 OUTPUT (an option; the workloads write fp32): the kernel rounds its
fp32 result o32 once more, to bf16, and that rounding alone moves an element
by up to the unit roundoff u = 2^-8 of its magnitude.  With |o32 - ref| <=
1e-2 (the stated bar) and |o32| <= |ref| + 1e-2, the bf16 value satisfies

    |o_bf16 - ref| <= 1e-2 + u (|ref| + 1e-2)

element by element, and that is the bound checked (out_bf16=True).  The
cosine bar is unchanged: the relative rms of the extra rounding is about
u / sqrt(3) = 2.3e-3, which lowers the cosine by ~u^2/6 = 2.5e-6 at most."""
import numpy as np
import torch

MAX_ABS = 1e-2
MIN_COS = 0.99999
LSE_ABS = 1e-3
BF16_U = 2.0 ** -8  # unit roundoff of bf16 (8 significant bits, round to nearest)


def as_np(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def check(o, o_ref, lse=None, lse_ref=None, max_abs=MAX_ABS, min_cos=MIN_COS, lse_abs=LSE_ABS, what="",
          out_bf16=None):
    if out_bf16 is None:
        out_bf16 = isinstance(o, torch.Tensor) and o.dtype == torch.bfloat16
    o, o_ref = as_np(o), as_np(o_ref)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.isfinite(o).all(), what + ": non-finite output"
    diff = np.abs(o - o_ref)
    if out_bf16:
        # the derived bound above: the stated bar plus the output's own rounding
        allow = max_abs + BF16_U * (np.abs(o_ref) + max_abs)
        excess = (diff - allow).max() if o.size else -1.0
        err = diff.max() if o.size else 0.0
        assert excess <= 0.0, "%s: bf16 output off by %.3e beyond 1e-2 + u(|ref| + 1e-2) (max abs err %.3e)" % (
            what, excess, err)
    else:
        err = diff.max() if o.size else 0.0
        assert err <= max_abs, "%s: max abs err %.3e > %.1e" % (what, err, max_abs)
    a, b = o.ravel(), o_ref.ravel()
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        cos = 1.0
    else:
        cos = float(a @ b / (na * nb)) if na > 0 and nb > 0 else 0.0
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
