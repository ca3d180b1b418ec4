"""fp64 CPU oracle for fused attention forward (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it, and
it shares no code with the CUDA library: the arithmetic lives in
``attention_oracle.c`` (plain C, double precision); this module only marshals
numpy arrays into it.

Inputs are bf16 bit patterns (numpy ``uint16``); outputs are ``float64``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc and OpenMP (in place)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_num_threads.restype = i32
        lib.oracle_attention.argtypes = [P, P, P] + [i32] * 7 + [i64] * 9 + [f64, i32, P, P]
        lib.oracle_attention.restype = i32
        lib.oracle_attention_ext.argtypes = ([P, P, P] + [i32] * 7 + [i64] * 9 + [f64, i32, P, i64, i64, i64]
                                             + [f64, f64, P, P, P])
        lib.oracle_attention_ext.restype = i32
        lib.oracle_alibi_slope.argtypes = [i32, i32, f64]
        lib.oracle_alibi_slope.restype = f64
        lib.oracle_paged_gather.argtypes = [P, i32, i32, i32, i32, P, i32, P, i32, i32, P]
        lib.oracle_paged_gather.restype = i32
        lib.oracle_decode_paged.argtypes = [P, P, P, P, i32, P] + [i32] * 7 + [f64, P, P]
        lib.oracle_decode_paged.restype = i32
        lib.oracle_latent_gather.argtypes = [P, i64, i64, i32, P, i32, i32, P, P]
        lib.oracle_latent_gather.restype = i32
        lib.oracle_decode_latent.argtypes = [P, P, i64, i64, i32, i32, i32, P, i32, P, P, i32, i32, f64, P, P]
        lib.oracle_decode_latent.restype = i32
        lib.oracle_lse_combine.argtypes = [i32, i32, i32, P, P, P, P]
        lib.oracle_lse_combine.restype = None
        lib.oracle_mla_tail.argtypes = [P, P, P, i32, i32, i32, i32, i32, P, P]
        lib.oracle_mla_tail.restype = i32
        lib.oracle_round_bf16.argtypes = [f64]
        lib.oracle_round_bf16.restype = ctypes.c_uint16
        lib.oracle_dequant_rows.argtypes = [P, i32, i64, i32, i64, P]
        lib.oracle_dequant_rows.restype = i32
        lib.oracle_dequant_rows_scaled.argtypes = [P, i32, i64, i32, i64, f64, P]
        lib.oracle_dequant_rows_scaled.restype = i32
        lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_to_double.restype = f64
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.asarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16), got %s" % a.dtype)
    return a


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def attention(q, k, v, scale, causal=False):
    """Dense attention.  q: [B,Hq,Sq,dk], k: [B,Hkv,Sk,dk], v: [B,Hkv,Sk,dv]
    (uint16 bf16 bits, any strides with a contiguous last dim).
    Returns (O [B,Hq,Sq,dv] float64, LSE [B,Hq,Sq] float64)."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Hq, Sq, dk = q.shape
    _, Hkv, Sk, _ = k.shape
    dv = v.shape[3]
    for t in (q, k, v):
        if t.size and t.strides[3] != 2:
            raise ValueError("last dimension must be contiguous")
    qs = [s // 2 for s in q.strides[:3]]
    ks = [s // 2 for s in k.strides[:3]]
    vs = [s // 2 for s in v.strides[:3]]
    o = np.zeros((B, Hq, Sq, dv), np.float64)
    lse = np.zeros((B, Hq, Sq), np.float64)
    rc = _load().oracle_attention(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Sk, dk, dv,
                                  *qs, *ks, *vs, float(scale), int(bool(causal)), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attention rejected its arguments")
    return o, lse


def alibi_slope(h, Hq, max_bias):
    """ALiBi slope of query head h (see oracle_alibi_slope)."""
    return float(_load().oracle_alibi_slope(int(h), int(Hq), float(max_bias)))


def attention_ext(q, k, v, scale, causal=False, mask=None, max_bias=0.0, softcap=0.0, sinks=None):
    """Dense attention with the score modifiers (oracle_attention_ext).
    mask: float16 array of shape [Bm, Hm, Sq, Sk] with Bm in {1, B} and
    Hm in {1, Hq} (size-1 dims broadcast), or None.  sinks: [Hq] or None.
    Returns (O [B,Hq,Sq,dv] float64, LSE [B,Hq,Sq] float64)."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, Hq, Sq, dk = q.shape
    _, Hkv, Sk, _ = k.shape
    dv = v.shape[3]
    for t in (q, k, v):
        if t.size and t.strides[3] != 2:
            raise ValueError("last dimension must be contiguous")
    qs = [s // 2 for s in q.strides[:3]]
    ks = [s // 2 for s in k.strides[:3]]
    vs = [s // 2 for s in v.strides[:3]]
    mptr, msb, msh, mss = None, 0, 0, 0
    if mask is not None:
        mask = np.ascontiguousarray(np.asarray(mask, dtype=np.float16))
        Bm, Hm, Sqm, Skm = mask.shape
        if Bm not in (1, B) or Hm not in (1, Hq) or Sqm != Sq or Skm != Sk:
            raise ValueError("mask must be [1|B, 1|Hq, Sq, Sk]")
        mask = mask.view(np.uint16)
        msb = 0 if Bm == 1 else mask.strides[0] // 2
        msh = 0 if Hm == 1 else mask.strides[1] // 2
        mss = mask.strides[2] // 2
        mptr = _ptr(mask)
    sk = None
    if sinks is not None:
        sk = np.ascontiguousarray(np.asarray(sinks, dtype=np.float64))
        if sk.shape != (Hq,):
            raise ValueError("sinks must have one value per query head")
    o = np.zeros((B, Hq, Sq, dv), np.float64)
    lse = np.zeros((B, Hq, Sq), np.float64)
    rc = _load().oracle_attention_ext(_ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, Sq, Sk, dk, dv, *qs, *ks, *vs,
                                      float(scale), int(bool(causal)), mptr, msb, msh, mss, float(max_bias),
                                      float(softcap), _ptr(sk), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attention_ext rejected its arguments")
    return o, lse


def paged_gather(cache, block_table, seq_lens, block_size):
    """Materialise each sequence's keys from a paged cache
    [num_blocks, Hkv, block_size, d]: returns [B, Hkv, max_len, d] uint16."""
    cache = np.ascontiguousarray(_u16(cache))
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    nb, hkv, bs, d = cache.shape
    assert bs == block_size
    B = sl.shape[0]
    max_len = int(sl.max()) if B else 0
    out = np.zeros((B, hkv, max_len, d), np.uint16)
    rc = _load().oracle_paged_gather(_ptr(cache), nb, hkv, bs, d, _ptr(bt), bt.shape[1], _ptr(sl), B,
                                     max_len, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_paged_gather: block table entry out of range")
    return out


def decode_paged(q, k_cache, v_cache, block_table, seq_lens, scale):
    """Paged decode.  q: [B,Hq,dk]; caches [num_blocks,Hkv,block_size,d];
    block_table int32 [B, max_blocks]; seq_lens int32 [B].
    Returns (O [B,Hq,dv] float64, LSE [B,Hq] float64)."""
    q = np.ascontiguousarray(_u16(q))
    kc = np.ascontiguousarray(_u16(k_cache))
    vc = np.ascontiguousarray(_u16(v_cache))
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    B, Hq, dk = q.shape
    nb, Hkv, bs, _ = kc.shape
    dv = vc.shape[3]
    o = np.zeros((B, Hq, dv), np.float64)
    lse = np.zeros((B, Hq), np.float64)
    rc = _load().oracle_decode_paged(_ptr(q), _ptr(kc), _ptr(vc), _ptr(bt), bt.shape[1], _ptr(sl),
                                     B, Hq, Hkv, dk, dv, bs, nb, float(scale), _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode_paged rejected its arguments")
    return o, lse


def prefill_paged(q, k_cache, v_cache, block_table, seq_lens, scale, causal=True, q_lens=None, mask=None,
                  max_bias=0.0, softcap=0.0, sinks=None):
    """Chunked prefill over a paged cache: per sequence b, its keys are
    gathered from the cache (paged_gather) and the dense oracle runs on
    them.  q [B,Hq,Sq,dk]; caches [num_blocks,Hkv,block_size,d]; seq_lens
    counts the new keys too.  q_lens: None, or the new rows per sequence
    (clamped to [0, Sq]); only rows 0 .. q_lens[b] - 1 of sequence b are
    queries, the rest come back as O = 0, LSE = -inf.  mask [1|B, 1|Hq,
    Sq, >= max seq_len] (f16), max_bias, softcap, sinks: the score
    modifiers of attention_ext, applied per sequence with key j of the
    sequence at mask column j.
    Returns (O [B,Hq,Sq,dv], LSE [B,Hq,Sq]) float64."""
    q = _u16(q)
    bs = k_cache.shape[2]
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    kk = paged_gather(k_cache, block_table, sl, bs)
    vv = paged_gather(v_cache, block_table, sl, bs)
    B, Hq, Sq, _ = q.shape
    o = np.zeros((B, Hq, Sq, vv.shape[3]), np.float64)
    lse = np.full((B, Hq, Sq), -np.inf, np.float64)
    for b in range(B):
        n = int(sl[b])
        nq = Sq if q_lens is None else min(max(int(q_lens[b]), 0), Sq)
        if nq == 0:
            continue
        if mask is None and not max_bias and not softcap and sinks is None:
            o[b:b + 1, :, :nq], lse[b:b + 1, :, :nq] = attention(q[b:b + 1, :, :nq], kk[b:b + 1, :, :n],
                                                                 vv[b:b + 1, :, :n], scale, causal)
        else:
            mb = None if mask is None else np.ascontiguousarray(mask[b % mask.shape[0]:b % mask.shape[0] + 1, :, :nq, :n])
            o[b:b + 1, :, :nq], lse[b:b + 1, :, :nq] = attention_ext(
                q[b:b + 1, :, :nq], kk[b:b + 1, :, :n], vv[b:b + 1, :, :n], scale, causal, mask=mb,
                max_bias=max_bias, softcap=softcap, sinks=sinks)
    return o, lse


def latent_gather(rows, idx, row_len):
    """Materialise the selected rows: returns (rows [T,topk,row_len] uint16,
    valid [T,topk] uint8)."""
    rows = _u16(rows)
    if rows.strides[1] != 2:
        raise ValueError("rows must have a contiguous last dim")
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, topk = idx.shape
    out = np.zeros((T, topk, row_len), np.uint16)
    valid = np.zeros((T, topk), np.uint8)
    rc = _load().oracle_latent_gather(_ptr(rows), rows.shape[0], rows.strides[0] // 2, row_len,
                                      _ptr(idx), topk, T, _ptr(out), _ptr(valid))
    if rc != 0:
        raise ValueError("oracle_latent_gather: row index out of range")
    return out, valid


def decode_latent(q, rows, idx, scale, dk, dv, v_offset, key_pos=None, q_pos=None):
    """Latent sparse decode.  q: [T,Hq,dk]; rows: [n_rows, row_stride]
    (uint16); idx int32 [T,topk] (-1 = empty); key_pos int32 [T,topk] or
    None; q_pos int32 [T] or None.  Returns (O [T,Hq,dv], LSE [T,Hq])."""
    q = np.ascontiguousarray(_u16(q))
    rows = _u16(rows)
    if rows.strides[1] != 2:
        raise ValueError("rows must have a contiguous last dim")
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    kp = None if key_pos is None else np.ascontiguousarray(key_pos, dtype=np.int32)
    qp = None if q_pos is None else np.ascontiguousarray(q_pos, dtype=np.int32)
    T, Hq, _ = q.shape
    topk = idx.shape[1]
    o = np.zeros((T, Hq, dv), np.float64)
    lse = np.zeros((T, Hq), np.float64)
    rc = _load().oracle_decode_latent(_ptr(q), _ptr(rows), rows.shape[0], rows.strides[0] // 2, dk, dv,
                                      v_offset, _ptr(idx), topk, _ptr(kp), _ptr(qp), T, Hq, float(scale),
                                      _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode_latent rejected its arguments")
    return o, lse


def lse_combine(o_parts, lse_parts):
    """Merge partial results over disjoint key sets.  o_parts [n,R,dv],
    lse_parts [n,R] (float64).  Returns (O [R,dv], LSE [R])."""
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
    n, R, dv = o_parts.shape
    o = np.zeros((R, dv), np.float64)
    lse = np.zeros((R,), np.float64)
    _load().oracle_lse_combine(n, R, dv, _ptr(o_parts), _ptr(lse_parts), _ptr(o), _ptr(lse))
    return o, lse


QUANT_TYPES = {"q8_0": (8, 34), "q4_0": (4, 18), "fp8_e4m3": (2, 32)}  # type code, bytes per 32 values


def round_bf16(x) -> int:
    """bf16 bit pattern of x, rounded to nearest with ties to even."""
    return int(_load().oracle_round_bf16(float(x)))


def e4m3_value(b) -> float:
    """The value of one FP8 E4M3 byte."""
    return float(_load().oracle_e4m3_to_double(int(b)))


def dequant_rows(src, qtype, row_elems, scale=1.0):
    """Quantised rows -> bf16 bit patterns.  src: uint8 [..., row_bytes]
    (each row holds row_elems values of type ``qtype`` -- 'q8_0' or 'q4_0'
    ggml blocks, or 'fp8_e4m3' bytes times ``scale`` -- then any padding);
    returns uint16 [..., row_elems]."""
    code, bb = QUANT_TYPES[qtype]
    src = np.ascontiguousarray(src, dtype=np.uint8)
    lead = src.shape[:-1]
    n_rows = int(np.prod(lead)) if lead else 1
    out = np.empty(lead + (row_elems,), np.uint16)
    rc = _load().oracle_dequant_rows_scaled(_ptr(src), code, n_rows, row_elems, src.shape[-1], float(scale),
                                            _ptr(out))
    if rc:
        raise ValueError("oracle_dequant_rows: bad arguments")
    return out


def mla_tail(o_lat, w_abs, w_o):
    """MLA decode tail.  o_lat [T, Hq, R] (latent attention output),
    w_abs [Hq, V, R] (out-absorb), w_o [Hd, Hq*V] (o-projection, row = output
    feature), all bf16 bits.  Returns (u [T, Hq*V], y [T, Hd]) float64."""
    o_lat = np.ascontiguousarray(_u16(o_lat))
    w_abs = np.ascontiguousarray(_u16(w_abs))
    w_o = np.ascontiguousarray(_u16(w_o))
    T, Hq, R = o_lat.shape
    _, V, R2 = w_abs.shape
    Hd, K = w_o.shape
    if w_abs.shape[0] != Hq or R2 != R or K != Hq * V:
        raise ValueError("mla_tail: shapes do not match")
    u = np.zeros((T, Hq * V), np.float64)
    y = np.zeros((T, Hd), np.float64)
    if _load().oracle_mla_tail(_ptr(o_lat), _ptr(w_abs), _ptr(w_o), T, Hq, R, V, Hd, _ptr(u), _ptr(y)):
        raise ValueError("oracle_mla_tail rejected its arguments")
    return u, y
