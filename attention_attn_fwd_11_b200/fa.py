"""ctypes binding over libfa.so (include/fa.h).  Argument marshalling only:
every step of the computation runs in the library's CUDA kernels.  PyTorch
supplies device memory and the current stream.  There is no CPU fallback:
if the library is missing or the tensors are not on a CUDA device, calls
raise.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa.so")

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_WORKSPACE, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(6)
FA_F32, FA_BF16 = 0, 1
STATUS_NAMES = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_WORKSPACE",
                4: "FA_ERR_CUDA", 5: "FA_ERR_TIMEOUT"}

_vp = ctypes.c_void_p
_i32 = ctypes.c_int
_i64 = ctypes.c_int64


class FwdParams(ctypes.Structure):
    _fields_ = [("q", _vp), ("k", _vp), ("v", _vp), ("o", _vp), ("lse", _vp),
                ("B", _i32), ("Hq", _i32), ("Hkv", _i32), ("Sq", _i32), ("Sk", _i32), ("dk", _i32), ("dv", _i32),
                ("q_sb", _i64), ("q_sh", _i64), ("q_ss", _i64),
                ("k_sb", _i64), ("k_sh", _i64), ("k_ss", _i64),
                ("v_sb", _i64), ("v_sh", _i64), ("v_ss", _i64),
                ("o_sb", _i64), ("o_sh", _i64), ("o_ss", _i64),
                ("scale", ctypes.c_float), ("causal", _i32), ("o_dtype", _i32),
                ("mask", _vp), ("m_sb", _i64), ("m_sh", _i64), ("m_ss", _i64),
                ("max_bias", ctypes.c_float), ("softcap", ctypes.c_float), ("sinks", _vp)]


class PagedParams(ctypes.Structure):
    _fields_ = [("q", _vp), ("k_cache", _vp), ("v_cache", _vp), ("block_table", _vp), ("seq_lens", _vp),
                ("max_blocks_per_seq", _i32), ("B", _i32), ("Hq", _i32), ("Hkv", _i32), ("dk", _i32),
                ("dv", _i32), ("block_size", _i32), ("num_blocks", _i32), ("scale", ctypes.c_float),
                ("num_splits", _i32), ("o", _vp), ("lse", _vp), ("o_dtype", _i32), ("workspace", _vp),
                ("workspace_bytes", ctypes.c_size_t), ("kv_type", _i32), ("k_scale", ctypes.c_float),
                ("v_scale", ctypes.c_float)]


class PrefillPagedParams(ctypes.Structure):
    _fields_ = [("q", _vp), ("q_sb", _i64), ("q_sh", _i64), ("q_ss", _i64), ("k_cache", _vp), ("v_cache", _vp),
                ("block_table", _vp), ("seq_lens", _vp), ("max_blocks_per_seq", _i32), ("B", _i32), ("Hq", _i32),
                ("Hkv", _i32), ("Sq", _i32), ("dk", _i32), ("dv", _i32), ("block_size", _i32), ("num_blocks", _i32),
                ("scale", ctypes.c_float), ("causal", _i32), ("o", _vp), ("o_sb", _i64), ("o_sh", _i64),
                ("o_ss", _i64), ("lse", _vp), ("o_dtype", _i32), ("q_lens", _vp), ("mask", _vp),
                ("m_sb", _i64), ("m_sh", _i64), ("m_ss", _i64), ("max_bias", ctypes.c_float),
                ("softcap", ctypes.c_float), ("sinks", _vp)]


class GatherParams(ctypes.Structure):
    _fields_ = [("q", _vp), ("kv_rows", _vp), ("n_rows", _i64), ("row_stride", _i64), ("dk", _i32), ("dv", _i32),
                ("v_offset", _i32), ("idx", _vp), ("topk", _i32), ("key_pos", _vp), ("q_pos", _vp), ("T", _i32),
                ("Hq", _i32), ("scale", ctypes.c_float), ("num_splits", _i32), ("o", _vp), ("lse", _vp),
                ("o_dtype", _i32), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


class MlaTailParams(ctypes.Structure):
    _fields_ = [("o_lat", _vp), ("w_abs", _vp), ("w_o", _vp), ("T", _i32), ("Hq", _i32), ("R", _i32), ("V", _i32),
                ("Hd", _i32), ("y", _vp), ("y_dtype", _i32), ("num_splits", _i32), ("workspace", _vp),
                ("workspace_bytes", ctypes.c_size_t)]


class KvDequantParams(ctypes.Structure):
    _fields_ = [("src", _vp), ("type", _i32), ("n_rows", _i64), ("row_elems", _i32), ("src_row_bytes", _i64),
                ("dst", _vp), ("dst_row_stride", _i64), ("scale", ctypes.c_float)]


FA_KV_Q8_0, FA_KV_Q4_0, FA_KV_FP8_E4M3 = 8, 4, 2
KV_QUANT = {"q8_0": (FA_KV_Q8_0, 34), "q4_0": (FA_KV_Q4_0, 18),
            "fp8_e4m3": (FA_KV_FP8_E4M3, 32)}  # type code, bytes per 32 values

_lib = None


def load():
    """Load libfa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libfa.so is not built (run python -m attention_attn_fwd_11_b200.build)")
        lib = ctypes.CDLL(LIB_PATH)
        lib.fa_fwd.argtypes = [ctypes.POINTER(FwdParams), _vp]
        lib.fa_fwd.restype = _i32
        lib.fa_prefill_paged.argtypes = [ctypes.POINTER(PrefillPagedParams), _vp]
        lib.fa_prefill_paged.restype = _i32
        lib.fa_decode_paged_workspace_size.argtypes = [ctypes.POINTER(PagedParams), ctypes.POINTER(ctypes.c_size_t)]
        lib.fa_decode_paged_workspace_size.restype = _i32
        lib.fa_decode_paged.argtypes = [ctypes.POINTER(PagedParams), _vp]
        lib.fa_decode_paged.restype = _i32
        lib.fa_decode_gather_workspace_size.argtypes = [ctypes.POINTER(GatherParams), ctypes.POINTER(ctypes.c_size_t)]
        lib.fa_decode_gather_workspace_size.restype = _i32
        lib.fa_decode_gather.argtypes = [ctypes.POINTER(GatherParams), _vp]
        lib.fa_decode_gather.restype = _i32
        lib.fa_mla_tail_workspace_size.argtypes = [ctypes.POINTER(MlaTailParams), ctypes.POINTER(ctypes.c_size_t)]
        lib.fa_mla_tail_workspace_size.restype = _i32
        lib.fa_mla_tail.argtypes = [ctypes.POINTER(MlaTailParams), _vp]
        lib.fa_mla_tail.restype = _i32
        lib.fa_kv_dequant.argtypes = [ctypes.POINTER(KvDequantParams), _vp]
        lib.fa_kv_dequant.restype = _i32
        lib.fa_kv_dequant_n.argtypes = [ctypes.POINTER(KvDequantParams), _i32, _vp]
        lib.fa_kv_dequant_n.restype = _i32
        lib.fa_last_error.argtypes = []
        lib.fa_last_error.restype = ctypes.c_char_p
        lib.fa_device_error.argtypes = [_i32, ctypes.POINTER(_i32)]
        lib.fa_device_error.restype = _i32
        lib.fa_version.restype = _i32
        _lib = lib
    return _lib


class FAError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__("%s: %s" % (STATUS_NAMES.get(status, status), msg))
        self.status = status


def _check(st):
    if st != FA_OK:
        raise FAError(st, load().fa_last_error().decode())


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return _vp(stream.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libfa works on CUDA tensors only (no CPU fallback)")


def _odt(dtype):
    if dtype == torch.float32:
        return FA_F32
    if dtype == torch.bfloat16:
        return FA_BF16
    raise ValueError("output dtype must be float32 or bfloat16")


# ------------------------------------------------------------------ prefill --

def fwd_params(q, k, v, o, lse, scale, causal, mask=None, max_bias=0.0, softcap=0.0, sinks=None):
    B, Hq, Sq, dk = q.shape
    _, Hkv, Sk, dv = v.shape
    p = FwdParams()
    p.q, p.k, p.v, p.o, p.lse = _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse)
    p.B, p.Hq, p.Hkv, p.Sq, p.Sk, p.dk, p.dv = B, Hq, Hkv, Sq, Sk, dk, dv
    p.q_sb, p.q_sh, p.q_ss = q.stride(0), q.stride(1), q.stride(2)
    p.k_sb, p.k_sh, p.k_ss = k.stride(0), k.stride(1), k.stride(2)
    p.v_sb, p.v_sh, p.v_ss = v.stride(0), v.stride(1), v.stride(2)
    p.o_sb, p.o_sh, p.o_ss = o.stride(0), o.stride(1), o.stride(2)
    p.scale = scale
    p.causal = 1 if causal else 0
    p.o_dtype = _odt(o.dtype)
    if mask is not None:  # [Bm, Hm, Sq, Sk] f16; a size-1 batch or head dim broadcasts
        p.mask = _ptr(mask)
        p.m_sb = 0 if mask.shape[0] == 1 else mask.stride(0)
        p.m_sh = 0 if mask.shape[1] == 1 else mask.stride(1)
        p.m_ss = mask.stride(2)
    p.max_bias = max_bias
    p.softcap = softcap
    p.sinks = _ptr(sinks)
    return p


def fwd(q, k, v, scale=None, causal=False, out=None, return_lse=True, out_dtype=torch.float32, stream=None,
        mask=None, max_bias=0.0, softcap=0.0, sinks=None, lse=None):
    """O = softmax(scale * Q K^T + mask) V.  q [B,Hq,Sq,dk], k [B,Hkv,Sk,dk],
    v [B,Hkv,Sk,dv] bf16 CUDA tensors (any strides, head dim contiguous).
    Score modifiers (see fa_fwd in include/fa.h): mask [1|B, 1|Hq, Sq, Sk]
    float16 CUDA tensor with a contiguous last dim, max_bias (ALiBi slopes
    applied to the mask), softcap, sinks [Hq] float32 CUDA tensor.  out and
    lse may be given preallocated (lse: contiguous float32 [B,Hq,Sq]).
    Returns (O [B,Hq,Sq,dv], LSE [B,Hq,Sq] fp32 or None)."""
    _need_cuda(q, k, v)
    if mask is not None:
        _need_cuda(mask)
        if mask.dtype != torch.float16 or mask.dim() != 4 or mask.stride(3) != 1:
            raise ValueError("mask must be a 4-D float16 tensor with a contiguous last dim")
    if sinks is not None:
        _need_cuda(sinks)
        if sinks.dtype != torch.float32 or sinks.shape != (q.shape[1],) or not sinks.is_contiguous():
            raise ValueError("sinks must be a contiguous float32 tensor of shape [Hq]")
    for t in (q, k, v):
        if t.dtype != torch.bfloat16 or t.dim() != 4 or t.stride(3) != 1:
            raise ValueError("q, k, v must be 4-D bf16 with a contiguous last dim")
    B, Hq, Sq, dk = q.shape
    dv = v.shape[3]
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    if out is None:
        out = torch.empty((B, Hq, Sq, dv), device=q.device, dtype=out_dtype)
    if lse is not None:
        if lse.dtype != torch.float32 or tuple(lse.shape) != (B, Hq, Sq) or not lse.is_contiguous() or not lse.is_cuda:
            raise ValueError("lse must be a contiguous float32 CUDA tensor [B, Hq, Sq]")
    elif return_lse:
        lse = torch.empty((B, Hq, Sq), device=q.device, dtype=torch.float32)
    params = fwd_params(q, k, v, out, lse, scale, causal, mask, max_bias, softcap, sinks)
    _check(load().fa_fwd(ctypes.byref(params), _stream(stream)))
    return out, lse


# ------------------------------------------------------------- paged decode --

def _paged_kv(q, v_cache, kv_type):
    """(cache type, dv) of a paged cache: bf16 rows, or uint8 rows of q8_0
    (34 bytes per 32 values), q4_0 (18) or fp8 e4m3 (32) -- told apart by
    the row length against dk when kv_type is not given."""
    if v_cache.dtype != torch.uint8:
        return None, v_cache.shape[3]
    if kv_type is None:
        dk, r = q.shape[-1], v_cache.shape[3]
        kv_type = {dk // 32 * 34: "q8_0", dk // 32 * 18: "q4_0", dk: "fp8_e4m3"}.get(r)
        if kv_type is None:
            raise ValueError("cannot tell the cache type from a row of %d bytes; pass kv_type" % r)
    return kv_type, v_cache.shape[3] // KV_QUANT[kv_type][1] * 32


def paged_params(q, k_cache, v_cache, block_table, seq_lens, o, lse, scale, num_splits, ws, kv_type=None,
                 k_scale=1.0, v_scale=1.0):
    B, Hq, dk = q.shape
    nb, Hkv, bs, _ = k_cache.shape
    p = PagedParams()
    p.q, p.k_cache, p.v_cache = _ptr(q), _ptr(k_cache), _ptr(v_cache)
    p.block_table, p.seq_lens = _ptr(block_table), _ptr(seq_lens)
    p.max_blocks_per_seq = block_table.shape[1]
    kv_type, dv = _paged_kv(q, v_cache, kv_type)
    if kv_type is not None:  # quantised rows, converted inside the kernel
        p.kv_type = KV_QUANT[kv_type][0]
        p.k_scale, p.v_scale = k_scale, v_scale
    p.B, p.Hq, p.Hkv, p.dk, p.dv, p.block_size, p.num_blocks = B, Hq, Hkv, dk, dv, bs, nb
    p.scale = scale
    p.num_splits = num_splits
    p.o, p.lse = _ptr(o), _ptr(lse)
    p.o_dtype = _odt(o.dtype) if o is not None else FA_F32
    p.workspace = _ptr(ws)
    p.workspace_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    return p


def paged_workspace_bytes(q, k_cache, v_cache, block_table, seq_lens, num_splits=0):
    p = paged_params(q, k_cache, v_cache, block_table, seq_lens, None, None, 1.0, num_splits, None)
    n = ctypes.c_size_t(0)
    _check(load().fa_decode_paged_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def decode_paged(q, k_cache, v_cache, block_table, seq_lens, scale=None, num_splits=0, out=None,
                 return_lse=True, out_dtype=torch.float32, workspace=None, stream=None, kv_type=None, k_scale=1.0,
                 v_scale=1.0):
    """Split-KV decode over a paged cache.  q [B,Hq,dk]; caches
    [num_blocks,Hkv,block_size,d] bf16, or uint8 [...,136] of q8_0 rows,
    [...,72] of q4_0 rows, or [...,128] of fp8 e4m3 bytes read as
    e4m3 * k_scale / v_scale (dequantised in the kernel); block_table int32
    [B,max_blocks]; seq_lens int32 [B].  Returns (O [B,Hq,dv], LSE [B,Hq] or
    None)."""
    _need_cuda(q, k_cache, v_cache, block_table, seq_lens)
    B, Hq, dk = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    kv_type, dv = _paged_kv(q, v_cache, kv_type)
    if out is None:
        out = torch.empty((B, Hq, dv), device=q.device, dtype=out_dtype)
    lse = torch.empty((B, Hq), device=q.device, dtype=torch.float32) if return_lse else None
    if workspace is None:
        n = paged_workspace_bytes(q, k_cache, v_cache, block_table, seq_lens, num_splits)
        workspace = torch.empty(max(n, 256), device=q.device, dtype=torch.uint8)
    p = paged_params(q, k_cache, v_cache, block_table, seq_lens, out, lse, scale, num_splits, workspace, kv_type,
                     k_scale, v_scale)
    _check(load().fa_decode_paged(ctypes.byref(p), _stream(stream)))
    return out, lse


# ----------------------------------------------------------- paged prefill --

def prefill_paged_params(q, k_cache, v_cache, block_table, seq_lens, o, lse, scale, causal, q_lens=None,
                         mask=None, max_bias=0.0, softcap=0.0, sinks=None):
    B, Hq, Sq, dk = q.shape
    nb, Hkv, bs, _ = k_cache.shape
    p = PrefillPagedParams()
    p.q, p.q_sb, p.q_sh, p.q_ss = _ptr(q), q.stride(0), q.stride(1), q.stride(2)
    p.k_cache, p.v_cache = _ptr(k_cache), _ptr(v_cache)
    p.block_table, p.seq_lens = _ptr(block_table), _ptr(seq_lens)
    p.max_blocks_per_seq = block_table.shape[1]
    p.B, p.Hq, p.Hkv, p.Sq, p.dk, p.dv = B, Hq, Hkv, Sq, dk, v_cache.shape[3]
    p.block_size, p.num_blocks = bs, nb
    p.scale, p.causal = scale, 1 if causal else 0
    p.o, p.o_sb, p.o_sh, p.o_ss = _ptr(o), o.stride(0), o.stride(1), o.stride(2)
    p.lse = _ptr(lse)
    p.o_dtype = _odt(o.dtype)
    p.q_lens = _ptr(q_lens)
    if mask is not None:
        p.mask = _ptr(mask)
        p.m_sb = mask.stride(0) if mask.shape[0] > 1 else 0
        p.m_sh = mask.stride(1) if mask.shape[1] > 1 else 0
        p.m_ss = mask.stride(2)
    p.max_bias, p.softcap, p.sinks = max_bias, softcap, _ptr(sinks)
    return p


def prefill_paged(q, k_cache, v_cache, block_table, seq_lens, scale=None, causal=True, out=None,
                  return_lse=True, out_dtype=torch.float32, stream=None, q_lens=None, mask=None, max_bias=0.0,
                  softcap=0.0, sinks=None):
    """Chunked prefill over a paged cache (fa_prefill_paged).  q [B,Hq,Sq,dk]
    bf16 (head dim contiguous); k_cache [num_blocks,Hkv,64,dk], v_cache
    [num_blocks,Hkv,64,dv] bf16 contiguous, (dk, dv) a pair fwd() takes; block_table int32 [B,max_blocks]; seq_lens int32 [B] (keys
    including the new ones); q_lens: None or int32 [B], new rows per
    sequence (rows past it come back as O = 0, LSE = -inf); mask [1|B, 1|Hq,
    Sq, >= max seq_len] float16 (last dim contiguous), max_bias, softcap,
    sinks [Hq] float32: the score modifiers of fwd().
    Returns (O [B,Hq,Sq,dv], LSE [B,Hq,Sq] or None)."""
    _need_cuda(mask, sinks)
    if mask is not None and (mask.dtype != torch.float16 or mask.dim() != 4 or mask.stride(3) != 1):
        raise ValueError("mask must be a 4-D float16 tensor with a contiguous last dim")
    if sinks is not None and (sinks.dtype != torch.float32 or not sinks.is_contiguous()):
        raise ValueError("sinks must be contiguous float32 [Hq]")
    _need_cuda(q, k_cache, v_cache, block_table, seq_lens, out, q_lens)
    if q_lens is not None and (q_lens.dtype != torch.int32 or not q_lens.is_contiguous()):
        raise ValueError("q_lens must be contiguous int32")
    for t in (q, k_cache, v_cache):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise ValueError("q and the caches must be bf16 with a contiguous head dimension")
    if not (k_cache.is_contiguous() and v_cache.is_contiguous()):
        raise ValueError("the caches must be contiguous")
    if block_table.dtype != torch.int32 or seq_lens.dtype != torch.int32 or not block_table.is_contiguous():
        raise ValueError("block_table and seq_lens must be contiguous int32")
    B, Hq, Sq, dk = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    if out is None:
        out = torch.empty((B, Hq, Sq, v_cache.shape[3]), device=q.device, dtype=out_dtype)
    lse = torch.empty((B, Hq, Sq), device=q.device, dtype=torch.float32) if return_lse else None
    p = prefill_paged_params(q, k_cache, v_cache, block_table, seq_lens, out, lse, scale, causal, q_lens, mask,
                             max_bias, softcap, sinks)
    _check(load().fa_prefill_paged(ctypes.byref(p), _stream(stream)))
    return out, lse


# ------------------------------------------------------------ gather decode --

def gather_params(q, rows, idx, key_pos, q_pos, o, lse, scale, num_splits, ws, dk=576, dv=512, v_offset=64,
                  topk=None):
    T, Hq, _ = q.shape
    p = GatherParams()
    p.q, p.kv_rows = _ptr(q), _ptr(rows)
    p.n_rows, p.row_stride = rows.shape[0], rows.stride(0)
    p.dk, p.dv, p.v_offset = dk, dv, v_offset
    p.idx, p.topk = _ptr(idx), (idx.shape[1] if idx is not None else int(topk))
    p.key_pos, p.q_pos = _ptr(key_pos), _ptr(q_pos)
    p.T, p.Hq = T, Hq
    p.scale = scale
    p.num_splits = num_splits
    p.o, p.lse = _ptr(o), _ptr(lse)
    p.o_dtype = _odt(o.dtype) if o is not None else FA_F32
    p.workspace = _ptr(ws)
    p.workspace_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    return p


def gather_workspace_bytes(q, rows, idx, num_splits=0, topk=None, dk=576):
    p = gather_params(q, rows, idx, None, None, None, None, 1.0, num_splits, None, topk=topk, dk=dk,
                      v_offset=64 if dk == 576 else 0)
    n = ctypes.c_size_t(0)
    _check(load().fa_decode_gather_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def decode_gather(q, rows, idx, key_pos=None, q_pos=None, scale=None, num_splits=0, out=None, return_lse=True,
                  out_dtype=torch.float32, workspace=None, stream=None, topk=None, dk=576):
    """Latent sparse decode.  q [T,Hq,576]; rows [n_rows, >=576] bf16 (row
    pitch = rows.stride(0)); idx int32 [T,topk] (-1 = empty), or None with
    ``topk`` given: every token reads rows 0 .. topk - 1; key_pos int32
    [T,topk] or None; q_pos int32 [T] or None.
    Returns (O [T,Hq,512], LSE [T,Hq] or None)."""
    _need_cuda(q, rows, idx, key_pos, q_pos)
    if rows.stride(1) != 1:
        raise ValueError("rows must have a contiguous last dim")
    T, Hq, dk = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(dk)
    if out is None:
        out = torch.empty((T, Hq, 512), device=q.device, dtype=out_dtype)
    lse = torch.empty((T, Hq), device=q.device, dtype=torch.float32) if return_lse else None
    if workspace is None:
        n = gather_workspace_bytes(q, rows, idx, num_splits, topk=topk, dk=dk)
        workspace = torch.empty(max(n, 256), device=q.device, dtype=torch.uint8)
    p = gather_params(q, rows, idx, key_pos, q_pos, out, lse, scale, num_splits, workspace, topk=topk,
                      dk=dk, v_offset=64 if dk == 576 else 0)
    _check(load().fa_decode_gather(ctypes.byref(p), _stream(stream)))
    return out, lse


def prefill_latent(q, rows, causal=True, scale=None, num_splits=0, out=None, return_lse=True,
                   out_dtype=torch.float32, workspace=None, stream=None, dk=576):
    """Prefill in latent space (MLA with the absorbed query): Sq new tokens,
    each with Hq = 128 heads, against the Sk latent rows [k_pe | kv_latent]
    of the sequence, rows 0 .. Sk - 1 of ``rows`` -- the (dk, dv) = (576,
    512) attention of the llama.cpp tensor path's head-size table, all heads
    sharing one latent row per key.  q [Sq, 128, 576]; with causal, new
    token t sits at position Sk - Sq + t.  dk=512: the (512, 512) pair, rows
    of 512 that are both key and value (q [Sq, 128, 512]).  Runs
    fa_decode_gather with contiguous rows (idx NULL).
    Returns (O [Sq, 128, 512], LSE [Sq, 128])."""
    _need_cuda(q, rows)
    Sq, Sk = q.shape[0], rows.shape[0]
    q_pos = None
    if causal:
        q_pos = torch.arange(Sk - Sq, Sk, device=q.device, dtype=torch.int32)
    return decode_gather(q, rows, None, q_pos=q_pos, scale=scale, num_splits=num_splits, out=out,
                         return_lse=return_lse, out_dtype=out_dtype, workspace=workspace, stream=stream, topk=Sk,
                         dk=dk)


def device_error(clear=True) -> int:
    """Device-side error word (FA_DEVERR_*); synchronises the device."""
    c = _i32(0)
    _check(load().fa_device_error(1 if clear else 0, ctypes.byref(c)))
    return c.value


# ------------------------------------------------------ quantised K/V rows --

def kv_dequant_params(src, qtype, row_elems, dst, kv_scale=1.0):
    """Marshal a fa_kv_dequant call: src uint8 [..., row_bytes] (rows of
    ggml blocks or fp8 bytes), dst bf16 [..., >= row_elems] with unit stride
    in the last dimension and the same leading shape, both contiguous over
    the rows; kv_scale: the fp8 tensor scale."""
    code, _ = KV_QUANT[qtype]
    p = KvDequantParams()
    p.src, p.type, p.row_elems, p.dst = _ptr(src), code, row_elems, _ptr(dst)
    p.scale = kv_scale
    p.n_rows = src.numel() // src.shape[-1] if src.dim() else 0
    p.src_row_bytes = src.stride(-2) if src.dim() > 1 else src.shape[-1]
    p.dst_row_stride = dst.stride(-2) if dst.dim() > 1 else dst.shape[-1]
    return p


def _dequant_entry(src, qtype, row_elems, out, kv_scale=1.0):
    _need_cuda(src, out)
    if src.dtype != torch.uint8:
        raise ValueError("src must be uint8 blocks")
    if src.stride(-1) != 1:
        raise ValueError("src rows must be contiguous")
    lead = src.shape[:-1]
    if out is None:
        out = torch.empty(lead + (row_elems,), device=src.device, dtype=torch.bfloat16)
    if out.dtype != torch.bfloat16 or out.shape[:-1] != lead or out.shape[-1] < row_elems or out.stride(-1) != 1:
        raise ValueError("out must be bf16 [..., >= row_elems] with the rows of src")
    s2, o2 = src.reshape(-1, src.shape[-1]), out.reshape(-1, out.shape[-1])
    if s2.data_ptr() != src.data_ptr() or o2.data_ptr() != out.data_ptr():
        raise ValueError("leading dimensions must collapse to one row stride")
    return kv_dequant_params(s2, qtype, row_elems, o2, kv_scale), out


def kv_dequant(src, qtype, row_elems, out=None, stream=None, kv_scale=1.0):
    """Quantised rows -> bf16 rows on the GPU (fa_kv_dequant).  src: uint8
    CUDA tensor [..., row_bytes] whose rows each hold row_elems values of
    ``qtype`` ('q8_0' or 'q4_0' ggml blocks, or 'fp8_e4m3' bytes read as
    e4m3 * kv_scale); the leading dimensions must collapse to one row index
    with a single stride.  Returns (or fills) a bf16 tensor [..., row_elems]."""
    p, out = _dequant_entry(src, qtype, row_elems, out, kv_scale)
    _check(load().fa_kv_dequant(ctypes.byref(p), _stream(stream)))
    return out


def kv_dequant_many(entries, stream=None):
    """Several conversions in one launch (fa_kv_dequant_n).  entries: list of
    (src, qtype, row_elems, out-or-None[, kv_scale]), 1 to 4 of them, one
    qtype.  Returns the list of outputs."""
    made = [_dequant_entry(*e) for e in entries]
    arr = (KvDequantParams * len(made))(*[m[0] for m in made])
    _check(load().fa_kv_dequant_n(arr, len(made), _stream(stream)))
    return [m[1] for m in made]


def fwd_quant(q, k_blocks, v_blocks, qtype, dk, dv, scale=None, causal=False, out=None, return_lse=True,
              out_dtype=torch.float32, k_buf=None, v_buf=None, stream=None, k_scale=1.0, v_scale=1.0, **mods):
    """Prefill over quantised K/V, the pages' way: dequantise K and V to bf16
    (one fa_kv_dequant_n launch for both) and run fa_fwd on them.  k_blocks /
    v_blocks: uint8 [B, Hkv, Sk, dk / 32 * block bytes] and [..., dv / 32 *
    block bytes]; k_buf / v_buf: optional bf16 [B, Hkv, Sk, dk / dv] buffers
    for the dequantised rows (allocated when absent); k_scale / v_scale: the
    fp8 tensor scales.  Other arguments as fwd()."""
    k, v = kv_dequant_many([(k_blocks, qtype, dk, k_buf, k_scale), (v_blocks, qtype, dv, v_buf, v_scale)],
                           stream=stream)
    return fwd(q, k, v, scale=scale, causal=causal, out=out, return_lse=return_lse, out_dtype=out_dtype,
               stream=stream, **mods)


# --------------------------------------------------------- MLA decode tail --

def mla_tail_params(o_lat, w_abs, w_o, y, num_splits=0, workspace=None):
    T, Hq, R = o_lat.shape
    p = MlaTailParams()
    p.o_lat, p.w_abs, p.w_o, p.y = _ptr(o_lat), _ptr(w_abs), _ptr(w_o), _ptr(y)
    p.T, p.Hq, p.R, p.V, p.Hd = T, Hq, R, w_abs.shape[1], w_o.shape[0]
    p.y_dtype = _odt(y.dtype)
    p.num_splits = num_splits
    p.workspace = _ptr(workspace)
    p.workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    return p


def mla_tail_workspace_bytes(o_lat, w_abs, w_o, num_splits=0):
    p = MlaTailParams()
    p.T, p.Hq, p.R = o_lat.shape
    p.V, p.Hd = w_abs.shape[1], w_o.shape[0]
    p.y_dtype, p.num_splits = FA_F32, num_splits
    n = ctypes.c_size_t(0)
    _check(load().fa_mla_tail_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def mla_tail(o_lat, w_abs, w_o, out=None, out_dtype=torch.float32, num_splits=0, workspace=None, stream=None):
    """MLA decode tail (fa_mla_tail): y [T, Hd] = o-projection of the
    per-head out-absorb of o_lat [T, Hq, R].  w_abs [Hq, V, R]; w_o
    [Hd, Hq*V] (row = output feature).  All bf16, contiguous."""
    _need_cuda(o_lat, w_abs, w_o, out, workspace)
    for t in (o_lat, w_abs, w_o):
        if t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("o_lat, w_abs and w_o must be contiguous bf16")
    T = o_lat.shape[0]
    if out is None:
        out = torch.empty((T, w_o.shape[0]), device=o_lat.device, dtype=out_dtype)
    if workspace is None:
        n = mla_tail_workspace_bytes(o_lat, w_abs, w_o, num_splits)
        workspace = torch.empty(max(n, 256), device=o_lat.device, dtype=torch.uint8)
    p = mla_tail_params(o_lat, w_abs, w_o, out, num_splits, workspace)
    _check(load().fa_mla_tail(ctypes.byref(p), _stream(stream)))
    return out
