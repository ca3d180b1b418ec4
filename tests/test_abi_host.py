"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/fa.h declares, and rejects bad arguments before any
CUDA call."""
import ctypes
import os
import re

import pytest

from attention_attn_fwd_11_b200 import fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(fa_[A-Za-z0-9_]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    lib = fa.load()
    names = declared_functions()
    assert "fa_fwd" in names and "fa_decode_paged" in names and "fa_decode_gather" in names
    for n in names:
        assert hasattr(lib, n), "libfa.so does not export " + n


def test_version():
    assert fa.load().fa_version() >= 100


def fwd_params(**kw):
    p = fa.FwdParams()
    base = dict(q=16, k=32, v=48, o=64, lse=0, B=1, Hq=2, Hkv=2, Sq=128, Sk=128, dk=128, dv=128,
                q_sb=2 * 128 * 128, q_sh=128 * 128, q_ss=128, k_sb=2 * 128 * 128, k_sh=128 * 128, k_ss=128,
                v_sb=2 * 128 * 128, v_sh=128 * 128, v_ss=128, o_sb=2 * 128 * 128, o_sh=128 * 128, o_ss=128,
                scale=0.088, causal=1, o_dtype=0)
    base.update(kw)
    for k_, v_ in base.items():
        setattr(p, k_, v_)
    return p


@pytest.mark.parametrize("kw,status", [
    (dict(dk=96, dv=96), fa.FA_ERR_UNSUPPORTED),
    (dict(dk=128, dv=64), fa.FA_ERR_UNSUPPORTED),
    (dict(Hq=3, Hkv=2), fa.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), fa.FA_ERR_INVALID_ARG),
    (dict(q=0), fa.FA_ERR_INVALID_ARG),
    (dict(k=8), fa.FA_ERR_INVALID_ARG),
    (dict(lse=2), fa.FA_ERR_INVALID_ARG),
    (dict(o_dtype=7), fa.FA_ERR_INVALID_ARG),
    (dict(o_ss=130), fa.FA_ERR_INVALID_ARG),
    (dict(Sq=-1), fa.FA_ERR_INVALID_ARG),
    # score modifiers
    (dict(softcap=-1.0), fa.FA_ERR_INVALID_ARG),
    (dict(softcap=float("inf")), fa.FA_ERR_INVALID_ARG),
    (dict(max_bias=-2.0), fa.FA_ERR_INVALID_ARG),
    (dict(mask=8, m_ss=128), fa.FA_ERR_INVALID_ARG),          # mask base not 16-byte aligned
    (dict(mask=16, m_ss=130), fa.FA_ERR_INVALID_ARG),         # row stride not a multiple of 8
    (dict(mask=16, m_ss=120), fa.FA_ERR_INVALID_ARG),         # row stride < Sk
    (dict(mask=16, m_ss=128, m_sh=4), fa.FA_ERR_INVALID_ARG),  # head stride not a multiple of 8
    (dict(sinks=2), fa.FA_ERR_INVALID_ARG),                   # sinks not 4-byte aligned
    # the dv = 512 pairs: separate K and V, no score modifiers
    (dict(dk=576, dv=256), fa.FA_ERR_UNSUPPORTED),
    (dict(dk=256, dv=512), fa.FA_ERR_UNSUPPORTED),
    (dict(dk=576, dv=512, o_ss=512, softcap=30.0), fa.FA_ERR_UNSUPPORTED),
    (dict(dk=512, dv=512, o_ss=512, mask=16, m_ss=128), fa.FA_ERR_UNSUPPORTED),
    (dict(dk=576, dv=512, o_ss=512, sinks=16), fa.FA_ERR_UNSUPPORTED),
    (dict(dk=576, dv=512, o_ss=512, max_bias=8.0), fa.FA_ERR_UNSUPPORTED),
    (dict(dk=576, dv=512, o_ss=510), fa.FA_ERR_INVALID_ARG),  # o rows shorter than dv
])
def test_fwd_rejects(kw, status):
    lib = fa.load()
    st = lib.fa_fwd(ctypes.byref(fwd_params(**kw)), None)
    assert st == status, lib.fa_last_error()
    assert lib.fa_last_error().decode().startswith("fa_fwd")


def test_fwd_accepts_the_dv512_pairs():
    # accepted by validation: with Sq == 0 nothing is launched
    lib = fa.load()
    for dk in (576, 512):
        assert lib.fa_fwd(ctypes.byref(fwd_params(dk=dk, dv=512, o_ss=512, Sq=0)), None) == fa.FA_OK


def test_fwd_null_params_and_noop():
    lib = fa.load()
    assert lib.fa_fwd(None, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_fwd(ctypes.byref(fwd_params(Sq=0)), None) == fa.FA_OK  # nothing to do, no launch
    assert lib.fa_fwd(ctypes.byref(fwd_params(B=0)), None) == fa.FA_OK


def paged_params(**kw):
    p = fa.PagedParams()
    base = dict(q=16, k_cache=32, v_cache=48, block_table=64, seq_lens=80, max_blocks_per_seq=128, B=64, Hq=32,
                Hkv=8, dk=128, dv=128, block_size=64, num_blocks=4608, scale=0.088, num_splits=0, o=96, lse=0,
                o_dtype=0, workspace=0, workspace_bytes=0)
    base.update(kw)
    for k_, v_ in base.items():
        setattr(p, k_, v_)
    return p


def test_paged_workspace_size_and_validation():
    import torch
    lib = fa.load()
    n = ctypes.c_size_t(0)
    st = lib.fa_decode_paged_workspace_size(ctypes.byref(paged_params()), ctypes.byref(n))
    if torch.cuda.is_available():
        # automatic splits: two CTAs an SM, six waves, splits of >= 8 blocks
        assert st == fa.FA_OK
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        splits = min(128, max(1, -(-sms * 2 * 6 // (64 * 8))), (128 + 7) // 8)
        rows = 64 * 32 * splits
        assert n.value == ((rows * 128 * 4 + 255) // 256) * 256 + ((rows * 4 + 255) // 256) * 256
    else:
        # the automatic split count is sized from the device's SM count
        assert st == fa.FA_ERR_CUDA
    assert lib.fa_decode_paged_workspace_size(ctypes.byref(paged_params(num_splits=5)), ctypes.byref(n)) == 0
    assert n.value == ((64 * 32 * 5 * 512 + 255) // 256) * 256 + ((64 * 32 * 5 * 4 + 255) // 256) * 256
    # the workspace check happens before any launch
    assert lib.fa_decode_paged(ctypes.byref(paged_params(num_splits=5)), None) == fa.FA_ERR_WORKSPACE
    assert lib.fa_decode_paged(ctypes.byref(paged_params(num_splits=5, workspace=256, workspace_bytes=10)),
                               None) == fa.FA_ERR_WORKSPACE
    assert lib.fa_decode_paged(ctypes.byref(paged_params(dk=64, dv=64)), None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_decode_paged(ctypes.byref(paged_params(block_size=16)), None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_decode_paged(ctypes.byref(paged_params(Hq=24, Hkv=8)), None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_decode_paged(ctypes.byref(paged_params(Hq=30, Hkv=8)), None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_decode_paged(ctypes.byref(paged_params(k_cache=40)), None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_decode_paged(ctypes.byref(paged_params(B=0)), None) == fa.FA_OK


@pytest.mark.parametrize("kv_type,status", [(0, 0), (8, 0), (4, 0), (2, 0), (5, None), (1, None)])
def test_paged_cache_types(kv_type, status):
    # bf16, q8_0, q4_0 and fp8 caches pass the shape check; other codes are unsupported
    n = ctypes.c_size_t(0)
    st = fa.load().fa_decode_paged_workspace_size(ctypes.byref(paged_params(kv_type=kv_type, num_splits=4)),
                                                  ctypes.byref(n))
    assert st == (fa.FA_OK if status == 0 else fa.FA_ERR_UNSUPPORTED)


def test_paged_kv_type_from_row_length():
    import torch
    q = torch.empty(2, 4, 128, dtype=torch.bfloat16)
    for width, name in ((136, "q8_0"), (72, "q4_0"), (128, "fp8_e4m3")):
        v = torch.empty(3, 2, 64, width, dtype=torch.uint8)
        assert fa._paged_kv(q, v, None) == (name, 128)
    assert fa._paged_kv(q, torch.empty(3, 2, 64, 128, dtype=torch.bfloat16), None) == (None, 128)
    with pytest.raises(ValueError):
        fa._paged_kv(q, torch.empty(3, 2, 64, 100, dtype=torch.uint8), None)


def gather_params(**kw):
    p = fa.GatherParams()
    base = dict(q=16, kv_rows=32, n_rows=65536, row_stride=576, dk=576, dv=512, v_offset=64, idx=48, topk=2048,
                key_pos=0, q_pos=64, T=32, Hq=128, scale=1 / 24, num_splits=2, o=80, lse=0, o_dtype=0,
                workspace=0, workspace_bytes=0)
    base.update(kw)
    for k_, v_ in base.items():
        setattr(p, k_, v_)
    return p


def test_gather_workspace_size_and_validation():
    import torch
    lib = fa.load()
    n = ctypes.c_size_t(0)
    assert lib.fa_decode_gather_workspace_size(ctypes.byref(gather_params()), ctypes.byref(n)) == fa.FA_OK
    assert n.value == ((32 * 128 * 2 * 512 * 4 + 255) // 256) * 256 + ((32 * 128 * 2 * 4 + 255) // 256) * 256
    st = lib.fa_decode_gather_workspace_size(ctypes.byref(gather_params(num_splits=0)), ctypes.byref(n))
    # automatic splits are sized from the current device's SM count
    assert st == (fa.FA_OK if torch.cuda.is_available() else fa.FA_ERR_CUDA)
    assert lib.fa_decode_gather(ctypes.byref(gather_params()), None) == fa.FA_ERR_WORKSPACE
    assert lib.fa_decode_gather(ctypes.byref(gather_params(dk=128)), None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_decode_gather(ctypes.byref(gather_params(Hq=64)), None) == fa.FA_ERR_UNSUPPORTED
    # 512-wide rows that are both key and value: accepted (then the missing workspace is reported)
    assert lib.fa_decode_gather(ctypes.byref(gather_params(dk=512, dv=512, v_offset=0, row_stride=512)),
                                None) == fa.FA_ERR_WORKSPACE
    assert lib.fa_decode_gather(ctypes.byref(gather_params(dk=512, dv=512, v_offset=64)), None) == fa.FA_ERR_UNSUPPORTED
    assert lib.fa_decode_gather(ctypes.byref(gather_params(dk=512, dv=512, v_offset=0, row_stride=504)),
                                None) == fa.FA_ERR_INVALID_ARG
    # idx NULL (contiguous rows): topk must not exceed n_rows
    assert lib.fa_decode_gather(ctypes.byref(gather_params(idx=0, topk=70000, workspace=256, workspace_bytes=1 << 40)),
                                None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_decode_gather(ctypes.byref(gather_params(row_stride=580)), None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_decode_gather(ctypes.byref(gather_params(idx=50)), None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_decode_gather(ctypes.byref(gather_params(T=0)), None) == fa.FA_OK


def prefill_paged_params(**kw):
    p = fa.PrefillPagedParams()
    base = dict(q=16, q_sb=16 * 32 * 512 * 128, q_sh=512 * 128, q_ss=128, k_cache=32, v_cache=48, block_table=64,
                seq_lens=80, max_blocks_per_seq=128, B=16, Hq=32, Hkv=8, Sq=512, dk=128, dv=128, block_size=64,
                num_blocks=4096, scale=0.088, causal=1, o=96, o_sb=16 * 32 * 512 * 128, o_sh=512 * 128, o_ss=128,
                lse=0, o_dtype=0)
    base.update(kw)
    for k_, v_ in base.items():
        setattr(p, k_, v_)
    return p


@pytest.mark.parametrize("kw,status", [
    (dict(dk=96, dv=96), fa.FA_ERR_UNSUPPORTED),
    (dict(dk=128, dv=64), fa.FA_ERR_UNSUPPORTED),
    (dict(dk=256, dv=128), fa.FA_ERR_UNSUPPORTED),
    (dict(block_size=16), fa.FA_ERR_UNSUPPORTED),
    (dict(Hq=30), fa.FA_ERR_INVALID_ARG),
    (dict(num_blocks=0), fa.FA_ERR_INVALID_ARG),
    (dict(max_blocks_per_seq=0), fa.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), fa.FA_ERR_INVALID_ARG),
    (dict(o_dtype=7), fa.FA_ERR_INVALID_ARG),
    (dict(k_cache=40), fa.FA_ERR_INVALID_ARG),             # not 16-byte aligned
    (dict(block_table=66), fa.FA_ERR_INVALID_ARG),         # not 4-byte aligned
    (dict(seq_lens=0), fa.FA_ERR_INVALID_ARG),
    (dict(o_ss=120), fa.FA_ERR_INVALID_ARG),               # o_ss < dv
    (dict(o_sh=6), fa.FA_ERR_INVALID_ARG),                 # fp32 strides must be multiples of 4
])
def test_prefill_paged_rejects(kw, status):
    assert fa.load().fa_prefill_paged(ctypes.byref(prefill_paged_params(**kw)), None) == status


@pytest.mark.parametrize("dk,dv", [(64, 64), (256, 256), (192, 128), (192, 192), (320, 256)])
def test_prefill_paged_accepts_every_prefill_pair(dk, dv):
    # validation passes; without a GPU the call then stops at the tensor-map
    # encoder (or the device), never with FA_ERR_UNSUPPORTED / INVALID_ARG.
    # The pointers are fake, so this must never reach a real launch.
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-only check: the fake pointers must not reach a GPU launch")
    st = fa.load().fa_prefill_paged(ctypes.byref(prefill_paged_params(
        dk=dk, dv=dv, q_sb=16 * 32 * 512 * dk, q_sh=512 * dk, q_ss=dk,
        o_sb=16 * 32 * 512 * dv, o_sh=512 * dv, o_ss=dv)), None)
    assert st not in (fa.FA_ERR_UNSUPPORTED, fa.FA_ERR_INVALID_ARG)


def test_prefill_paged_null_and_noop():
    lib = fa.load()
    assert lib.fa_prefill_paged(None, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_prefill_paged(ctypes.byref(prefill_paged_params(B=0)), None) == fa.FA_OK
    assert lib.fa_prefill_paged(ctypes.byref(prefill_paged_params(Sq=0)), None) == fa.FA_OK


def tail_params(**kw):
    p = fa.MlaTailParams()
    base = dict(o_lat=16, w_abs=32, w_o=48, T=32, Hq=128, R=512, V=128, Hd=7168, y=64, y_dtype=0, num_splits=0,
                workspace=0, workspace_bytes=0)
    base.update(kw)
    for k_, v_ in base.items():
        setattr(p, k_, v_)
    return p


def test_mla_tail_workspace_size_and_validation():
    lib = fa.load()
    n = ctypes.c_size_t(0)
    # the workspace holds u (32 x 16384 bf16) whatever the split count
    for ns in (0, 3, 200):
        assert lib.fa_mla_tail_workspace_size(ctypes.byref(tail_params(num_splits=ns)), ctypes.byref(n)) == fa.FA_OK
        assert n.value == 32 * 16384 * 2
    assert lib.fa_mla_tail(ctypes.byref(tail_params()), None) == fa.FA_ERR_WORKSPACE
    for kw in (dict(V=64), dict(R=500), dict(Hd=7000)):
        assert lib.fa_mla_tail(ctypes.byref(tail_params(**kw)), None) == fa.FA_ERR_UNSUPPORTED, kw
    for kw in (dict(T=-1), dict(Hq=0), dict(y_dtype=5), dict(num_splits=-2), dict(w_o=40)):
        st = lib.fa_mla_tail(ctypes.byref(tail_params(workspace=256, workspace_bytes=1 << 30, **kw)), None)
        assert st == fa.FA_ERR_INVALID_ARG, kw
    assert lib.fa_mla_tail(ctypes.byref(tail_params(T=0)), None) == fa.FA_OK
    assert lib.fa_mla_tail(None, None) == fa.FA_ERR_INVALID_ARG


def dequant_params(**kw):
    p = fa.KvDequantParams()
    base = dict(src=2, type=fa.FA_KV_Q8_0, n_rows=1024, row_elems=128, src_row_bytes=136, dst=16, dst_row_stride=128,
                scale=1.0)
    base.update(kw)
    for k_, v_ in base.items():
        setattr(p, k_, v_)
    return p


@pytest.mark.parametrize("kw,status", [
    (dict(type=5), fa.FA_ERR_UNSUPPORTED),
    (dict(row_elems=48), fa.FA_ERR_INVALID_ARG),             # not a multiple of 32
    (dict(row_elems=0), fa.FA_ERR_INVALID_ARG),
    (dict(n_rows=-1), fa.FA_ERR_INVALID_ARG),
    (dict(src_row_bytes=134), fa.FA_ERR_INVALID_ARG),        # shorter than 4 q8_0 blocks
    (dict(src_row_bytes=137), fa.FA_ERR_INVALID_ARG),        # odd pitch
    (dict(dst_row_stride=120), fa.FA_ERR_INVALID_ARG),       # < row_elems
    (dict(dst_row_stride=132), fa.FA_ERR_INVALID_ARG),       # not a multiple of 8
    (dict(src=3), fa.FA_ERR_INVALID_ARG),                    # src not 2-byte aligned
    (dict(dst=24), fa.FA_ERR_INVALID_ARG),                   # dst not 16-byte aligned
    (dict(src=0), fa.FA_ERR_INVALID_ARG),
    (dict(type=fa.FA_KV_Q4_0, src_row_bytes=70), fa.FA_ERR_INVALID_ARG),   # 4 q4_0 blocks need 72
    (dict(type=fa.FA_KV_FP8_E4M3, src_row_bytes=132, src=8), fa.FA_ERR_INVALID_ARG),  # fp8 pitch % 8
    (dict(type=fa.FA_KV_FP8_E4M3, src_row_bytes=136, src=4), fa.FA_ERR_INVALID_ARG),  # fp8 src % 8
    (dict(type=fa.FA_KV_FP8_E4M3, src_row_bytes=120, src=8), fa.FA_ERR_INVALID_ARG),  # < 128 bytes
    (dict(type=fa.FA_KV_FP8_E4M3, src_row_bytes=128, src=8, scale=float("inf")), fa.FA_ERR_INVALID_ARG),
])
def test_kv_dequant_rejects(kw, status):
    assert fa.load().fa_kv_dequant(ctypes.byref(dequant_params(**kw)), None) == status


def test_kv_dequant_n_checks_every_entry():
    lib = fa.load()
    two = (fa.KvDequantParams * 2)(dequant_params(), dequant_params(type=fa.FA_KV_Q4_0, src_row_bytes=72))
    assert lib.fa_kv_dequant_n(two, 2, None) == fa.FA_ERR_INVALID_ARG          # mixed types
    two = (fa.KvDequantParams * 2)(dequant_params(), dequant_params(dst=8))
    assert lib.fa_kv_dequant_n(two, 2, None) == fa.FA_ERR_INVALID_ARG          # second entry misaligned
    assert lib.fa_kv_dequant_n(two, 0, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_kv_dequant_n(two, 5, None) == fa.FA_ERR_INVALID_ARG
    empty = (fa.KvDequantParams * 2)(dequant_params(n_rows=0, src=0, dst=0), dequant_params(n_rows=0))
    assert lib.fa_kv_dequant_n(empty, 2, None) == fa.FA_OK


def test_kv_dequant_null_params_and_noop():
    lib = fa.load()
    assert lib.fa_kv_dequant(None, None) == fa.FA_ERR_INVALID_ARG
    assert lib.fa_kv_dequant(ctypes.byref(dequant_params(n_rows=0, src=0, dst=0)), None) == fa.FA_OK


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        fa.fwd(q, q, q)
