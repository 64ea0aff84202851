"""The C ABI without a GPU: the library loads, exports every symbol include/fpx.h declares, and
its host-side validation and size queries behave as documented (no device work is launched)."""
import ctypes
import os
import re

import numpy as np
import pytest

import dynamic_block_sparse_pooled_b200 as fpx
from oracle import fpx_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fpx.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fpx_[a-z_0-9]+)\s*\(", src)))


def test_header_and_binding_agree():
    assert sorted(fpx.EXPORTS) == declared_functions()


def test_library_exports_every_declared_symbol():
    lib = fpx.load()
    for name in declared_functions():
        assert hasattr(lib, name), name


def make(seqlens=None, t=0, hq=4, hkv=2, d=128, block=128, dtype=fpx.BF16, scales=False):
    p = fpx.Problem()
    keep = []
    if seqlens is not None:
        cu = np.zeros(len(seqlens) + 1, np.int32)
        cu[1:] = np.cumsum(seqlens)
        keep.append(cu)
        p.num_seqs = len(seqlens)
        p.cu_seqlens_h = cu.ctypes.data
        p.cu_seqlens_d = 0x1000  # never dereferenced on the host
        t = int(cu[-1])
    else:
        p.num_seqs = 1
    p.total_tokens, p.hq, p.hkv, p.d, p.block, p.dtype = t, hq, hkv, d, block, dtype
    if scales:
        p.q_scale_d = p.k_scale_d = p.v_scale_d = 0x2000
    return p, keep


@pytest.mark.parametrize("seqlens,block", [([2048], 64), ([8192], 128), ([131072], 128),
                                           ([4096, 8192, 16384, 65536, 2048, 32768, 4096, 131072], 128),
                                           ([1000, 0, 129, 1], 128), ([77, 130], 32)])
def test_sizes_match_the_oracle_layout(seqlens, block):
    lib = fpx.load()
    p, keep = make(seqlens, block=block)
    cu = keep[0]
    nb = O.total_blocks(cu, block)
    tri = O.total_pairs(cu, block)
    ref = ctypes.byref(p)
    assert lib.fpx_num_blocks(ref) == nb
    assert lib.fpx_rows(ref) == 4 * nb
    assert lib.fpx_scores_elems(ref) == 4 * tri
    assert lib.fpx_max_nnz(ref) == 4 * tri
    ws = [lib.fpx_workspace_bytes(ref, w) for w in (0, 1, 2)]
    assert all(x > 0 for x in ws) and lib.fpx_workspace_bytes(ref, -1) == max(ws)
    assert ws[0] >= 4 * nb * (4 + 2) * 128  # pooled Q and K, fp32


def test_attention_path_choice():
    lib = fpx.load()
    assert lib.fpx_attention_path(ctypes.byref(make([1000])[0])) == 1
    assert lib.fpx_attention_path(ctypes.byref(make([1000], dtype=fpx.E4M3, scales=True)[0])) == 1
    assert lib.fpx_attention_path(ctypes.byref(make([1000], dtype=fpx.F32)[0])) == 0
    assert lib.fpx_attention_path(ctypes.byref(make([1000], block=64)[0])) == 0
    assert lib.fpx_attention_path(ctypes.byref(make([1000], d=64)[0])) == 0


BAD = {
    "hq_not_multiple": dict(hq=6, hkv=4),
    "bad_head_dim": dict(d=96),
    "block_not_pow2": dict(block=96),
    "block_too_large": dict(block=256),
    "e4m3_without_scales": dict(dtype=fpx.E4M3),
    "bad_dtype": dict(dtype=7),
}


@pytest.mark.parametrize("name", sorted(BAD))
def test_invalid_problems_are_rejected_on_the_host(name):
    lib = fpx.load()
    kw = BAD[name]
    p, keep = make([300], **kw)
    ref = ctypes.byref(p)
    assert lib.fpx_num_blocks(ref) == 0
    assert lib.fpx_workspace_bytes(ref, -1) == 0
    rc = lib.fpx_block_scores(ref, 0x10000, 0x10000, 0x10000, 0x10000, 1 << 30, None)
    assert rc in (-1, -2)


def test_csr_beyond_int32_is_rejected_and_just_below_is_accepted():
    """row_ptr / col_idx are int32: a problem whose worst-case CSR (Hq x TRI entries, alpha = 0)
    would not fit is refused on the host before any launch; one just inside fits."""
    lib = fpx.load()
    a, big = 0x100000, 1 << 40
    p, keep = make([2_000_000], hq=32, hkv=8)  # 32 x 15625*15626/2 = 3.9e9 entries
    ref = ctypes.byref(p)
    assert lib.fpx_num_blocks(ref) == 0
    assert lib.fpx_workspace_bytes(ref, -1) == 0
    assert lib.fpx_block_scores(ref, a, a, a, a, big, None) == -2
    p, keep = make([1_048_576], hq=32, hkv=8)  # 32 x 8192*8193/2 = 1.07e9 entries
    ref = ctypes.byref(p)
    assert lib.fpx_num_blocks(ref) == 8192
    assert lib.fpx_max_nnz(ref) == 32 * 8192 * 8193 // 2 < 2**31 - 1
    assert lib.fpx_workspace_bytes(ref, -1) > 0


def test_host_argument_errors():
    lib = fpx.load()
    p, keep = make([300])
    ref = ctypes.byref(p)
    big = 1 << 30
    a = 0x100000  # 256-aligned fake device address, never dereferenced on the host
    assert lib.fpx_block_scores(None, a, a, a, a, big, None) == -1
    assert lib.fpx_block_scores(ref, a, a, a, None, big, None) == -1            # no workspace
    assert lib.fpx_block_scores(ref, a, a, a, a + 16, big, None) == -3          # ws misaligned
    assert lib.fpx_block_scores(ref, a, a, a, a, 16, None) == -4                # ws too small
    assert lib.fpx_block_scores(ref, a + 2, a, a, a, big, None) == -3           # q misaligned
    assert lib.fpx_select(ref, a, float("nan"), 1, 1, a, a, 10, a, a, big, None) == -1
    assert lib.fpx_select(ref, a, -0.5, 1, 1, a, a, 10, a, a, big, None) == -1
    assert lib.fpx_select(ref, a, 0.1, -1, 1, a, a, 10, a, a, big, None) == -1
    assert lib.fpx_sparse_prefill(ref, a, a, a, a, a, a + 8, a, a, big, None) == -3  # o misaligned
    # cu_seqlens host mirror inconsistent with total_tokens
    p2, keep2 = make([300, 10])
    p2.total_tokens = 311
    assert lib.fpx_block_scores(ctypes.byref(p2), a, a, a, a, big, None) == -1
    # device cu_seqlens without its host mirror
    p3, _ = make([300])
    p3.cu_seqlens_h = None
    assert lib.fpx_block_scores(ctypes.byref(p3), a, a, a, a, big, None) == -1


def test_status_strings():
    lib = fpx.load()
    for code in range(-7, 1):
        assert lib.fpx_status_string(code)


def test_paged_argument_errors():
    lib = fpx.load()
    p, keep = make([300, 1000])  # nb_s = 3 and 8
    ref = ctypes.byref(p)
    big = 1 << 30
    a = 0x100000
    ok_kv = fpx.PagedKV(0x3000, 8, 64)
    assert lib.fpx_block_scores_paged(ref, a, a, None, a, a, big, None) == -1          # no table
    assert lib.fpx_block_scores_paged(ref, a, a, ctypes.byref(fpx.PagedKV(None, 8, 64)), a, a,
                                      big, None) == -1
    assert lib.fpx_block_scores_paged(ref, a, a, ctypes.byref(fpx.PagedKV(0x3000, 7, 64)), a, a,
                                      big, None) == -1                                  # < nb_max
    assert lib.fpx_block_scores_paged(ref, a, a, ctypes.byref(fpx.PagedKV(0x3000, 8, 0)), a, a,
                                      big, None) == -1                                  # no pages
    assert lib.fpx_block_scores_paged(ref, a, a, ctypes.byref(fpx.PagedKV(0x3002, 8, 64)), a, a,
                                      big, None) == -3                                  # misaligned
    assert lib.fpx_sparse_prefill_paged(ref, a, a, a, None, a, a, a, a, a, big, None) == -1
    # paged attention runs on the tensor-core path only
    pf, keep2 = make([300, 1000], dtype=fpx.F32)
    assert lib.fpx_sparse_prefill_paged(ctypes.byref(pf), a, a, a, ctypes.byref(ok_kv), a, a, a,
                                        a, a, big, None) == -2
    pd, keep3 = make([300, 1000], d=64)
    assert lib.fpx_sparse_prefill_paged(ctypes.byref(pd), a, a, a, ctypes.byref(ok_kv), a, a, a,
                                        a, a, big, None) == -2


def test_rescue_argument_errors():
    lib = fpx.load()
    p, keep = make([300])
    ref = ctypes.byref(p)
    big = 1 << 30
    a = 0x100000
    assert lib.fpx_block_scores_rescue(ref, a, a, None, a, None, a, a, big, None) == -1  # no qnorm
    assert lib.fpx_block_scores_rescue(ref, a, a, None, a, a + 2, a, a, big, None) == -3
    assert lib.fpx_select_rescue(ref, a, a, a, 0.1, float("nan"), 1, 1, a, a, 10, a, a, big,
                                 None) == -1
    assert lib.fpx_select_rescue(ref, a, a, a, 0.1, -1.0, 1, 1, a, a, 10, a, a, big, None) == -1
    assert lib.fpx_select_rescue(ref, a, None, a, 0.1, 0.2, 1, 1, a, a, 10, a, a, big, None) == -1
