"""The C ABI without a GPU: the library loads, exports every function include/csa.h declares,
its structs match a C compiler's layout, and host-side validation rejects bad arguments
with a status (no launch happens on any of these paths)."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

import long_context_sparse_08_b200 as csa
from long_context_sparse_08_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(csa_\w+|hca_\w+)\s*\(", src,
                       flags=re.M)
    return sorted(set(names))


def test_every_declared_function_is_exported():
    names = declared_functions()
    assert len(names) >= 12
    L = ctypes.CDLL(csa.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(csa.EXPORTS)


def declared_parameter_counts():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*((?:csa|hca)_\w+)\s*\(([^)]*)\)\s*;",
                         src, flags=re.M):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header():
    counts = declared_parameter_counts()
    assert set(counts) == set(csa.EXPORTS)
    for name, n in counts.items():
        assert len(csa._SIGS[name]) == n, f"{name}: binding {len(csa._SIGS[name])} vs header {n}"


def test_status_strings_and_version():
    assert csa.status_string(0) == "CSA_OK"
    assert csa.status_string(3) == "CSA_ERR_WORKSPACE"
    assert "sm_100a" in csa.version()


def test_struct_layout_matches_the_c_compiler():
    prog = r'''
#include <stdio.h>
#include <stddef.h>
#include "csa.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(csa_params), sizeof(csa_forward_args),
         offsetof(csa_forward_args, idx_dtype), offsetof(csa_forward_args, N_cap),
         offsetof(csa_forward_args, out), offsetof(csa_params, n_win), sizeof(csa_paged_kv),
         offsetof(csa_paged_kv, page_table), offsetof(csa_paged_kv, max_pages));
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(prog)
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe])
        vals = [int(x) for x in subprocess.check_output([exe]).split()]
    A = csa.CsaForwardArgs
    K = csa.CsaPagedKv
    assert vals == [ctypes.sizeof(csa.CsaParams), ctypes.sizeof(A), A.idx_dtype.offset,
                    A.N_cap.offset, A.out.offset, csa.CsaParams.n_win.offset, ctypes.sizeof(K),
                    K.page_table.offset, K.max_pages.offset]


def _p(**kw):
    return csa.make_params(**kw)


FAKE = 0x10000  # an aligned non-NULL address; never dereferenced on these paths


def _call(name, *args):
    fn = getattr(csa.lib(), name)
    return fn(*args)


def test_validation_rejects_bad_params():
    L = csa.lib()
    cases = [
        dict(c=48), dict(c=0), dict(rope_dims=3), dict(rope_dims=1024), dict(m=0),
        dict(rms_eps=-1.0),
    ]
    for kw in cases:
        p = _p(**kw)
        s = L.csa_compress(ctypes.byref(p), 1, 1, 16, 0, 8, FAKE, FAKE, FAKE, FAKE, FAKE, None,
                           None, None, 1, FAKE, None)
        assert s == csa.CSA_ERR_INVALID_ARG, kw
        assert csa.last_error()
    s = L.csa_compress(None, 1, 1, 16, 0, 8, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1,
                       FAKE, None)
    assert s == csa.CSA_ERR_INVALID_ARG


def test_compress_argument_checks():
    L = csa.lib()
    p = _p()
    base = [ctypes.byref(p), 1, 1, 16, 0, 8, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, 1,
            FAKE, None]

    def with_(**kw):
        a = list(base)
        pos = {"n_tok": 3, "first": 4, "n_cap": 5, "Ca": 6, "bias": 10, "prev_Cb": 11,
               "out": 15, "io": 1, "finalize": 14}
        for k, v in kw.items():
            a[pos[k]] = v
        return L.csa_compress(*a)

    assert with_(n_tok=15) == csa.CSA_ERR_INVALID_ARG  # not a multiple of m
    assert with_(first=6) == csa.CSA_ERR_INVALID_ARG  # 6 + 4 > 8
    assert with_(Ca=None) == csa.CSA_ERR_INVALID_ARG
    assert with_(Ca=FAKE + 4) == csa.CSA_ERR_INVALID_ARG  # misaligned
    assert with_(prev_Cb=FAKE) == csa.CSA_ERR_INVALID_ARG  # prev_Cb without prev_Zb
    assert with_(io=2) == csa.CSA_ERR_INVALID_ARG  # fp8 is not a compression io type
    assert with_(finalize=2) == csa.CSA_ERR_INVALID_ARG
    assert with_(n_tok=0) == csa.CSA_OK  # empty chunk: nothing to do, nothing launched
    p2 = _p(overlap=0, m=16)
    a = list(base)
    a[0] = ctypes.byref(p2)
    assert L.csa_compress(*a) == csa.CSA_ERR_INVALID_ARG  # HCA takes no b-branch


def test_index_and_topk_checks():
    L = csa.lib()
    p = _p(topk=4096)
    s = L.csa_topk(ctypes.byref(p), 1, 1, 100, FAKE, FAKE, FAKE, None, 0, None)
    assert s == csa.CSA_ERR_INVALID_ARG
    p = _p()
    s = L.csa_index_scores(ctypes.byref(p), 7, 1, 1, 100, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                           FAKE, None)
    assert s == csa.CSA_ERR_INVALID_ARG  # unknown key format
    s = L.csa_index_scores(ctypes.byref(p), csa.CSA_MXFP4, 1, 1, 100, FAKE, None, FAKE, FAKE,
                           FAKE, FAKE, FAKE, None)
    assert s == csa.CSA_ERR_INVALID_ARG  # MXFP4 queries need their scales
    s = L.csa_index_scores(ctypes.byref(p), csa.CSA_BF16, 0, 1, 100, None, None, None, None,
                           None, None, None, None)
    assert s == csa.CSA_OK  # B = 0: nothing to do
    p = _p(d_idx=48)
    s = L.csa_index_scores(ctypes.byref(p), csa.CSA_BF16, 1, 1, 100, FAKE, None, FAKE, FAKE,
                           None, FAKE, FAKE, None)
    assert s == csa.CSA_ERR_INVALID_ARG


def test_workspace_checks():
    L = csa.lib()
    p = _p()
    need = csa.workspace_size(p, csa.CSA_WS_INDEX_TOPK, csa.CSA_BF16, 2, 3, 1000)
    assert need >= 2 * 3 * 1000 * 4
    s = L.csa_index_topk(ctypes.byref(p), csa.CSA_BF16, 2, 3, 1000, FAKE, None, FAKE, FAKE,
                         None, FAKE, FAKE, None, FAKE, need - 1, None)
    assert s == csa.CSA_ERR_WORKSPACE
    assert csa.workspace_size(p, 99, 0, 1, 1, 10) == 0


def test_attention_checks():
    L = csa.lib()
    p = _p(n_heads=24)  # > 16 and not a multiple of 16
    s = L.hca_dense_mqa(ctypes.byref(p), 1, 1, 1, FAKE, FAKE, FAKE, 10, FAKE, 128, FAKE, None,
                        None, FAKE, None, 0, None)
    assert s == csa.CSA_ERR_INVALID_ARG
    p = _p()
    s = L.hca_dense_mqa(ctypes.byref(p), 1, 1, 1, FAKE, FAKE, FAKE, 10, None, 0, None, None,
                        None, FAKE, None, 0, None)
    assert s == csa.CSA_ERR_INVALID_ARG  # n_win > 0 but no window rows
    s = L.csa_sparse_mqa(ctypes.byref(p), 1, 1, 1, FAKE, FAKE, FAKE, 10, None, FAKE, 128, FAKE,
                         None, None, FAKE, None, 0, None)
    assert s == csa.CSA_ERR_INVALID_ARG  # no index list
    p = _p(c=1024)
    s = L.hca_dense_mqa(ctypes.byref(p), 1, 1, 1, FAKE, FAKE, FAKE, 10, FAKE, 128, FAKE, None,
                        None, FAKE, None, 0, None)
    assert s == csa.CSA_ERR_UNSUPPORTED


def test_state_append_checks():
    L = csa.lib()
    p = _p()
    # p, io, B, pos, Ca, Cb, Za, Zb, win_row, bias, rms_w, finalize, state, win_ring, out_fmt,
    # pages, page_scales, n_pages, page_rows, page_table, max_pages, stream
    base = [ctypes.byref(p), 1, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, FAKE, FAKE,
            1, FAKE, None, 8, 32, FAKE, 4, None]

    def with_(**kw):
        a = list(base)
        pos = {"io": 1, "B": 2, "pos": 3, "Cb": 5, "win_row": 8, "finalize": 11, "state": 12,
               "win_ring": 13, "out": 14, "scales": 16, "n_pages": 17, "page_rows": 18,
               "table": 19, "max_pages": 20}
        for k, v in kw.items():
            a[pos[k]] = v
        return L.csa_state_append(*a)

    assert with_(io=csa.CSA_MXFP4) == csa.CSA_ERR_INVALID_ARG
    assert with_(B=-1) == csa.CSA_ERR_INVALID_ARG
    assert with_(finalize=3) == csa.CSA_ERR_INVALID_ARG
    assert with_(n_pages=0) == csa.CSA_ERR_INVALID_ARG
    assert with_(page_rows=0) == csa.CSA_ERR_INVALID_ARG
    assert with_(max_pages=0) == csa.CSA_ERR_INVALID_ARG
    assert with_(win_ring=None) == csa.CSA_ERR_INVALID_ARG  # window row without a ring
    assert with_(Cb=None) == csa.CSA_ERR_INVALID_ARG  # CSA needs its b-branch rows
    assert with_(pos=None) == csa.CSA_ERR_INVALID_ARG
    assert with_(state=FAKE + 8) == csa.CSA_ERR_INVALID_ARG  # misaligned
    assert with_(table=None) == csa.CSA_ERR_INVALID_ARG
    assert with_(B=0) == csa.CSA_OK  # nothing to append, nothing launched
    assert with_(out=csa.CSA_F32) == csa.CSA_ERR_INVALID_ARG  # neither io nor an indexer format
    assert with_(out=csa.CSA_FP8_E4M3_ROWSCALE) == csa.CSA_ERR_INVALID_ARG  # no scales
    assert with_(out=csa.CSA_MXFP4, scales=FAKE) == csa.CSA_ERR_INVALID_ARG  # c = 512
    keys = _p(c=128)
    a = list(base)
    a[0], a[14], a[16] = ctypes.byref(keys), csa.CSA_MXFP4, FAKE
    assert L.csa_state_append(*a) == csa.CSA_ERR_INVALID_ARG  # 32-row pages split a block
    a[18] = 128
    a[2] = 0
    assert L.csa_state_append(*a) == csa.CSA_OK
    norope = _p(rope_dims=0)
    a = list(base)
    a[0], a[14], a[16] = ctypes.byref(norope), csa.CSA_MIXED_FP8_BF16, FAKE
    assert L.csa_state_append(*a) == csa.CSA_ERR_INVALID_ARG  # mixed rows need RoPE dims
    for r in (8, 24, 40):  # the attention reads mixed rows in 16-byte pieces: r % 16 == 0
        odd = _p(rope_dims=r)
        a[0] = ctypes.byref(odd)
        a[2] = 0  # even with nothing to append, a pool no reader accepts is refused
        assert L.csa_state_append(*a) == csa.CSA_ERR_INVALID_ARG, r
    assert with_(out=csa.CSA_MIXED_FP8_BF16) == csa.CSA_ERR_INVALID_ARG  # no scales
    assert with_(out=csa.CSA_MIXED_FP8_BF16, scales=FAKE, B=0) == csa.CSA_OK
    hca = _p(overlap=0, m=128)
    a = list(base)
    a[0] = ctypes.byref(hca)
    assert L.csa_state_append(*a) == csa.CSA_ERR_INVALID_ARG  # HCA takes no b-branch rows
    nowin = _p(n_win=0)
    a = list(base)
    a[0] = ctypes.byref(nowin)
    assert L.csa_state_append(*a) == csa.CSA_ERR_INVALID_ARG  # a ring needs n_win >= 1


def test_mixed_kv_attention_checks():
    L = csa.lib()
    p = _p()
    # p, B, T, q, q_pos, kv_rows, kv_scale, N_cap, idx, win_kv, L_raw, win_pos0, sink, q_rms_w,
    # out, ws, ws_bytes, stream
    base = [ctypes.byref(p), 1, 1, FAKE, FAKE, FAKE, FAKE, 1024, FAKE, FAKE, 128, FAKE, None,
            None, FAKE, None, 0, None]

    def call(i=None, v=None, params=None):
        a = list(base)
        if i is not None:
            a[i] = v
        if params is not None:
            a[0] = ctypes.byref(params)
        return L.csa_sparse_mqa_mixed_kv(*a)

    assert call(6, None) == csa.CSA_ERR_INVALID_ARG   # cache rows without their scales
    assert call(8, None) == csa.CSA_ERR_INVALID_ARG   # no index list
    assert call(1, 0) == csa.CSA_OK                   # nothing to do
    assert call(params=_p(rope_dims=8)) == csa.CSA_ERR_UNSUPPORTED   # r not a multiple of 16
    assert call(params=_p(rope_dims=0)) == csa.CSA_ERR_UNSUPPORTED   # no bf16 part
    assert call(params=_p(n_heads=16)) == csa.CSA_ERR_UNSUPPORTED    # heads in groups of 64
    assert call(params=_p(c=256)) == csa.CSA_ERR_UNSUPPORTED
    h = [ctypes.byref(_p(m=128, overlap=0)), 1, 1, FAKE, FAKE, FAKE, None, 64, FAKE, 128, FAKE,
         None, None, FAKE, None, 0, None]
    assert L.hca_dense_mqa_mixed_kv(*h) == csa.CSA_ERR_INVALID_ARG  # no scales


def test_paged_attention_checks():
    L = csa.lib()
    p = _p()
    kv = csa.CsaPagedKv(csa.CSA_BF16, FAKE, None, FAKE, 64, 32, 16)

    def call(kvd, idx=FAKE, params=p):
        return L.csa_sparse_mqa_paged(ctypes.byref(params), 1, 1, FAKE, FAKE, ctypes.byref(kvd),
                                      idx, FAKE, 128, FAKE, None, None, FAKE, None, 0, None)

    assert L.csa_sparse_mqa_paged(ctypes.byref(p), 1, 1, FAKE, FAKE, None, FAKE, FAKE, 128, FAKE,
                                  None, None, FAKE, None, 0, None) == csa.CSA_ERR_INVALID_ARG
    assert call(csa.CsaPagedKv(csa.CSA_FP8_E4M3_ROWSCALE, FAKE, FAKE, FAKE, 64, 32, 16)) == \
        csa.CSA_ERR_INVALID_ARG  # not a cache format
    assert call(csa.CsaPagedKv(csa.CSA_BF16, FAKE, None, None, 64, 32, 16)) == \
        csa.CSA_ERR_INVALID_ARG  # no page table
    assert call(csa.CsaPagedKv(csa.CSA_BF16, FAKE, None, FAKE, 0, 32, 16)) == \
        csa.CSA_ERR_INVALID_ARG  # empty pool
    assert call(csa.CsaPagedKv(csa.CSA_MIXED_FP8_BF16, FAKE, None, FAKE, 64, 32, 16)) == \
        csa.CSA_ERR_INVALID_ARG  # mixed rows without scales
    assert call(kv, idx=None) == csa.CSA_ERR_INVALID_ARG
    assert call(kv, params=_p(n_heads=32)) == csa.CSA_ERR_UNSUPPORTED
    # the window ring: win_pos0 = NULL needs L_raw = n_win and one query per request
    ring = lambda B, T, L: L.csa_sparse_mqa_paged(  # noqa: E731
        ctypes.byref(p), B, T, FAKE, FAKE, ctypes.byref(kv), FAKE, FAKE, 64, None, None, None,
        FAKE, None, 0, None)
    assert ring(1, 1, L) == csa.CSA_ERR_INVALID_ARG  # L_raw 64 != n_win 128
    assert L.csa_sparse_mqa_paged(ctypes.byref(p), 1, 2, FAKE, FAKE, ctypes.byref(kv), FAKE,
                                  FAKE, 128, None, None, None, FAKE, None, 0,
                                  None) == csa.CSA_ERR_INVALID_ARG  # T = 2
    assert L.csa_sparse_mqa(ctypes.byref(p), 1, 1, 1, FAKE, FAKE, FAKE, 10, FAKE, FAKE, 128, None,
                            None, None, FAKE, None, 0, None) == csa.CSA_ERR_INVALID_ARG
    assert L.hca_dense_mqa_paged(ctypes.byref(_p(m=128, overlap=0)), 0, 1, None, None,
                                 ctypes.byref(kv), None, 0, None, None, None, None, None, 0,
                                 None) == csa.CSA_OK  # nothing to do


def test_paged_index_checks():
    L = csa.lib()
    p = _p(topk=512)

    def call(kv, bf16=0, qs=None):
        return L.csa_index_topk_paged(ctypes.byref(p), 2, 1, ctypes.byref(kv), FAKE, qs, FAKE,
                                      FAKE, bf16, FAKE, None, FAKE, 1 << 30, None)

    assert call(csa.CsaPagedKv(csa.CSA_FP8_E4M3_ROWSCALE, FAKE, FAKE, FAKE, 64, 32, 16)) == \
        csa.CSA_ERR_UNSUPPORTED  # 32-row pages split a 128-key tile
    assert call(csa.CsaPagedKv(csa.CSA_MIXED_FP8_BF16, FAKE, FAKE, FAKE, 64, 128, 4)) == \
        csa.CSA_ERR_INVALID_ARG  # not an indexer key format
    assert call(csa.CsaPagedKv(csa.CSA_BF16, FAKE, None, None, 64, 128, 4)) == \
        csa.CSA_ERR_INVALID_ARG  # no page table
    assert call(csa.CsaPagedKv(csa.CSA_FP8_E4M3_ROWSCALE, FAKE, None, FAKE, 64, 128, 4)) == \
        csa.CSA_ERR_INVALID_ARG  # FP8 keys without their scales
    assert call(csa.CsaPagedKv(csa.CSA_BF16, FAKE, None, FAKE, 64, 128, 4), bf16=2) == \
        csa.CSA_ERR_INVALID_ARG
    # MXFP4 keys: the queries' scales are required, other formats take none
    assert call(csa.CsaPagedKv(csa.CSA_MXFP4, FAKE, FAKE, FAKE, 64, 128, 4)) == \
        csa.CSA_ERR_INVALID_ARG  # MXFP4 queries without their scales
    assert call(csa.CsaPagedKv(csa.CSA_MXFP4, FAKE, None, FAKE, 64, 128, 4), qs=FAKE) == \
        csa.CSA_ERR_INVALID_ARG  # MXFP4 keys without their exponent blocks
    assert call(csa.CsaPagedKv(csa.CSA_MXFP4, FAKE, FAKE, FAKE, 64, 64, 8), qs=FAKE) == \
        csa.CSA_ERR_UNSUPPORTED  # 64-row pages split a 128-key scale block
    assert call(csa.CsaPagedKv(csa.CSA_BF16, FAKE, None, FAKE, 64, 128, 4), qs=FAKE) == \
        csa.CSA_ERR_INVALID_ARG  # bf16 queries carry no scales


def test_prefill_handover_checks():
    L = csa.lib()
    p = _p()
    pages = csa.CsaPagedKv(csa.CSA_BF16, FAKE, None, FAKE, 8, 32, 4)
    args = [ctypes.byref(p), csa.CSA_BF16, 1, 16, 0, FAKE, FAKE, FAKE, FAKE, FAKE, None, None,
            None, 1, ctypes.byref(pages), None]
    bad_fmt = csa.CsaPagedKv(csa.CSA_F32, FAKE, None, FAKE, 8, 32, 4)
    a = list(args)
    a[14] = ctypes.byref(bad_fmt)
    assert L.csa_compress_paged(*a) == csa.CSA_ERR_INVALID_ARG  # pages not in the io dtype
    small = csa.CsaPagedKv(csa.CSA_BF16, FAKE, None, FAKE, 8, 1, 1)
    a = list(args)
    a[14] = ctypes.byref(small)
    assert L.csa_compress_paged(*a) == csa.CSA_ERR_INVALID_ARG  # 4 entries past 1 page of 1 row
    a = list(args)
    a[14] = None
    assert L.csa_compress_paged(*a) == csa.CSA_ERR_INVALID_ARG
    r = [ctypes.byref(p), csa.CSA_BF16, 1, 0, 16, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None]
    assert L.csa_state_resume(*r) == csa.CSA_ERR_INVALID_ARG  # window rows without a ring
    r[1] = csa.CSA_FP8_E4M3_ROWSCALE
    assert L.csa_state_resume(*r) == csa.CSA_ERR_INVALID_ARG
    r = [ctypes.byref(p), csa.CSA_BF16, 1, -1, 16, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, None]
    assert L.csa_state_resume(*r) == csa.CSA_ERR_INVALID_ARG  # negative first token
    r[3], r[4] = 0, 0
    assert L.csa_state_resume(*r) == csa.CSA_OK  # an empty chunk: nothing to copy


def test_binding_refuses_host_tensors():
    import torch

    with pytest.raises(ValueError):
        csa._ptr(torch.zeros(4))


def test_noalloc_topk_rejects_oversize_on_the_host():
    # 64 rows of 65536 candidates need ~32 MB of lists: refused before any device work, so
    # this runs without a GPU (the pointers are never dereferenced)
    p = csa.make_params(topk=1024)
    need = csa.workspace_size(p, csa.CSA_WS_TOPK, 0, 64, 1, 65536)
    assert need > csa.TOPK_NOALLOC_SCRATCH_BYTES
    s = csa.lib().csa_topk_noalloc(ctypes.byref(p), 64, 1, 65536, 0x1000, 0x2000, 0x3000, None)
    assert s == csa.CSA_ERR_WORKSPACE
    assert "scratch" in csa.last_error()


def test_kernel_launch_counter_is_exported():
    assert csa.kernel_launches() >= 0


def test_a_c_program_drives_the_page_allocator():
    # the host-only calls of the C ABI, from C, linked against libcsa.so
    prog = r'''
#include <stdio.h>
#include "csa.h"
int main(void) {
  csa_page_alloc* a = NULL;
  if (csa_page_alloc_create(5, 2, 3, &a) != CSA_OK) return 1;
  if (csa_page_alloc_reserve(a, 0, csa_state_pages_needed(4, 32, 132)) != CSA_OK) return 2;
  if (csa_page_alloc_reserve(a, 1, 3) != CSA_OK) return 3;
  if (csa_page_alloc_reserve(a, 0, 3) != CSA_ERR_NO_PAGES) return 4;
  csa_page_alloc_release(a, 1);
  if (csa_page_alloc_reserve(a, 0, 3) != CSA_OK) return 5;
  const int32_t* t = csa_page_alloc_table(a);
  for (int i = 0; i < 6; ++i) printf("%d ", t[i]);
  printf("%d %s\n", csa_page_alloc_free_pages(a), csa_status_string(CSA_ERR_NO_PAGES));
  csa_page_alloc_destroy(a);
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(prog)
        libdir = os.path.dirname(csa.LIB_PATH)
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe,
                               "-L", libdir, "-lcsa", f"-Wl,-rpath,{libdir}"])
        out = subprocess.check_output([exe]).decode().split()
    # request 0: 132 tokens make 33 entries, 2 pages of 32 (0, 1); request 1: 3 pages (2, 3,
    # 4); request 0's third page fails with none free, then takes page 2 once request 1 gave
    # 2, 3, 4 back
    assert out == ["0", "1", "2", "-1", "-1", "-1", "2", "CSA_ERR_NO_PAGES"]
