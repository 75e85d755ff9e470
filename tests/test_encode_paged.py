"""Entries given as rows, stored into a page pool in a storage format (csa_encode_paged): the
prefill -> decode hand-over for pools kept quantised (MXFP4 indexer keys, FP8 keys, mixed
KV rows).

Expected bytes come from the input encoders (workloads.py) applied to the same values,
placed through the page table: e4m3 codes and amax/448 scales, MXFP4 codes with their
exponents in 128-row blocks, mixed rows (e4m3 + scale, bf16 RoPE values). Entries starting
mid-page and crossing pages; a page id outside the pool skips its entries (error 325) and
leaves their rows untouched.

The CPU tests run the kernel's arithmetic built for the host (tests/host_check); the device
test runs the library's kernel.
"""
import ctypes
import zlib

import numpy as np
import pytest

from long_context_sparse_08_b200 import workloads as W
import tests.test_state_append as SA

OUT_IO, OUT_FP8, OUT_MXFP4, OUT_MIXED = 0, 1, 2, 3
# (name, out format, c, page rows, n, first entry)
CASES = [("fp8_keys", OUT_FP8, 128, 128, 300, 50), ("mxfp4_keys", OUT_MXFP4, 128, 128, 300, 50),
         ("mixed_kv", OUT_MIXED, 512, 32, 70, 20), ("bf16_kv", OUT_IO, 512, 32, 70, 20)]
R = 64
B = 2


class Case:
    def __init__(self, name, out, c, page_rows, n, first, bad_page=False):
        self.name, self.out, self.c, self.page_rows, self.n, self.first = \
            name, out, c, page_rows, n, first
        g = np.random.default_rng(zlib.crc32(name.encode()))
        self.rows = W.f32_to_bf16_bits(g.standard_normal((B, n, c), np.float32) *
                                       g.uniform(0.1, 4.0, size=(B, n, 1)).astype(np.float32))
        self.max_pages = -(-(first + n) // page_rows)
        self.n_pages = B * self.max_pages + 2
        self.table = g.permutation(self.n_pages)[:B * self.max_pages].astype(np.int32) \
            .reshape(B, self.max_pages)
        if bad_page:
            self.table[1, self.max_pages - 1] = self.n_pages  # outside the pool
        rb = {OUT_IO: 2 * c, OUT_FP8: c, OUT_MXFP4: c // 2, OUT_MIXED: c + R}[out]
        self.pages = np.zeros((self.n_pages, page_rows, rb), np.uint8)
        sb = {OUT_IO: 0, OUT_FP8: 4, OUT_MXFP4: 4, OUT_MIXED: 4}[out]
        self.scales = np.zeros((self.n_pages, page_rows, max(sb, 1)), np.uint8)

    def expected(self):
        """(pages, scales) the encoders give, and which (b, i) are stored."""
        pages, scales = np.zeros_like(self.pages), np.zeros_like(self.scales)
        x = W.bf16_bits_to_f32(self.rows)
        stored = np.zeros((B, self.n), bool)
        for b in range(B):
            for i in range(self.n):
                e = self.first + i
                pg = self.table[b, e // self.page_rows]
                if not 0 <= pg < self.n_pages:
                    continue
                stored[b, i] = True
                slot = e % self.page_rows
                v = x[b, i]
                if self.out == OUT_IO:
                    pages[pg, slot] = self.rows[b, i].view(np.uint8)
                elif self.out == OUT_FP8:
                    codes, sc = W.quant_fp8_rowwise(v[None])
                    pages[pg, slot] = codes[0]
                    scales[pg, slot] = sc.view(np.uint8)
                elif self.out == OUT_MIXED:
                    codes, sc, rope = W.quant_mixed_kv(v[None], R)
                    pages[pg, slot] = np.concatenate([codes[0], rope[0].view(np.uint8)])
                    scales[pg, slot] = sc.view(np.uint8)
                else:
                    packed, ex = W.quant_mxfp4(v[None])
                    pages[pg, slot] = packed[0]
                    scales[pg, slot] = ex[0]  # key order; blocked below
        if self.out == OUT_MXFP4:
            for pg in range(self.n_pages):
                scales[pg] = W.block_key_scales(scales[pg])
        return pages, scales, stored


def _host(case: Case):
    L = SA.host_lib()
    L.encode_paged_host.restype = ctypes.c_int
    status = np.zeros((B, case.n), np.int32)
    p = SA._np_ptr
    rc = L.encode_paged_host(1, B, ctypes.c_int64(case.n), ctypes.c_int64(case.first), case.c, R,
                             case.out, case.n_pages, case.page_rows, case.max_pages,
                             p(case.rows), p(case.pages), ctypes.c_size_t(case.pages.nbytes),
                             p(case.scales), ctypes.c_size_t(case.scales.nbytes),
                             p(case.table), p(status))
    assert rc == 0, f"offset outside a buffer ({rc})"
    return case.pages, case.scales, status


@pytest.mark.parametrize("bad_page", [False, True], ids=["all_pages", "a_bad_page"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_host_build_matches_the_encoders(case, bad_page):
    cs = Case(*case, bad_page=bad_page)
    want_p, want_s, stored = cs.expected()
    pages, scales, status = _host(cs)
    assert np.array_equal(status == 1, stored)
    assert np.all(status[~stored] == -3)
    assert np.array_equal(pages, want_p), f"{case[0]}: page bytes"
    if case[1] != OUT_IO:
        assert np.array_equal(scales, want_s), f"{case[0]}: scales"


def test_checks_on_the_host():
    import long_context_sparse_08_b200 as csa

    L = csa.lib()
    F = 0x10000
    p = csa.make_params(c=128)
    call = lambda kv, n=10, first=0, io=csa.CSA_BF16, pp=p: L.csa_encode_paged(  # noqa: E731
        ctypes.byref(pp), io, 2, n, first, F, ctypes.byref(kv), None)
    kv = lambda fmt, rows=128, mp=2, sc=F, tb=F: csa.CsaPagedKv(fmt, F, sc, tb, 8, rows, mp)  # noqa
    assert call(kv(csa.CSA_MXFP4, rows=64, mp=4)) == csa.CSA_ERR_INVALID_ARG  # half a block
    assert call(kv(csa.CSA_MXFP4), io=csa.CSA_FP8_E4M3_ROWSCALE) == csa.CSA_ERR_INVALID_ARG
    assert call(kv(csa.CSA_FP8_E4M3_ROWSCALE), n=200, first=100) == csa.CSA_ERR_INVALID_ARG
    assert call(kv(csa.CSA_FP8_E4M3_ROWSCALE, sc=None)) == csa.CSA_ERR_INVALID_ARG
    assert call(kv(csa.CSA_FP8_E4M3_ROWSCALE, tb=None)) == csa.CSA_ERR_INVALID_ARG
    assert call(kv(csa.CSA_F32)) == csa.CSA_ERR_INVALID_ARG  # neither io nor a storage format
    assert call(kv(csa.CSA_MIXED_FP8_BF16), pp=csa.make_params(c=128, rope_dims=0)) == \
        csa.CSA_ERR_INVALID_ARG
    for r in (8, 24, 40):  # mixed rows as the attention reads them: rope_dims % 16 == 0
        assert call(kv(csa.CSA_MIXED_FP8_BF16), pp=csa.make_params(c=128, rope_dims=r)) == \
            csa.CSA_ERR_INVALID_ARG, r
    assert call(kv(csa.CSA_MIXED_FP8_BF16), n=0, pp=csa.make_params(c=128, rope_dims=32)) == \
        csa.CSA_OK
    p512 = csa.make_params(c=512)
    assert L.csa_encode_paged(ctypes.byref(p512), csa.CSA_BF16, 2, 10, 0, F,
                              ctypes.byref(kv(csa.CSA_MXFP4)), None) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_encode_paged(ctypes.byref(p), csa.CSA_BF16, 2, 10, 0, F, None, None) == \
        csa.CSA_ERR_INVALID_ARG
    assert call(kv(csa.CSA_MXFP4), n=0) == csa.CSA_OK  # nothing to store


@pytest.mark.gpu
@pytest.mark.parametrize("bad_page", [False, True], ids=["all_pages", "a_bad_page"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gpu_matches_the_encoders(case, bad_page):
    import torch
    import long_context_sparse_08_b200 as csa

    cs = Case(*case, bad_page=bad_page)
    want_p, want_s, stored = cs.expected()
    fmt = {OUT_IO: csa.CSA_BF16, OUT_FP8: csa.CSA_FP8_E4M3_ROWSCALE, OUT_MXFP4: csa.CSA_MXFP4,
           OUT_MIXED: csa.CSA_MIXED_FP8_BF16}[cs.out]
    p = csa.make_params(c=cs.c, rope_dims=R)
    pages = torch.zeros(cs.pages.shape, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(cs.scales.shape, dtype=torch.uint8, device="cuda")
    table = torch.from_numpy(cs.table).cuda()
    rows = torch.from_numpy(cs.rows.view(np.int16)).cuda()
    kv = csa.paged_kv(fmt, pages, None if cs.out == OUT_IO else scales, table, cs.n_pages,
                      cs.page_rows, cs.max_pages)
    torch.cuda.synchronize()
    csa.device_error()
    csa.csa_encode_paged(p, csa.CSA_BF16, B, cs.n, cs.first, rows, kv)
    torch.cuda.synchronize()
    assert csa.device_error() == (325 if bad_page else 0)
    assert np.array_equal(pages.cpu().numpy(), want_p), f"{case[0]}: page bytes"
    if cs.out != OUT_IO:
        assert np.array_equal(scales.cpu().numpy(), want_s), f"{case[0]}: scales"
