"""Python binding of libcsa, the CUDA (sm_100a) library of the CSA / HCA attention hot path.

Argument marshalling only: every call forwards torch CUDA tensors (their data pointers)
and the current CUDA stream to the C ABI of include/csa.h under the same name. All
compute runs in the library's kernels; there is no other code path. The library is
loaded on first use and a missing or unloadable ``libcsa.so`` raises at that point.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcsa.so")

(CSA_OK, CSA_ERR_INVALID_ARG, CSA_ERR_UNSUPPORTED, CSA_ERR_WORKSPACE, CSA_ERR_CUDA,
 CSA_ERR_NO_PAGES) = range(6)
CSA_F32, CSA_BF16, CSA_FP8_E4M3_ROWSCALE, CSA_MXFP4, CSA_MIXED_FP8_BF16 = range(5)
DTYPES = {"f32": CSA_F32, "bf16": CSA_BF16, "fp8": CSA_FP8_E4M3_ROWSCALE, "mxfp4": CSA_MXFP4}
(CSA_WS_INDEX_TOPK, CSA_WS_TOPK, CSA_WS_SPARSE_MQA, CSA_WS_HCA_MQA, CSA_WS_FORWARD,
 CSA_WS_INDEX_TOPK_BF16) = range(1, 7)

EXPORTS = (
    "csa_compress", "csa_index_scores", "csa_topk", "csa_index_topk", "csa_sparse_mqa",
    "hca_dense_mqa", "csa_forward", "csa_workspace_size", "csa_status_string",
    "csa_last_error", "csa_set_index_timing_events", "csa_version", "csa_device_error",
    "csa_topk_noalloc", "csa_kernel_launches", "csa_state_append", "csa_sparse_mqa_mixed_kv",
    "hca_dense_mqa_mixed_kv", "csa_grouped_out_proj", "csa_grouped_out_proj_workspace_size",
    "csa_sparse_mqa_paged", "hca_dense_mqa_paged", "csa_index_topk_bf16",
    "csa_index_topk_paged", "csa_forward_paged", "csa_compress_paged", "csa_state_resume",
    "csa_page_alloc_create", "csa_page_alloc_destroy", "csa_page_alloc_reserve",
    "csa_page_alloc_release", "csa_page_alloc_table", "csa_page_alloc_free_pages",
    "csa_page_alloc_mapped", "csa_state_pages_needed", "csa_encode_paged",
)
# size of the library-owned scratch array behind csa_topk_noalloc (bytes, per device)
TOPK_NOALLOC_SCRATCH_BYTES = 16 << 20


class CsaParams(ctypes.Structure):
    """Mirror of ``csa_params``."""

    _fields_ = [
        ("m", ctypes.c_int32), ("overlap", ctypes.c_int32), ("c", ctypes.c_int32),
        ("rope_dims", ctypes.c_int32), ("rope_base", ctypes.c_float),
        ("rms_eps", ctypes.c_float), ("sm_scale", ctypes.c_float),
        ("n_heads", ctypes.c_int32), ("n_idx_heads", ctypes.c_int32),
        ("d_idx", ctypes.c_int32), ("topk", ctypes.c_int32), ("n_win", ctypes.c_int32),
    ]


class CsaForwardArgs(ctypes.Structure):
    """Mirror of ``csa_forward_args``."""

    _fields_ = [
        ("n_tok", ctypes.c_int64), ("first_entry", ctypes.c_int64),
        ("Ca", ctypes.c_void_p), ("Cb", ctypes.c_void_p), ("Za", ctypes.c_void_p),
        ("Zb", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("prev_Cb", ctypes.c_void_p),
        ("prev_Zb", ctypes.c_void_p), ("kv_rms_w", ctypes.c_void_p),
        ("idx_dtype", ctypes.c_int), ("qI", ctypes.c_void_p), ("qI_scale", ctypes.c_void_p),
        ("w", ctypes.c_void_p), ("KI", ctypes.c_void_p), ("KI_scale", ctypes.c_void_p),
        ("q", ctypes.c_void_p), ("q_rms_w", ctypes.c_void_p), ("q_pos", ctypes.c_void_p),
        ("kv_cache", ctypes.c_void_p), ("N_cap", ctypes.c_int64),
        ("win_kv", ctypes.c_void_p), ("L_raw", ctypes.c_int64), ("win_pos0", ctypes.c_void_p),
        ("sink", ctypes.c_void_p), ("out_idx", ctypes.c_void_p),
        ("out_scores", ctypes.c_void_p), ("out", ctypes.c_void_p),
    ]


class CsaPagedKv(ctypes.Structure):
    """Mirror of ``csa_paged_kv``."""

    _fields_ = [
        ("fmt", ctypes.c_int), ("pages", ctypes.c_void_p), ("scales", ctypes.c_void_p),
        ("page_table", ctypes.c_void_p), ("n_pages", ctypes.c_int32),
        ("page_rows", ctypes.c_int32), ("max_pages", ctypes.c_int32),
    ]


_LIB = None
_VP, _I32, _I64, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_PP = ctypes.POINTER(CsaParams)
_SIGS = {
    "csa_compress": [_PP, ctypes.c_int, _I32, _I64, _I64, _I64] + [_VP] * 8 + [_I32, _VP, _VP],
    "csa_index_scores": [_PP, ctypes.c_int, _I32, _I32, _I64] + [_VP] * 7 + [_VP],
    "csa_topk": [_PP, _I32, _I32, _I64, _VP, _VP, _VP, _VP, _SZ, _VP],
    "csa_topk_noalloc": [_PP, _I32, _I32, _I64, _VP, _VP, _VP, _VP],
    "csa_index_topk": [_PP, ctypes.c_int, _I32, _I32, _I64] + [_VP] * 9 + [_SZ, _VP],
    "csa_sparse_mqa": [_PP, ctypes.c_int, _I32, _I32, _VP, _VP, _VP, _I64, _VP, _VP, _I64,
                       _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "hca_dense_mqa": [_PP, ctypes.c_int, _I32, _I32, _VP, _VP, _VP, _I64, _VP, _I64, _VP,
                      _VP, _VP, _VP, _VP, _SZ, _VP],
    "csa_forward": [_PP, ctypes.c_int, _I32, _I32, ctypes.POINTER(CsaForwardArgs), _VP, _SZ,
                    _VP],
    "csa_workspace_size": [_PP, _I32, ctypes.c_int, _I32, _I32, _I64],
    "csa_status_string": [ctypes.c_int],
    "csa_last_error": [],
    "csa_set_index_timing_events": [ctypes.POINTER(_VP), ctypes.POINTER(_VP), _I32],
    "csa_version": [],
    "csa_device_error": [ctypes.POINTER(ctypes.c_int32)],
    "csa_kernel_launches": [],
    "csa_sparse_mqa_paged": [_PP, _I32, _I32, _VP, _VP, ctypes.POINTER(CsaPagedKv), _VP, _VP,
                             _I64, _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "hca_dense_mqa_paged": [_PP, _I32, _I32, _VP, _VP, ctypes.POINTER(CsaPagedKv), _VP, _I64,
                            _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "csa_index_topk_bf16": [_PP, ctypes.c_int, _I32, _I32, _I64] + [_VP] * 9 + [_SZ, _VP],
    "csa_index_topk_paged": [_PP, _I32, _I32, ctypes.POINTER(CsaPagedKv), _VP, _VP, _VP, _VP,
                             _I32, _VP, _VP, _VP, _SZ, _VP],
    "csa_forward_paged": [_PP, _I32, _I32, ctypes.POINTER(CsaPagedKv), ctypes.POINTER(CsaPagedKv),
                          _I32] + [_VP] * 6 + [_VP, _I64] + [_VP] * 6 + [_SZ, _VP],
    "csa_compress_paged": [_PP, ctypes.c_int, _I32, _I64, _I64] + [_VP] * 8 +
                          [_I32, ctypes.POINTER(CsaPagedKv), _VP],
    "csa_state_resume": [_PP, ctypes.c_int, _I32, _I64, _I64] + [_VP] * 8,
    "csa_grouped_out_proj": [_PP, _I32, _I32, _I32, _I32, _VP, _VP, _VP, _VP, _VP, _SZ, _VP],
    "csa_grouped_out_proj_workspace_size": [_PP, _I32, _I32, _I32, _I32],
    "csa_sparse_mqa_mixed_kv": [_PP, _I32, _I32, _VP, _VP, _VP, _VP, _I64, _VP, _VP, _I64, _VP,
                                _VP, _VP, _VP, _VP, _SZ, _VP],
    "hca_dense_mqa_mixed_kv": [_PP, _I32, _I32, _VP, _VP, _VP, _VP, _I64, _VP, _I64, _VP, _VP,
                               _VP, _VP, _VP, _SZ, _VP],
    "csa_state_append": [_PP, ctypes.c_int, _I32] + [_VP] * 8 + [_I32, _VP, _VP, ctypes.c_int,
                                                             _VP, _VP, _I32, _I32, _VP, _I32, _VP],
    "csa_page_alloc_create": [_I32, _I32, _I32, ctypes.POINTER(_VP)],
    "csa_page_alloc_destroy": [_VP],
    "csa_page_alloc_reserve": [_VP, _I32, _I32],
    "csa_page_alloc_release": [_VP, _I32],
    "csa_page_alloc_table": [_VP],
    "csa_page_alloc_free_pages": [_VP],
    "csa_page_alloc_mapped": [_VP, _I32],
    "csa_state_pages_needed": [_I32, _I32, _I64],
    "csa_encode_paged": [_PP, ctypes.c_int, _I32, _I64, _I64, _VP, ctypes.POINTER(CsaPagedKv),
                         _VP],
}
_RES = {"csa_workspace_size": _SZ, "csa_grouped_out_proj_workspace_size": _SZ, "csa_kernel_launches": ctypes.c_uint64, "csa_status_string": ctypes.c_char_p,
        "csa_last_error": ctypes.c_char_p, "csa_version": ctypes.c_char_p,
        "csa_set_index_timing_events": None, "csa_page_alloc_destroy": None,
        "csa_page_alloc_table": ctypes.POINTER(ctypes.c_int32),
        "csa_page_alloc_free_pages": ctypes.c_int32, "csa_page_alloc_mapped": ctypes.c_int32,
        "csa_state_pages_needed": ctypes.c_int32}


class CsaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {status_string(status)}: {msg}")
        self.status = status


def lib():
    """The loaded libcsa (ctypes.CDLL); raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m long_context_sparse_08_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = _RES.get(name, ctypes.c_int)
        _LIB = L
    return _LIB


def status_string(s: int) -> str:
    return lib().csa_status_string(int(s)).decode()


def last_error() -> str:
    return lib().csa_last_error().decode()


def kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib().csa_kernel_launches())


def version() -> str:
    return lib().csa_version().decode()


def device_error() -> int:
    """Read and clear the library's device error word (0 = no bounded wait ran out and no
    state append was skipped)."""
    c = ctypes.c_int32(0)
    _check("csa_device_error", lib().csa_device_error(ctypes.byref(c)))
    return int(c.value)


def _check(fn: str, status: int):
    if status != CSA_OK:
        raise CsaError(fn, status, last_error())


def state_pages_needed(m: int, page_rows: int, n_tok: int) -> int:
    """Logical pages that hold the entries of a request's first n_tok tokens."""
    return int(lib().csa_state_pages_needed(m, page_rows, n_tok))


class PageAlloc:
    """A csa_page_alloc: physical pages of one pool handed to B requests' page tables (host
    memory; copy ``table`` to the device before the launches that read it)."""

    def __init__(self, n_pages: int, B: int, max_pages: int):
        h = _VP()
        _check("csa_page_alloc_create",
               lib().csa_page_alloc_create(n_pages, B, max_pages, ctypes.byref(h)))
        self._h, self.B, self.max_pages = h, B, max_pages

    def close(self):
        if self._h:
            lib().csa_page_alloc_destroy(self._h)
            self._h = _VP()

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown
            pass

    def reserve(self, b: int, n_logical: int) -> None:
        _check("csa_page_alloc_reserve", lib().csa_page_alloc_reserve(self._h, b, n_logical))

    def release(self, b: int) -> None:
        _check("csa_page_alloc_release", lib().csa_page_alloc_release(self._h, b))

    @property
    def table(self):
        """The host page table as a numpy int32 [B, max_pages] view (no copy)."""
        import numpy as np

        ptr = lib().csa_page_alloc_table(self._h)
        return np.ctypeslib.as_array(ptr, shape=(self.B, self.max_pages))

    @property
    def free_pages(self) -> int:
        return int(lib().csa_page_alloc_free_pages(self._h))

    def mapped(self, b: int) -> int:
        return int(lib().csa_page_alloc_mapped(self._h, b))


def _ptr(t) -> Optional[int]:
    """Device address of a CUDA tensor (None -> NULL). Host tensors are refused."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("libcsa takes CUDA tensors (device memory) only")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch

    return torch.cuda.current_stream().cuda_stream


def make_params(m=4, overlap=1, c=512, rope_dims=64, rope_base=10000.0, rms_eps=1e-6,
                sm_scale=0.0, n_heads=64, n_idx_heads=64, d_idx=128, topk=512,
                n_win=128) -> CsaParams:
    return CsaParams(m, overlap, c, rope_dims, rope_base, rms_eps, sm_scale, n_heads,
                     n_idx_heads, d_idx, topk, n_win)


def workspace_size(p: CsaParams, entry: int, kdt: int, B: int, T: int, N_cap: int) -> int:
    return int(lib().csa_workspace_size(ctypes.byref(p), entry, kdt, B, T, N_cap))


def csa_compress(p, io, B, n_tok, first_entry, n_cap, Ca, Cb, Za, Zb, bias, prev_Cb, prev_Zb,
                 kv_rms_w, finalize, out_cache, stream=None):
    s = lib().csa_compress(ctypes.byref(p), io, B, n_tok, first_entry, n_cap, _ptr(Ca),
                           _ptr(Cb), _ptr(Za), _ptr(Zb), _ptr(bias), _ptr(prev_Cb),
                           _ptr(prev_Zb), _ptr(kv_rms_w), int(finalize), _ptr(out_cache),
                           _stream(stream))
    _check("csa_compress", s)


def csa_state_append(p, io, B, pos, Ca, Cb, Za, Zb, win_row, bias, kv_rms_w, finalize, state,
                     win_ring, out_fmt, pages, page_scales, n_pages, page_rows, page_table,
                     max_pages, stream=None):
    s = lib().csa_state_append(ctypes.byref(p), io, B, _ptr(pos), _ptr(Ca), _ptr(Cb), _ptr(Za),
                               _ptr(Zb), _ptr(win_row), _ptr(bias), _ptr(kv_rms_w),
                               int(finalize), _ptr(state), _ptr(win_ring), int(out_fmt),
                               _ptr(pages), _ptr(page_scales), n_pages, page_rows,
                               _ptr(page_table), max_pages, _stream(stream))
    _check("csa_state_append", s)


def csa_index_scores(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos, out_scores,
                     stream=None):
    s = lib().csa_index_scores(ctypes.byref(p), kdt, B, T, N_cap, _ptr(qI), _ptr(qI_scale),
                               _ptr(w), _ptr(KI), _ptr(KI_scale), _ptr(q_pos),
                               _ptr(out_scores), _stream(stream))
    _check("csa_index_scores", s)


def csa_topk(p, B, T, N_cap, scores, q_pos, out_idx, ws, ws_bytes, stream=None):
    s = lib().csa_topk(ctypes.byref(p), B, T, N_cap, _ptr(scores), _ptr(q_pos), _ptr(out_idx),
                       _ptr(ws), ws_bytes, _stream(stream))
    _check("csa_topk", s)


def csa_topk_noalloc(p, B, T, N_cap, scores, q_pos, out_idx, stream=None):
    """csa_topk without caller scratch: the library's own device array serves as scratch
    (nothing is allocated). Calls on one device share that array, so they must not overlap
    in execution; the first call on a device should come before any stream capture."""
    s = lib().csa_topk_noalloc(ctypes.byref(p), B, T, N_cap, _ptr(scores), _ptr(q_pos),
                               _ptr(out_idx), _stream(stream))
    _check("csa_topk_noalloc", s)


def csa_index_topk(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos, out_idx,
                   out_scores, ws, ws_bytes, stream=None):
    s = lib().csa_index_topk(ctypes.byref(p), kdt, B, T, N_cap, _ptr(qI), _ptr(qI_scale),
                             _ptr(w), _ptr(KI), _ptr(KI_scale), _ptr(q_pos), _ptr(out_idx),
                             _ptr(out_scores), _ptr(ws), ws_bytes, _stream(stream))
    _check("csa_index_topk", s)


def csa_index_topk_bf16(p, kdt, B, T, N_cap, qI, qI_scale, w, KI, KI_scale, q_pos, out_idx,
                        out_scores16, ws, ws_bytes, stream=None):
    s = lib().csa_index_topk_bf16(ctypes.byref(p), kdt, B, T, N_cap, _ptr(qI), _ptr(qI_scale),
                                  _ptr(w), _ptr(KI), _ptr(KI_scale), _ptr(q_pos), _ptr(out_idx),
                                  _ptr(out_scores16), _ptr(ws), ws_bytes, _stream(stream))
    _check("csa_index_topk_bf16", s)


def csa_sparse_mqa(p, io, B, T, q, q_pos, kv_cache, N_cap, idx, win_kv, L_raw, win_pos0, sink,
                   q_rms_w, out, ws, ws_bytes, stream=None):
    s = lib().csa_sparse_mqa(ctypes.byref(p), io, B, T, _ptr(q), _ptr(q_pos), _ptr(kv_cache),
                             N_cap, _ptr(idx), _ptr(win_kv), L_raw, _ptr(win_pos0), _ptr(sink),
                             _ptr(q_rms_w), _ptr(out), _ptr(ws), ws_bytes, _stream(stream))
    _check("csa_sparse_mqa", s)


def hca_dense_mqa(p, io, B, T, q, q_pos, kv_cache, N_cap, win_kv, L_raw, win_pos0, sink,
                  q_rms_w, out, ws, ws_bytes, stream=None):
    s = lib().hca_dense_mqa(ctypes.byref(p), io, B, T, _ptr(q), _ptr(q_pos), _ptr(kv_cache),
                            N_cap, _ptr(win_kv), L_raw, _ptr(win_pos0), _ptr(sink),
                            _ptr(q_rms_w), _ptr(out), _ptr(ws), ws_bytes, _stream(stream))
    _check("hca_dense_mqa", s)


def csa_sparse_mqa_mixed_kv(p, B, T, q, q_pos, kv_rows, kv_scale, N_cap, idx, win_kv, L_raw,
                            win_pos0, sink, q_rms_w, out, ws, ws_bytes, stream=None):
    s = lib().csa_sparse_mqa_mixed_kv(ctypes.byref(p), B, T, _ptr(q), _ptr(q_pos),
                                      _ptr(kv_rows), _ptr(kv_scale), N_cap, _ptr(idx),
                                      _ptr(win_kv), L_raw, _ptr(win_pos0), _ptr(sink),
                                      _ptr(q_rms_w), _ptr(out), _ptr(ws), ws_bytes,
                                      _stream(stream))
    _check("csa_sparse_mqa_mixed_kv", s)


def hca_dense_mqa_mixed_kv(p, B, T, q, q_pos, kv_rows, kv_scale, N_cap, win_kv, L_raw,
                           win_pos0, sink, q_rms_w, out, ws, ws_bytes, stream=None):
    s = lib().hca_dense_mqa_mixed_kv(ctypes.byref(p), B, T, _ptr(q), _ptr(q_pos), _ptr(kv_rows),
                                     _ptr(kv_scale), N_cap, _ptr(win_kv), L_raw, _ptr(win_pos0),
                                     _ptr(sink), _ptr(q_rms_w), _ptr(out), _ptr(ws), ws_bytes,
                                     _stream(stream))
    _check("hca_dense_mqa_mixed_kv", s)


def paged_kv(fmt, pages, scales, page_table, n_pages, page_rows, max_pages) -> CsaPagedKv:
    """A csa_paged_kv over device tensors. The descriptor holds only their addresses, so it
    also keeps a reference to each tensor: a pool or page table passed as a temporary would
    otherwise be freed at once, and its memory reused before the kernels read it."""
    kv = CsaPagedKv(int(fmt), _ptr(pages), _ptr(scales), _ptr(page_table), n_pages,
                    page_rows, max_pages)
    kv._tensors = (pages, scales, page_table)
    return kv


def csa_sparse_mqa_paged(p, B, T, q, q_pos, kv: CsaPagedKv, idx, win_kv, L_raw, win_pos0, sink,
                         q_rms_w, out, ws, ws_bytes, stream=None):
    s = lib().csa_sparse_mqa_paged(ctypes.byref(p), B, T, _ptr(q), _ptr(q_pos), ctypes.byref(kv),
                                   _ptr(idx), _ptr(win_kv), L_raw, _ptr(win_pos0), _ptr(sink),
                                   _ptr(q_rms_w), _ptr(out), _ptr(ws), ws_bytes,
                                   _stream(stream))
    _check("csa_sparse_mqa_paged", s)


def hca_dense_mqa_paged(p, B, T, q, q_pos, kv: CsaPagedKv, win_kv, L_raw, win_pos0, sink,
                        q_rms_w, out, ws, ws_bytes, stream=None):
    s = lib().hca_dense_mqa_paged(ctypes.byref(p), B, T, _ptr(q), _ptr(q_pos), ctypes.byref(kv),
                                  _ptr(win_kv), L_raw, _ptr(win_pos0), _ptr(sink),
                                  _ptr(q_rms_w), _ptr(out), _ptr(ws), ws_bytes, _stream(stream))
    _check("hca_dense_mqa_paged", s)


def csa_index_topk_paged(p, B, T, keys: CsaPagedKv, qI, qI_scale, w, q_pos, bf16_scores, out_idx,
                         out_scores, ws, ws_bytes, stream=None):
    s = lib().csa_index_topk_paged(ctypes.byref(p), B, T, ctypes.byref(keys), _ptr(qI),
                                   _ptr(qI_scale), _ptr(w), _ptr(q_pos), int(bf16_scores),
                                   _ptr(out_idx), _ptr(out_scores), _ptr(ws), ws_bytes,
                                   _stream(stream))
    _check("csa_index_topk_paged", s)


def csa_forward_paged(p, B, T, kv: CsaPagedKv, keys: CsaPagedKv, bf16_scores, qI, qI_scale, w, q,
                      q_rms_w, q_pos, win_kv, L_raw, win_pos0, sink, out_idx, out_scores, out, ws,
                      ws_bytes, stream=None):
    s = lib().csa_forward_paged(ctypes.byref(p), B, T, ctypes.byref(kv), ctypes.byref(keys),
                                int(bf16_scores), _ptr(qI), _ptr(qI_scale), _ptr(w), _ptr(q),
                                _ptr(q_rms_w), _ptr(q_pos), _ptr(win_kv), L_raw, _ptr(win_pos0),
                                _ptr(sink), _ptr(out_idx), _ptr(out_scores), _ptr(out), _ptr(ws),
                                ws_bytes, _stream(stream))
    _check("csa_forward_paged", s)


def csa_compress_paged(p, io, B, n_tok, first_entry, Ca, Cb, Za, Zb, bias, prev_Cb, prev_Zb,
                       kv_rms_w, finalize, out_pages: CsaPagedKv, stream=None):
    s = lib().csa_compress_paged(ctypes.byref(p), io, B, n_tok, first_entry, _ptr(Ca), _ptr(Cb),
                                 _ptr(Za), _ptr(Zb), _ptr(bias), _ptr(prev_Cb), _ptr(prev_Zb),
                                 _ptr(kv_rms_w), int(finalize), ctypes.byref(out_pages),
                                 _stream(stream))
    _check("csa_compress_paged", s)


def csa_encode_paged(p, io, B, n, first_entry, rows, out_pages: CsaPagedKv, stream=None):
    s = lib().csa_encode_paged(ctypes.byref(p), io, B, n, first_entry, _ptr(rows),
                               ctypes.byref(out_pages), _stream(stream))
    _check("csa_encode_paged", s)


def csa_state_resume(p, io, B, first_tok, n_tok, Ca, Cb, Za, Zb, win_rows, state, win_ring,
                     stream=None):
    s = lib().csa_state_resume(ctypes.byref(p), io, B, first_tok, n_tok, _ptr(Ca), _ptr(Cb),
                               _ptr(Za), _ptr(Zb), _ptr(win_rows), _ptr(state), _ptr(win_ring),
                               _stream(stream))
    _check("csa_state_resume", s)


def grouped_out_proj_workspace_size(p, Q, g, d_g, d) -> int:
    return int(lib().csa_grouped_out_proj_workspace_size(ctypes.byref(p), Q, g, d_g, d))


def csa_grouped_out_proj(p, Q, g, d_g, d, o, w_grp, w_out, out, ws, ws_bytes, stream=None):
    s = lib().csa_grouped_out_proj(ctypes.byref(p), Q, g, d_g, d, _ptr(o), _ptr(w_grp),
                                   _ptr(w_out), _ptr(out), _ptr(ws), ws_bytes, _stream(stream))
    _check("csa_grouped_out_proj", s)


def forward_args(**kw) -> CsaForwardArgs:
    """Build a csa_forward_args from tensors / ints (pointers are taken with _ptr)."""
    a = CsaForwardArgs()
    ints = {"n_tok", "first_entry", "N_cap", "L_raw", "idx_dtype"}
    for k, v in kw.items():
        setattr(a, k, int(v) if k in ints else _ptr(v))
    return a


def csa_forward(p, io, B, T, args: CsaForwardArgs, ws, ws_bytes, stream=None):
    s = lib().csa_forward(ctypes.byref(p), io, B, T, ctypes.byref(args), _ptr(ws), ws_bytes,
                          _stream(stream))
    _check("csa_forward", s)


def set_index_timing_events(events_before, events_after):
    """Hand the library K (before, after) torch.cuda.Event pairs for the indexer kernel;
    pass empty lists to clear."""
    n = len(events_before)
    arr_t = _VP * max(n, 1)
    b = arr_t(*[e.cuda_event for e in events_before]) if n else arr_t()
    a = arr_t(*[e.cuda_event for e in events_after]) if n else arr_t()
    lib().csa_set_index_timing_events(b, a, n)
