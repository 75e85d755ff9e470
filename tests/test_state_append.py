"""Decode-time compression with a state cache (csa_state_append) against the float64
oracle of the state cache.

Every request appends one token per call, in position order: a request that starts the
sequence, one resumed mid-block after a prefill and one resumed on a page boundary. After
the appends, the finished entries (read through a shuffled page table), the window ring and
the raw state slots are compared with the oracle's state cache fed the same tokens. The
compressed indexer keys (c = 128, no RMSNorm / RoPE) are also stored in the formats the
indexers read: FP8 with a row scale, and MXFP4 with exponents in 128-row blocks. Their
codes must equal the input encoders' codes of the same fp32 keys bit for bit, and decode to
within the format's rounding of the oracle's keys.

The CPU tests run the kernel's own arithmetic (csrc/state_append.cuh) built for the host
by tests/host_check/state_append_host.cu, with every offset checked against its buffer;
the `gpu` tests run the library's kernel through the C ABI on the same streams.
"""
import ctypes
import functools
import os
import subprocess

import numpy as np
import pytest

from oracle import csa_oracle as O
from oracle import state_cache as SC
from long_context_sparse_08_b200 import workloads as W
import tests.parity_util as U

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, m, overlap, page_rows, starts, appends): CSA m = 4 with 128-token pages of 32
# entries; HCA m' = 128 with pages of 1 entry. c = 512, r = 64, n_win = 128 throughout.
CASES = [
    ("csa", 4, 1, 32, (0, 150, 256), 200),
    ("hca", 128, 0, 1, (0, 300), 300),
]
C, R, N_WIN, BASE, EPS = 512, 64, 128, 10000.0, 1e-6
OUT_IO, OUT_FP8, OUT_MXFP4, OUT_MIXED = 0, 1, 2, 3


@functools.lru_cache(maxsize=1)
def host_lib():
    out = os.path.join(ROOT, "tests", "host_check", "_build")
    os.makedirs(out, exist_ok=True)
    so = os.path.join(out, "libstate_append_host.so")
    src = os.path.join(ROOT, "tests", "host_check", "state_append_host.cu")
    hdr = os.path.join(ROOT, "long_context_sparse_08_b200", "csrc", "state_append.cuh")
    if not os.path.exists(so) or os.path.getmtime(so) < max(os.path.getmtime(src),
                                                            os.path.getmtime(hdr)):
        subprocess.run(["nvcc", "-O2", "-shared", "-Xcompiler", "-fPIC", "-arch=sm_100a",
                        "-I", os.path.join(ROOT, "include"),
                        "-I", os.path.join(ROOT, "long_context_sparse_08_b200", "csrc"),
                        src, "-o", so], check=True, capture_output=True)
    L = ctypes.CDLL(so)
    L.state_append_host.restype = ctypes.c_int
    L.encode_rows_host.restype = ctypes.c_int
    L.state_resume_host.restype = ctypes.c_int
    return L


def _np_ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Scenario:
    """Token streams, page tables and buffers of one case (host numpy arrays)."""

    def __init__(self, name, m, overlap, page_rows, starts, appends, io, seed=900, c=C,
                 finalize=1, out=OUT_IO, n_win=N_WIN):
        self.name, self.m, self.overlap, self.page_rows = name, m, overlap, page_rows
        self.starts, self.appends, self.io = np.array(starts), appends, io
        self.c, self.finalize, self.out, self.n_win = c, finalize, out, n_win
        self.B = len(starts)
        n_tok = max(starts) + appends
        self.inp = W.make_state_stream(B=self.B, n_tok=n_tok, m=m, c=c, overlap=overlap, io=io,
                                       seed=seed + m)
        self.max_pages = -(-(n_tok // m) // page_rows) + 1
        self.n_pages = self.B * self.max_pages + 3
        g = np.random.default_rng(seed)
        perm = g.permutation(self.n_pages).astype(np.int32)
        self.page_table = perm[:self.B * self.max_pages].reshape(self.B, self.max_pages).copy()
        S = 2 * m if overlap else m
        Rr = 4 if overlap else 2
        dt = np.uint16 if io == "bf16" else np.float32
        self.state = np.zeros((self.B, S, Rr, c), dt)
        self.ring = np.zeros((self.B, n_win, c), dt)
        self.alloc_pages()
        # a resumed request's state holds the raw rows of its last 2m (m') prefill tokens,
        # and its ring the last n_win prefill window rows
        names = ("Ca", "Za", "Cb", "Zb") if overlap else ("Ca", "Za")
        for b, t0 in enumerate(starts):
            for p in range(max(t0 - S, 0), t0):
                for r, k in enumerate(names):
                    self.state[b, p % S, r] = self.inp[k][b, p]
            for p in range(max(t0 - n_win, 0), t0):
                self.ring[b, p % n_win] = self.inp["win"][b, p]

    def alloc_pages(self):
        n, pr, c = self.n_pages, self.page_rows, self.c
        if self.out == OUT_IO:
            self.pages = np.zeros((n, pr, c), np.uint16 if self.io == "bf16" else np.float32)
            self.scales = None
        elif self.out == OUT_FP8:
            self.pages = np.zeros((n, pr, c), np.uint8)
            self.scales = np.zeros((n, pr), np.float32)
        elif self.out == OUT_MIXED:
            self.pages = np.zeros((n, pr, c + R), np.uint8)
            self.scales = np.zeros((n, pr), np.float32)
        else:
            self.pages = np.zeros((n, pr, c // 2), np.uint8)
            self.scales = np.zeros((n, pr, 4), np.uint8)

    def step_rows(self, k, step):
        """[B, c] rows of tensor k for append number `step` of every request."""
        return np.ascontiguousarray(self.inp[k][np.arange(self.B), self.starts + step])

    def dec(self, x):
        return O.dec_io(x, self.io)

    def entry_range(self, b):
        t0 = int(self.starts[b])
        return t0 // self.m, (t0 + self.appends) // self.m  # entries made by the appends

    def page_row(self, b, i):
        return self.page_table[b, i // self.page_rows], i % self.page_rows

    def oracle(self):
        """Oracle state caches after the same appends, one per request."""
        out = []
        bias = self.dec(self.inp["bias"])

        def fin(ent):
            return O.finalize_entries(ent, 0, self.m, R, BASE, EPS) if self.finalize else ent

        for b, t0 in enumerate(self.starts):
            kw = dict(m=self.m, c=self.c, bias=bias, n_win=self.n_win, r=R, base=BASE, eps=EPS,
                      block_tokens=self.m * self.page_rows, finalize=bool(self.finalize))
            pool = SC.PagePool(self.max_pages, self.page_rows, self.c)
            rows = {k: self.dec(self.inp[k][b]) for k in self.inp if k != "bias"}
            nb = t0 // self.m
            if self.overlap:
                st = SC.CsaState(pool, **kw)
                ent = O.compress_csa(rows["Ca"][:self.m * nb], rows["Cb"][:self.m * nb],
                                     rows["Za"][:self.m * nb], rows["Zb"][:self.m * nb], bias,
                                     self.m)
                st.resume(rows["Ca"][:t0], rows["Cb"][:t0], rows["Za"][:t0], rows["Zb"][:t0],
                          fin(ent), rows["win"][:t0])
                for t in range(t0, t0 + self.appends):
                    st.append(rows["Ca"][t], rows["Cb"][t], rows["Za"][t], rows["Zb"][t],
                              rows["win"][t])
            else:
                st = SC.HcaState(pool, **kw)
                ent = O.compress_hca(rows["Ca"][:self.m * nb], rows["Za"][:self.m * nb], bias,
                                     self.m)
                st.resume(rows["Ca"][:t0], rows["Za"][:t0], fin(ent), rows["win"][:t0])
                for t in range(t0, t0 + self.appends):
                    st.append(rows["Ca"][t], rows["Za"][t], rows["win"][t])
            out.append(st)
        return out

    def check(self, pages, ring, state, what):
        """Compare the appended entries (stored in the io dtype), the ring and the raw
        slots with the oracle."""
        assert self.out == OUT_IO
        pages, ring, state = (self.dec(x) for x in (pages, ring, state))
        for b, st in enumerate(self.oracle()):
            first, last = self.entry_range(b)
            t1 = int(self.starts[b]) + self.appends
            assert st.n_entries == last
            ref = st.entries()[first:last]
            got = np.stack([pages[self.page_row(b, i)] for i in range(first, last)])
            U.check_rows(got, ref, self.io, f"{what} request {b} entries {first}..{last - 1}")
            # window ring: exactly the last n_win window rows, each in slot p % n_win
            for p in range(max(t1 - self.n_win, 0), t1):
                assert np.array_equal(ring[b, p % self.n_win], self.dec(self.inp["win"][b, p])), \
                    f"{what} request {b}: ring slot of position {p}"
            # raw state: the rows of the last S tokens, each in slot p % S
            S = state.shape[1]
            names = ("Ca", "Za", "Cb", "Zb") if self.overlap else ("Ca", "Za")  # slot rows
            for p in range(max(t1 - S, 0), t1):
                for r, k in enumerate(names):
                    assert np.array_equal(state[b, p % S, r], self.dec(self.inp[k][b, p]))

    def appended(self):
        """(request, entry) pairs the appends finished, in order."""
        return [(b, i) for b in range(self.B) for i in range(*self.entry_range(b))]

    def keys(self, pages):
        """fp32 rows (keys or KV entries) the appends finished, [n, c], from pages stored as
        f32."""
        return np.stack([pages[self.page_row(b, i)] for b, i in self.appended()])

    def check_encoded(self, keys_f32, pages, scales, what):
        """Quantised pages against (1) the input encoders applied to the same fp32 keys, bit
        for bit, and (2) the oracle's keys within the format's rounding."""
        at = self.appended()
        ora = self.oracle()
        ref = np.stack([ora[b].entries()[i] for b, i in at])
        U.check_rows(keys_f32, ref, "f32", f"{what}: fp32 keys")
        got = np.stack([pages[self.page_row(b, i)] for b, i in at])
        if self.out == OUT_MIXED:
            codes, sc, rope = W.quant_mixed_kv(keys_f32, R)
            got_sc = np.array([scales[self.page_row(b, i)] for b, i in at])
            r0 = self.c - R
            got_rope = np.ascontiguousarray(got[:, r0:]).view(np.uint16)
            assert np.array_equal(got[:, :r0], codes), f"{what}: e4m3 codes"
            assert np.array_equal(got_sc, sc), f"{what}: row scales"
            assert np.array_equal(got_rope, rope), f"{what}: bf16 RoPE values"
            dq = O.dec_mixed_kv(got[:, :r0], got_sc, got_rope)
            rms = np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
            bound = np.concatenate([
                np.maximum(np.abs(ref[:, :r0]) * 2.0 ** -4, got_sc[:, None] * 2.0 ** -10) * 1.01,
                np.abs(ref[:, r0:]) * 2.0 ** -8 * 1.01], axis=1) + 2e-4 * rms
            assert np.all(np.abs(dq - ref) <= bound), f"{what}: mixed rows vs oracle"
            return
        if self.out == OUT_FP8:
            codes, sc = W.quant_fp8_rowwise(keys_f32)
            got_sc = np.array([scales[self.page_row(b, i)] for b, i in at])
            assert np.array_equal(got, codes), f"{what}: e4m3 codes"
            assert np.array_equal(got_sc, sc), f"{what}: row scales"
            dq = O.dec_fp8_rows(got, got_sc)
            # half an e4m3 step (2^-4 of |x|, or 2^-10 x scale below the normal range) plus
            # the fp32 keys' own error against the oracle
            bound = np.maximum(np.abs(ref) * 2.0 ** -4, got_sc[:, None] * 2.0 ** -10) * 1.01 + \
                2e-4 * np.sqrt(np.mean(ref * ref, axis=1, keepdims=True))
            assert np.all(np.abs(dq - ref) <= bound), f"{what}: FP8 keys vs oracle"
            return
        packed, ex = W.quant_mxfp4(keys_f32)
        assert np.array_equal(got, packed), f"{what}: e2m1 codes"
        e = np.stack([O.unblock_key_scales(scales[self.page_row(b, i)[0]])[self.page_row(b, i)[1]]
                      for b, i in at])
        assert np.array_equal(e, ex), f"{what}: exponents"
        dq = O.dec_mxfp4(got, e)
        # at most one e2m1 step of 2 * 2^E (the widest, between 4 and 6, and saturation
        # from below 8 to 6) plus the fp32 keys' own error
        step = np.repeat(np.exp2(e.astype(np.float64) - 127.0 + 1.0), 32, axis=1)
        assert np.all(np.abs(dq - ref) <= step + 2e-4 * np.abs(ref).max()), \
            f"{what}: MXFP4 keys vs oracle"


def _run_host(sc: Scenario):
    L = host_lib()
    status = np.zeros(sc.B, np.int32)
    for step in range(sc.appends):
        pos = (sc.starts + step).astype(np.int64)
        rows = {k: sc.step_rows(k, step) for k in sc.inp if k != "bias"}
        rc = L.state_append_host(
            int(sc.io == "bf16"), sc.B, sc.m, sc.c, sc.overlap, R, ctypes.c_double(BASE),
            sc.finalize, sc.n_win, sc.n_pages, sc.page_rows, sc.max_pages, ctypes.c_float(EPS),
            sc.out, _np_ptr(pos), _np_ptr(rows["Ca"]), _np_ptr(rows.get("Cb")),
            _np_ptr(rows["Za"]), _np_ptr(rows.get("Zb")), _np_ptr(rows["win"]),
            _np_ptr(sc.inp["bias"]), None, _np_ptr(sc.state), _np_ptr(sc.ring),
            _np_ptr(sc.pages), ctypes.c_size_t(sc.pages.nbytes), _np_ptr(sc.scales),
            ctypes.c_size_t(0 if sc.scales is None else sc.scales.nbytes),
            _np_ptr(sc.page_table), _np_ptr(status))
        assert rc == 0, f"offset outside a buffer ({rc}) at append {step}"
        assert (status >= 0).all()
    return sc.pages, sc.ring, sc.state


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_host_build_of_the_kernel_arithmetic_matches_the_oracle(case, io):
    sc = Scenario(*case, io=io)
    sc.check(*_run_host(sc), what=f"host {case[0]} {io}")


# odd geometries for the host build: pages of 7 and 3 entries, a window shorter than a
# block, c = 128 and c = 64, finalize off, HCA with a small m'
ODD = [
    dict(name="csa", m=4, overlap=1, page_rows=7, starts=(0, 57, 130), appends=90, c=128, n_win=3),
    dict(name="csa", m=4, overlap=1, page_rows=3, starts=(5, 64), appends=70, c=64, n_win=9,
         finalize=0),
    dict(name="hca", m=16, overlap=0, page_rows=1, starts=(0, 37), appends=80, c=64, n_win=5),
]


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("cfg", ODD, ids=["csa_pages7", "csa_pages3_raw", "hca_m16"])
def test_host_build_on_odd_geometries(cfg, io):
    cfg = dict(cfg)
    sc = Scenario(cfg.pop("name"), cfg.pop("m"), cfg.pop("overlap"), cfg.pop("page_rows"),
                  cfg.pop("starts"), cfg.pop("appends"), io=io, seed=55, **cfg)
    pages, ring, state = _run_host(sc)
    sc.check(pages, ring, state, what=f"host odd {io}")


def _key_scenarios(out):
    # CSA indexer keys: c = 128, no RMSNorm / RoPE, pages of 128 rows (a multiple of the
    # 32-entry block, as the MXFP4 exponent blocks need); the request resumed at 480 crosses
    # from its first page to its second (entry 128)
    return [Scenario("keys", 4, 1, 128, (0, 150, 480), 200, io="f32", c=128, finalize=0,
                     out=o, seed=31) for o in (OUT_IO, out)]


@pytest.mark.parametrize("out", [OUT_FP8, OUT_MXFP4], ids=["fp8", "mxfp4"])
def test_host_build_stores_indexer_keys_in_the_indexer_formats(out):
    plain, enc = _key_scenarios(out)
    pages_f32 = _run_host(plain)[0]
    pages = _run_host(enc)[0]
    enc.check_encoded(plain.keys(pages_f32), pages, enc.scales, f"host keys {out}")


def _mixed_scenarios():
    # KV entries (c = 512, RMSNorm + RoPE) stored with their RoPE dims in bf16 and the rest
    # in FP8; pages of 32 entries
    return [Scenario("kv", 4, 1, 32, (0, 150, 256), 120, io="f32", out=o, seed=41)
            for o in (OUT_IO, OUT_MIXED)]


def test_host_build_stores_mixed_precision_kv_rows():
    plain, enc = _mixed_scenarios()
    pages_f32 = _run_host(plain)[0]
    pages = _run_host(enc)[0]
    enc.check_encoded(plain.keys(pages_f32), pages, enc.scales, "host mixed KV")


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_host_build_of_the_resume_fills_the_state_of_a_prefill(case):
    """csa_state_resume's arithmetic fills the state slots and the window ring of requests
    resumed after a prefill exactly as the scenario's own (independently written) fill."""
    name, m, overlap, page_rows, starts, appends = case
    L = host_lib()
    for t0 in starts:
        if t0 == 0:
            continue
        sc = Scenario(name, m, overlap, page_rows, (t0,), appends, io="bf16")
        st = np.zeros_like(sc.state)
        ring = np.zeros_like(sc.ring)
        rows = {k: np.ascontiguousarray(sc.inp[k][:, :t0]) for k in sc.inp if k != "bias"}
        rc = L.state_resume_host(1, 1, m, C, overlap, N_WIN, ctypes.c_int64(0),
                                 ctypes.c_int64(t0), _np_ptr(rows["Ca"]),
                                 _np_ptr(rows.get("Cb")), _np_ptr(rows["Za"]),
                                 _np_ptr(rows.get("Zb")), _np_ptr(rows["win"]), _np_ptr(st),
                                 _np_ptr(ring))
        assert rc == 0
        assert np.array_equal(st, sc.state) and np.array_equal(ring, sc.ring)


def test_host_encoders_equal_the_input_encoders():
    """The row encoders alone, on rows with zero, tiny, huge and midpoint values."""
    L = host_lib()
    g = np.random.default_rng(5)
    n = 256
    x = (g.standard_normal((n, 128)) * np.exp2(g.integers(-20, 20, size=(n, 1)))).astype(np.float32)
    x[0] = 0.0
    x[1, :] = 1e-30
    x[2, :32] = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5] * 4, np.float32)
    x[2, 0] = 4.0  # block amax 6.5 -> exponent 0, so the others sit on e2m1 midpoints
    x[3, :] = 3e38
    codes = np.zeros((n, 128), np.uint8)
    scales = np.zeros(n, np.float32)
    assert L.encode_rows_host(OUT_FP8, n, 128, _np_ptr(x), _np_ptr(codes), _np_ptr(scales)) == 0
    want_codes, want_scales = W.quant_fp8_rowwise(x)
    assert np.array_equal(codes, want_codes)
    assert np.array_equal(scales, want_scales)
    packed = np.zeros((n, 64), np.uint8)
    exps = np.zeros((n, 4), np.uint8)
    assert L.encode_rows_host(OUT_MXFP4, n, 128, _np_ptr(x), _np_ptr(packed), _np_ptr(exps)) == 0
    want_packed, want_exps = W.quant_mxfp4(x)
    assert np.array_equal(packed, want_packed)
    assert np.array_equal(exps, W.block_key_scales(want_exps))


def _host_one_step(sc, pos):
    L = host_lib()
    status = np.zeros(sc.B, np.int32)
    rows = {k: sc.step_rows(k, 0) for k in sc.inp if k != "bias"}
    before = sc.state.copy()
    rc = L.state_append_host(0, sc.B, sc.m, sc.c, 1, R, ctypes.c_double(BASE), 1, sc.n_win,
                             sc.n_pages, sc.page_rows, sc.max_pages, ctypes.c_float(EPS), OUT_IO,
                             _np_ptr(pos), _np_ptr(rows["Ca"]), _np_ptr(rows["Cb"]),
                             _np_ptr(rows["Za"]), _np_ptr(rows["Zb"]), _np_ptr(rows["win"]),
                             _np_ptr(sc.inp["bias"]), None, _np_ptr(sc.state), _np_ptr(sc.ring),
                             _np_ptr(sc.pages), ctypes.c_size_t(sc.pages.nbytes), None,
                             ctypes.c_size_t(0), _np_ptr(sc.page_table), _np_ptr(status))
    assert rc == 0
    bad = status < 0
    assert np.array_equal(sc.state[bad], before[bad])  # skipped requests wrote nothing
    return status


def test_host_build_skips_requests_with_bad_pages():
    sc = Scenario("csa", 4, 1, 32, (124, 127, 3), 1, io="f32")
    sc.page_table[0, 0] = -1          # entry 31 of request 0: page id -1
    sc.page_table[1, 0] = sc.n_pages  # entry 31 of request 1: page id out of range
    assert _host_one_step(sc, np.array([127, 127, 3], np.int64)).tolist() == [-3, -3, 1]
    sc2 = Scenario("csa", 4, 1, 32, (0,), 1, io="f32")
    # entry 32 * max_pages: its logical page is past the table
    assert _host_one_step(sc2, np.array([4 * 32 * sc2.max_pages + 3], np.int64))[0] == -2
    assert _host_one_step(sc2, np.array([-5], np.int64))[0] == -1


# ---------------------------------------------------------------------------
# the library's kernel (GPU)
# ---------------------------------------------------------------------------


def _run_gpu(sc: Scenario, check_error=True):
    import torch
    import long_context_sparse_08_b200 as csa

    torch.cuda.synchronize()
    csa.device_error()  # start from a clear error word

    def up(x):
        a = np.ascontiguousarray(x)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()

    def down(t, like):
        a = t.cpu().numpy()
        return a.view(np.uint16) if like.dtype == np.uint16 else a

    p = csa.make_params(m=sc.m, overlap=sc.overlap, c=sc.c, rope_dims=R, rope_base=BASE,
                        rms_eps=EPS, n_win=sc.n_win)
    io = csa.CSA_BF16 if sc.io == "bf16" else csa.CSA_F32
    out_fmt = {OUT_IO: io, OUT_FP8: csa.CSA_FP8_E4M3_ROWSCALE, OUT_MXFP4: csa.CSA_MXFP4,
               OUT_MIXED: csa.CSA_MIXED_FP8_BF16}[sc.out]
    state, ring, pages = up(sc.state), up(sc.ring), up(sc.pages)
    scales = None if sc.scales is None else up(sc.scales)
    table = up(sc.page_table)
    bias = up(sc.inp["bias"])
    streams = {k: up(sc.inp[k]) for k in sc.inp if k != "bias"}  # [B, n_tok, c]
    starts = up(sc.starts.astype(np.int64))
    ar = torch.arange(sc.B, device="cuda")
    for step in range(sc.appends):
        pos = starts + step
        rows = {k: v[ar, pos].contiguous() for k, v in streams.items()}
        csa.csa_state_append(p, io, sc.B, pos, rows["Ca"], rows.get("Cb"), rows["Za"],
                             rows.get("Zb"), rows["win"], bias, None, sc.finalize, state, ring,
                             out_fmt, pages, scales, sc.n_pages, sc.page_rows, table,
                             sc.max_pages)
    torch.cuda.synchronize()
    if check_error:
        assert csa.device_error() == 0
    return (down(pages, sc.pages), down(ring, sc.ring), down(state, sc.state),
            None if scales is None else scales.cpu().numpy())


@pytest.mark.gpu
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gpu_state_append_matches_the_oracle(case, io):
    sc = Scenario(*case, io=io)
    sc.check(*_run_gpu(sc)[:3], what=f"gpu {case[0]} {io}")


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", ODD, ids=["csa_pages7", "csa_pages3_raw", "hca_m16"])
def test_gpu_state_append_on_odd_geometries(cfg):
    cfg = dict(cfg)
    sc = Scenario(cfg.pop("name"), cfg.pop("m"), cfg.pop("overlap"), cfg.pop("page_rows"),
                  cfg.pop("starts"), cfg.pop("appends"), io="bf16", seed=55, **cfg)
    sc.check(*_run_gpu(sc)[:3], what="gpu odd")


@pytest.mark.gpu
@pytest.mark.parametrize("out", [OUT_FP8, OUT_MXFP4], ids=["fp8", "mxfp4"])
def test_gpu_stores_indexer_keys_in_the_indexer_formats(out):
    plain, enc = _key_scenarios(out)
    pages_f32 = _run_gpu(plain)[0]
    pages, _, _, scales = _run_gpu(enc)
    enc.check_encoded(plain.keys(pages_f32), pages, scales, f"gpu keys {out}")


@pytest.mark.gpu
def test_gpu_stores_mixed_precision_kv_rows():
    plain, enc = _mixed_scenarios()
    pages_f32 = _run_gpu(plain)[0]
    pages, _, _, scales = _run_gpu(enc)
    enc.check_encoded(plain.keys(pages_f32), pages, scales, "gpu mixed KV")


@pytest.mark.gpu
def test_gpu_appends_equal_the_whole_chunk_compression():
    """Token-by-token appends into identity pages give the cache csa_compress writes for the
    whole 512-token chunk (same arithmetic, so equal to within one bf16 rounding)."""
    import torch
    import long_context_sparse_08_b200 as csa

    sc = Scenario("csa", 4, 1, 32, (0, 0), 512, io="bf16", seed=77)
    sc.max_pages, sc.n_pages = 4, 8
    sc.page_table = np.arange(8, dtype=np.int32).reshape(2, 4)
    sc.alloc_pages()
    pages = _run_gpu(sc)[0]
    p = csa.make_params(m=4, overlap=1, c=C, rope_dims=R, rope_base=BASE, rms_eps=EPS,
                        n_win=N_WIN)
    dev = lambda k: torch.from_numpy(sc.inp[k].view(np.int16)).cuda()  # noqa: E731
    cache = torch.zeros((2, 128, C), dtype=torch.int16, device="cuda")
    csa.csa_compress(p, csa.CSA_BF16, 2, 512, 0, 128, dev("Ca"), dev("Cb"), dev("Za"),
                     dev("Zb"), dev("bias"), None, None, None, 1, cache)
    torch.cuda.synchronize()
    whole = O.dec_bf16(cache.cpu().numpy().view(np.uint16))
    got = O.dec_bf16(pages.reshape(2, 128, C))
    assert np.all(np.abs(got - whole) <= U.bf16_ulp(whole))


@pytest.mark.gpu
def test_gpu_state_append_skips_requests_with_bad_pages():
    import long_context_sparse_08_b200 as csa

    # requests 0 and 1 finish entry 31 into a page id outside the pool; request 2 (t = 3)
    # finishes its entry 0 normally
    sc = Scenario("csa", 4, 1, 32, (127, 127, 3), 1, io="f32")
    sc.page_table[0, 0] = -1
    sc.page_table[1, 0] = sc.n_pages
    before = sc.state.copy()
    pages, _, state, _ = _run_gpu(sc, check_error=False)
    assert csa.device_error() == 323
    assert np.array_equal(state[:2], before[:2])  # skipped requests stored nothing
    own = sc.page_table[2, 0]
    assert np.abs(pages[own, 0]).sum() > 0
    rest = pages.copy()
    rest[own, 0] = 0
    assert not rest.any()


# ---------------------------------------------------------------------------
# prefill -> decode hand-over on paged caches
# ---------------------------------------------------------------------------

@pytest.mark.gpu
def test_gpu_paged_compression_equals_contiguous():
    import torch
    import long_context_sparse_08_b200 as csa

    sc = Scenario("csa", 4, 1, 32, (0, 0), 512, io="bf16", seed=78)
    p = csa.make_params(m=4, overlap=1, c=C, rope_dims=R, rope_base=BASE, rms_eps=EPS,
                        n_win=N_WIN)
    dev = lambda k: torch.from_numpy(sc.inp[k].view(np.int16)).cuda()  # noqa: E731
    cache = torch.zeros((2, 128, C), dtype=torch.int16, device="cuda")
    csa.csa_compress(p, csa.CSA_BF16, 2, 512, 0, 128, dev("Ca"), dev("Cb"), dev("Za"),
                     dev("Zb"), dev("bias"), None, None, None, 1, cache)
    perm = np.random.default_rng(3).permutation(8).astype(np.int32)
    table = torch.from_numpy(perm.reshape(2, 4)).cuda()
    pool = torch.zeros((8, 32, C), dtype=torch.int16, device="cuda")
    pages = csa.paged_kv(csa.CSA_BF16, pool, None, table, 8, 32, 4)
    torch.cuda.synchronize()
    csa.device_error()
    csa.csa_compress_paged(p, csa.CSA_BF16, 2, 512, 0, dev("Ca"), dev("Cb"), dev("Za"),
                           dev("Zb"), dev("bias"), None, None, None, 1, pages)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    got = pool[table.view(-1).long()].view(2, 128, C)
    assert torch.equal(got, cache)


@pytest.mark.gpu
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gpu_resume_fills_the_state_of_a_prefill(case):
    import torch
    import long_context_sparse_08_b200 as csa

    name, m, overlap, page_rows, starts, appends = case
    t0 = max(starts)
    sc = Scenario(name, m, overlap, page_rows, (t0,), appends, io="bf16")
    p = csa.make_params(m=m, overlap=overlap, c=C, rope_dims=R, rope_base=BASE, rms_eps=EPS,
                        n_win=N_WIN)
    up = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()  # noqa
    rows = {k: up(sc.inp[k][:, :t0]) for k in sc.inp if k != "bias"}
    st = torch.zeros(sc.state.shape, dtype=torch.int16, device="cuda")
    ring = torch.zeros(sc.ring.shape, dtype=torch.int16, device="cuda")
    csa.csa_state_resume(p, csa.CSA_BF16, 1, 0, t0, rows["Ca"], rows.get("Cb"), rows["Za"],
                         rows.get("Zb"), rows["win"], st, ring)
    torch.cuda.synchronize()
    assert np.array_equal(st.cpu().numpy().view(np.uint16), sc.state)
    assert np.array_equal(ring.cpu().numpy().view(np.uint16), sc.ring)

