"""Decode-time compression with a state cache (csa_state_append) against the float64
oracle of the state cache.

Every request appends one token per call, in position order: a request that starts the
sequence, one resumed mid-block after a prefill and one resumed on a page boundary. After
the appends, the finished entries (read through a shuffled page table), the window ring and
the raw state slots are compared with the oracle's state cache fed the same tokens.

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
    return L


def _np_ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


class Scenario:
    """Token streams, page tables and buffers of one case (host numpy arrays)."""

    def __init__(self, name, m, overlap, page_rows, starts, appends, io, seed=900):
        self.name, self.m, self.overlap, self.page_rows = name, m, overlap, page_rows
        self.starts, self.appends, self.io = np.array(starts), appends, io
        self.B = len(starts)
        n_tok = max(starts) + appends
        self.inp = W.make_state_stream(B=self.B, n_tok=n_tok, m=m, c=C, overlap=overlap, io=io,
                                       seed=seed + m)
        self.max_pages = -(-(n_tok // m) // page_rows) + 1
        self.n_pages = self.B * self.max_pages + 3
        g = np.random.default_rng(seed)
        perm = g.permutation(self.n_pages).astype(np.int32)
        self.page_table = perm[:self.B * self.max_pages].reshape(self.B, self.max_pages).copy()
        S = 2 * m if overlap else m
        Rr = 4 if overlap else 2
        dt = np.uint16 if io == "bf16" else np.float32
        self.state = np.zeros((self.B, S, Rr, C), dt)
        self.ring = np.zeros((self.B, N_WIN, C), dt)
        self.pages = np.zeros((self.n_pages, page_rows, C), dt)
        # a resumed request's state holds the raw rows of its last 2m (m') prefill tokens,
        # and its ring the last n_win prefill window rows
        names = ("Ca", "Za", "Cb", "Zb") if overlap else ("Ca", "Za")
        for b, t0 in enumerate(starts):
            for p in range(max(t0 - S, 0), t0):
                for r, k in enumerate(names):
                    self.state[b, p % S, r] = self.inp[k][b, p]
            for p in range(max(t0 - N_WIN, 0), t0):
                self.ring[b, p % N_WIN] = self.inp["win"][b, p]

    def step_rows(self, k, step):
        """[B, c] rows of tensor k for append number `step` of every request."""
        return np.ascontiguousarray(self.inp[k][np.arange(self.B), self.starts + step])

    def dec(self, x):
        return O.dec_io(x, self.io)

    def oracle(self):
        """Oracle state caches after the same appends, one per request."""
        out = []
        bias = self.dec(self.inp["bias"])
        for b, t0 in enumerate(self.starts):
            kw = dict(m=self.m, c=C, bias=bias, n_win=N_WIN, r=R, base=BASE, eps=EPS,
                      block_tokens=self.m * self.page_rows)
            pool = SC.PagePool(self.max_pages, self.page_rows, C)
            rows = {k: self.dec(self.inp[k][b]) for k in self.inp if k != "bias"}
            if self.overlap:
                st = SC.CsaState(pool, **kw)
                nb = t0 // self.m
                ent = O.compress_csa(rows["Ca"][:self.m * nb], rows["Cb"][:self.m * nb],
                                     rows["Za"][:self.m * nb], rows["Zb"][:self.m * nb], bias,
                                     self.m)
                st.resume(rows["Ca"][:t0], rows["Cb"][:t0], rows["Za"][:t0], rows["Zb"][:t0],
                          O.finalize_entries(ent, 0, self.m, R, BASE, EPS), rows["win"][:t0])
                for t in range(t0, t0 + self.appends):
                    st.append(rows["Ca"][t], rows["Cb"][t], rows["Za"][t], rows["Zb"][t],
                              rows["win"][t])
            else:
                st = SC.HcaState(pool, **kw)
                nb = t0 // self.m
                ent = O.compress_hca(rows["Ca"][:self.m * nb], rows["Za"][:self.m * nb], bias,
                                     self.m)
                st.resume(rows["Ca"][:t0], rows["Za"][:t0],
                          O.finalize_entries(ent, 0, self.m, R, BASE, EPS), rows["win"][:t0])
                for t in range(t0, t0 + self.appends):
                    st.append(rows["Ca"][t], rows["Za"][t], rows["win"][t])
            out.append(st)
        return out

    def check(self, pages, ring, state, what):
        """Compare the appended entries, the ring and the raw slots with the oracle."""
        pages, ring, state = (self.dec(x) for x in (pages, ring, state))
        for b, st in enumerate(self.oracle()):
            t0, t1 = int(self.starts[b]), int(self.starts[b]) + self.appends
            first, last = t0 // self.m, t1 // self.m  # entries made by the appends
            assert st.n_entries == last
            ref = st.entries()[first:last]
            got = np.stack([pages[self.page_table[b, i // self.page_rows], i % self.page_rows]
                            for i in range(first, last)]) if last > first else ref
            U.check_rows(got, ref, self.io, f"{what} request {b} entries {first}..{last - 1}")
            # window ring: exactly the last n_win window rows, each in slot p % n_win
            for p in range(max(t1 - N_WIN, 0), t1):
                assert np.array_equal(ring[b, p % N_WIN], self.dec(self.inp["win"][b, p])), \
                    f"{what} request {b}: ring slot of position {p}"
            # raw state: the rows of the last S tokens, each in slot p % S
            S = state.shape[1]
            names = ("Ca", "Za", "Cb", "Zb") if self.overlap else ("Ca", "Za")
            for p in range(max(t1 - S, 0), t1):
                for r, k in enumerate(names):
                    assert np.array_equal(state[b, p % S, r], self.dec(self.inp[k][b, p]))


def _run_host(sc: Scenario):
    L = host_lib()
    bias = sc.inp["bias"]
    status = np.zeros(sc.B, np.int32)
    for step in range(sc.appends):
        pos = (sc.starts + step).astype(np.int64)
        rows = {k: sc.step_rows(k, step) for k in sc.inp if k != "bias"}
        rc = L.state_append_host(
            int(sc.io == "bf16"), sc.B, sc.m, C, sc.overlap, R, ctypes.c_double(BASE), 1, N_WIN,
            sc.n_pages, sc.page_rows, sc.max_pages, ctypes.c_float(EPS), _np_ptr(pos),
            _np_ptr(rows["Ca"]), _np_ptr(rows.get("Cb")), _np_ptr(rows["Za"]),
            _np_ptr(rows.get("Zb")), _np_ptr(rows["win"]), _np_ptr(bias), None,
            _np_ptr(sc.state), _np_ptr(sc.ring), _np_ptr(sc.pages), _np_ptr(sc.page_table),
            _np_ptr(status))
        assert rc == 0, f"offset outside a buffer ({rc}) at append {step}"
        assert (status >= 0).all()
    return sc.pages, sc.ring, sc.state


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_host_build_of_the_kernel_arithmetic_matches_the_oracle(case, io):
    sc = Scenario(*case, io=io)
    sc.check(*_run_host(sc), what=f"host {case[0]} {io}")


def test_host_build_skips_requests_with_bad_pages():
    sc = Scenario("csa", 4, 1, 32, (124, 127, 3), 1, io="f32")
    sc.page_table[0, 31 // 32] = -1            # entry 31 of request 0: page id -1
    sc.page_table[1, 0] = sc.n_pages           # entry 31 of request 1: page id out of range
    L = host_lib()
    status = np.zeros(sc.B, np.int32)
    pos = np.array([127, 127, 3], np.int64)
    rows = {k: sc.step_rows(k, 0) for k in sc.inp if k != "bias"}
    before = sc.state.copy()
    rc = L.state_append_host(0, sc.B, 4, C, 1, R, ctypes.c_double(BASE), 1, N_WIN, sc.n_pages,
                             32, sc.max_pages, ctypes.c_float(EPS), _np_ptr(pos),
                             _np_ptr(rows["Ca"]), _np_ptr(rows["Cb"]), _np_ptr(rows["Za"]),
                             _np_ptr(rows["Zb"]), _np_ptr(rows["win"]), _np_ptr(sc.inp["bias"]),
                             None, _np_ptr(sc.state), _np_ptr(sc.ring), _np_ptr(sc.pages),
                             _np_ptr(sc.page_table), _np_ptr(status))
    assert rc == 0
    assert status.tolist() == [-3, -3, 1]
    assert np.array_equal(sc.state[:2], before[:2])  # skipped requests wrote nothing
    # a logical page past the table
    sc2 = Scenario("csa", 4, 1, 32, (0,), 1, io="f32")
    pos = np.array([4 * 32 * sc2.max_pages + 3], np.int64)  # entry 32 * max_pages
    rc = L.state_append_host(0, 1, 4, C, 1, R, ctypes.c_double(BASE), 1, N_WIN, sc2.n_pages, 32,
                             sc2.max_pages, ctypes.c_float(EPS), _np_ptr(pos),
                             *[_np_ptr(sc2.step_rows(k, 0)) for k in ("Ca", "Cb", "Za", "Zb", "win")],
                             _np_ptr(sc2.inp["bias"]), None, _np_ptr(sc2.state), _np_ptr(sc2.ring),
                             _np_ptr(sc2.pages), _np_ptr(sc2.page_table), _np_ptr(status))
    assert rc == 0 and status[0] == -2


# ---------------------------------------------------------------------------
# the library's kernel (GPU)
# ---------------------------------------------------------------------------


def _run_gpu(sc: Scenario):
    import torch
    import long_context_sparse_08_b200 as csa

    dev = "cuda"
    torch.cuda.synchronize()
    csa.device_error()  # start from a clear error word

    def up(x):
        a = np.ascontiguousarray(x)
        t = torch.from_numpy(a.view(np.int16) if sc.io == "bf16" else a)
        return t.to(dev)

    p = csa.make_params(m=sc.m, overlap=sc.overlap, c=C, rope_dims=R, rope_base=BASE,
                        rms_eps=EPS, n_win=N_WIN)
    io = csa.CSA_BF16 if sc.io == "bf16" else csa.CSA_F32
    state, ring, pages = up(sc.state), up(sc.ring), up(sc.pages)
    table = torch.from_numpy(sc.page_table).to(dev)
    bias = up(sc.inp["bias"])
    streams = {k: up(sc.inp[k]) for k in sc.inp if k != "bias"}  # [B, n_tok, c]
    starts = torch.from_numpy(sc.starts.astype(np.int64)).to(dev)
    ar = torch.arange(sc.B, device=dev)
    for step in range(sc.appends):
        pos = starts + step
        rows = {k: v[ar, pos].contiguous() for k, v in streams.items()}
        csa.csa_state_append(p, io, sc.B, pos, rows["Ca"], rows.get("Cb"), rows["Za"],
                             rows.get("Zb"), rows["win"], bias, None, 1, state, ring, pages,
                             sc.n_pages, sc.page_rows, table, sc.max_pages)
    torch.cuda.synchronize()
    assert csa.device_error() == 0

    def down(t):
        a = t.cpu().numpy()
        return a.view(np.uint16) if sc.io == "bf16" else a

    return down(pages), down(ring), down(state)


@pytest.mark.gpu
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gpu_state_append_matches_the_oracle(case, io):
    sc = Scenario(*case, io=io)
    sc.check(*_run_gpu(sc), what=f"gpu {case[0]} {io}")


@pytest.mark.gpu
def test_gpu_appends_equal_the_whole_chunk_compression():
    """Token-by-token appends into identity pages give the cache csa_compress writes for the
    whole 512-token chunk (same arithmetic, so equal to within one bf16 rounding)."""
    import torch
    import long_context_sparse_08_b200 as csa

    sc = Scenario("csa", 4, 1, 32, (0, 0), 512, io="bf16", seed=77)
    sc.max_pages = 4
    sc.n_pages = 8
    sc.page_table = np.arange(8, dtype=np.int32).reshape(2, 4)
    sc.pages = np.zeros((8, 32, C), np.uint16)
    pages, _, _ = _run_gpu(sc)
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
    pages, _, state = _run_gpu_raw(sc)
    assert csa.device_error() == 303
    assert np.array_equal(state[:2], before[:2])  # skipped requests stored nothing
    own = sc.page_table[2, 0]
    assert np.abs(pages[own, 0]).sum() > 0
    rest = pages.copy()
    rest[own, 0] = 0
    assert not rest.any()


def _run_gpu_raw(sc):
    """One append step without the error-word check (the caller reads it)."""
    import torch
    import long_context_sparse_08_b200 as csa

    torch.cuda.synchronize()
    csa.device_error()  # start from a clear error word
    p = csa.make_params(m=sc.m, overlap=sc.overlap, c=C, rope_dims=R, rope_base=BASE,
                        rms_eps=EPS, n_win=N_WIN)
    up = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()  # noqa: E731
    state, ring, pages = up(sc.state), up(sc.ring), up(sc.pages)
    pos = up(sc.starts.astype(np.int64))
    rows = {k: up(sc.step_rows(k, 0)) for k in sc.inp if k != "bias"}
    csa.csa_state_append(p, csa.CSA_F32, sc.B, pos, rows["Ca"], rows["Cb"], rows["Za"],
                         rows["Zb"], rows["win"], up(sc.inp["bias"]), None, 1, state, ring, pages,
                         sc.n_pages, sc.page_rows, up(sc.page_table), sc.max_pages)
    torch.cuda.synchronize()
    return pages.cpu().numpy(), ring.cpu().numpy(), state.cpu().numpy()
