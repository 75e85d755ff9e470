"""Grouped output projection (csa_grouped_out_proj) against the float64 oracle.

The CPU tests run the kernels' arithmetic (csrc/out_proj.cuh: split geometry, index
functions, order of the sums) built for the host by tests/host_check/out_proj_host.cu; the
`gpu` tests run the library's kernels through the C ABI, on reduced shapes and on the
Flash / Pro decode shapes (sampled output columns). The fp32 sums and the single rounding
to bf16 allow half a bf16 ulp plus 1e-4 of the row's RMS per element.
"""
import ctypes
import functools
import os
import subprocess

import numpy as np
import pytest

from oracle import csa_oracle as O
from long_context_sparse_08_b200 import workloads as W
import tests.parity_util as U

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (Q, H, c, g, d_g, d): odd sizes, a reduced model-like shape, the 16-query path
SMALL = [(3, 8, 64, 2, 96, 136), (4, 16, 512, 4, 256, 1000), (16, 8, 64, 4, 64, 72),
         (1, 4, 128, 1, 8, 8)]
# decode shapes of the model table: Flash (Q = 8 requests) and Pro (Q = 4)
FULL = [(8, 64, 512, 8, 1024, 4096), (4, 128, 512, 16, 1024, 7168)]


@functools.lru_cache(maxsize=1)
def host_lib():
    out = os.path.join(ROOT, "tests", "host_check", "_build")
    os.makedirs(out, exist_ok=True)
    so = os.path.join(out, "libout_proj_host.so")
    src = os.path.join(ROOT, "tests", "host_check", "out_proj_host.cu")
    hdr = os.path.join(ROOT, "long_context_sparse_08_b200", "csrc", "out_proj.cuh")
    if not os.path.exists(so) or os.path.getmtime(so) < max(os.path.getmtime(src),
                                                            os.path.getmtime(hdr)):
        subprocess.run(["nvcc", "-O2", "-shared", "-Xcompiler", "-fPIC", "-arch=sm_100a",
                        "-I", os.path.join(ROOT, "include"),
                        "-I", os.path.join(ROOT, "long_context_sparse_08_b200", "csrc"),
                        src, "-o", so], check=True, capture_output=True)
    L = ctypes.CDLL(so)
    L.out_proj_host.restype = ctypes.c_int
    return L


def _p(H, c):
    import long_context_sparse_08_b200 as csa

    return csa.make_params(c=c, n_heads=H, rope_dims=min(64, c))


def _oracle(inp, Q, H, c, g, d_g, d, cols=None):
    """Oracle outputs [Q, len(cols)] (all columns by default): the oracle's projection with
    the sampled columns of w_out (decoded once; float64)."""
    w_grp = O.dec_bf16(inp["w_grp"])
    w_out = O.dec_bf16(inp["w_out"] if cols is None else inp["w_out"][:, cols])
    return np.stack([O.grouped_output_projection(O.dec_bf16(inp["o"][q]).reshape(H, c), w_grp,
                                                 w_out) for q in range(Q)])


def _check(got_bits, ref, what):
    got = O.dec_bf16(got_bits)
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    lim = 0.5 * U.bf16_ulp(ref) * 1.01 + 1e-4 * rms
    bad = np.abs(got - ref) > lim
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} values off " \
                          f"(max err {np.abs(got - ref).max():.3e})"


@pytest.mark.parametrize("shape", SMALL, ids=[str(s) for s in SMALL])
@pytest.mark.parametrize("sms", [148, 5])
def test_host_build_matches_the_oracle(shape, sms):
    Q, H, c, g, d_g, d = shape
    inp = W.make_out_proj_inputs(Q=Q, H=H, c=c, g=g, d_g=d_g, d=d, seed=sum(shape))
    out = np.zeros((Q, d), np.uint16)
    geom = np.zeros(4, np.int32)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    rc = host_lib().out_proj_host(Q, H, c, g, d_g, d, sms, ptr(inp["o"]), ptr(inp["w_grp"]),
                                  ptr(inp["w_out"]), ptr(out), ptr(geom))
    assert rc == 0, f"index outside a buffer ({rc})"
    S1, S2, ks1, ks2 = geom.tolist()
    assert S1 * ks1 >= c * H // g > (S1 - 1) * ks1 and ks1 <= 512
    assert S2 * ks2 >= g * d_g > (S2 - 1) * ks2 and ks2 <= 512
    _check(out, _oracle(inp, Q, H, c, g, d_g, d), f"host {shape} sms={sms}")


@pytest.mark.parametrize("shape", FULL, ids=["flash_decode", "pro_decode"])
def test_host_build_on_the_decode_shapes_sampled(shape):
    # the model's decode shapes with the B200's 148 SMs: every column computed by the host
    # build, sampled columns against the oracle
    Q, H, c, g, d_g, d = shape
    inp = W.make_out_proj_inputs(Q=Q, H=H, c=c, g=g, d_g=d_g, d=d, seed=7)
    out = np.zeros((Q, d), np.uint16)
    geom = np.zeros(4, np.int32)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    rc = host_lib().out_proj_host(Q, H, c, g, d_g, d, 148, ptr(inp["o"]), ptr(inp["w_grp"]),
                                  ptr(inp["w_out"]), ptr(out), ptr(geom))
    assert rc == 0, f"index outside a buffer ({rc})"
    cols = np.unique(np.concatenate([np.arange(0, d, 97), [d - 1]]))
    _check(out[:, cols], _oracle(inp, Q, H, c, g, d_g, d, cols=cols), f"host {shape} sampled")


def test_checks_on_the_host():
    import long_context_sparse_08_b200 as csa

    L = csa.lib()
    F = 0x10000
    p = _p(128, 512)
    args = lambda Q, g, dg, d: (ctypes.byref(p), Q, g, dg, d, F, F, F, F, F, 1 << 30, None)  # noqa
    # the tensor-core form (Q >= 128) needs g * d_g a multiple of 64 and d_g >= 64
    assert L.csa_grouped_out_proj(*args(128, 1, 8, 7168)) == csa.CSA_ERR_UNSUPPORTED
    assert L.csa_grouped_out_proj(*args(128, 16, 8, 7168)) == csa.CSA_ERR_UNSUPPORTED
    assert L.csa_grouped_out_proj(*args(4, 16, 1024, 7100 + 1)) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_grouped_out_proj(*args(4, 48, 1024, 7168)) == csa.CSA_ERR_INVALID_ARG
    assert L.csa_grouped_out_proj(*args(0, 16, 1024, 7168)) == csa.CSA_OK
    a = list(args(4, 16, 1024, 7168))
    a[5] = None
    assert L.csa_grouped_out_proj(*a) == csa.CSA_ERR_INVALID_ARG
    need = csa.grouped_out_proj_workspace_size(p, 4, 16, 1024, 7168)
    assert need >= (4 * 16 * 1024 + 4 * 7168) * 4
    # larger decode batches run 16 queries per pass in the same workspace; prefill keeps the
    # bf16 intermediate
    assert csa.grouped_out_proj_workspace_size(p, 100, 16, 1024, 7168) == \
        csa.grouped_out_proj_workspace_size(p, 16, 16, 1024, 7168)
    assert csa.grouped_out_proj_workspace_size(p, 4096, 16, 1024, 7168) == \
        4096 * 16 * 1024 * 2 + 256
    a = list(args(4, 16, 1024, 7168))
    a[10] = need - 1
    assert L.csa_grouped_out_proj(*a) == csa.CSA_ERR_WORKSPACE
    # every operand 16-byte aligned (weights are read 16 bytes at a time)
    for i in (5, 6, 7, 8):
        for q in (4, 128):
            a = list(args(q, 16, 1024, 7168))
            a[i] = F + 8
            assert L.csa_grouped_out_proj(*a) == csa.CSA_ERR_INVALID_ARG, (i, q)


# ---------------------------------------------------------------------------
# the library's kernels (GPU)
# ---------------------------------------------------------------------------


def _run_gpu(inp, Q, H, c, g, d_g, d):
    import torch
    import long_context_sparse_08_b200 as csa

    p = _p(H, c)
    dev = {k: torch.from_numpy(v.view(np.int16)).cuda() for k, v in inp.items()}
    out = torch.zeros((Q, d), dtype=torch.int16, device="cuda")
    need = csa.grouped_out_proj_workspace_size(p, Q, g, d_g, d)
    ws = torch.empty((need,), dtype=torch.uint8, device="cuda")
    csa.csa_grouped_out_proj(p, Q, g, d_g, d, dev["o"], dev["w_grp"], dev["w_out"], out, ws,
                             need)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16)


@pytest.mark.gpu
@pytest.mark.parametrize("shape", SMALL, ids=[str(s) for s in SMALL])
def test_gpu_matches_the_oracle(shape):
    Q, H, c, g, d_g, d = shape
    inp = W.make_out_proj_inputs(Q=Q, H=H, c=c, g=g, d_g=d_g, d=d, seed=sum(shape))
    _check(_run_gpu(inp, *shape), _oracle(inp, *shape), f"gpu {shape}")


@pytest.mark.gpu
@pytest.mark.parametrize("shape", FULL, ids=["flash_decode", "pro_decode"])
def test_gpu_decode_shapes_sampled(shape):
    Q, H, c, g, d_g, d = shape
    inp = W.make_out_proj_inputs(Q=Q, H=H, c=c, g=g, d_g=d_g, d=d, seed=7)
    got = _run_gpu(inp, *shape)
    cols = np.unique(np.concatenate([np.arange(0, d, 97), [d - 1]]))
    _check(got[:, cols], _oracle(inp, *shape, cols=cols), f"gpu {shape} sampled")


@pytest.mark.gpu
def test_gpu_decode_batch_of_forty_queries():
    # 40 queries: three passes of the weight-streaming kernels (16 + 16 + 8)
    shape = (40, 8, 64, 2, 96, 136)
    Q, H, c, g, d_g, d = shape
    inp = W.make_out_proj_inputs(Q=Q, H=H, c=c, g=g, d_g=d_g, d=d, seed=40)
    _check(_run_gpu(inp, *shape), _oracle(inp, *shape), f"gpu {shape}")


# prefill (tensor-core GEMMs)
PREFILL = [(128, 8, 64, 2, 64, 128), (1000, 64, 512, 8, 1024, 4096)]


@pytest.mark.gpu
@pytest.mark.parametrize("shape", PREFILL, ids=["small", "flash_1000_queries"])
def test_gpu_prefill_gemm_sampled(shape):
    Q, H, c, g, d_g, d = shape
    inp = W.make_out_proj_inputs(Q=Q, H=H, c=c, g=g, d_g=d_g, d=d, seed=8)
    got = _run_gpu(inp, *shape)
    import long_context_sparse_08_b200 as csa

    assert csa.device_error() == 0
    qs = np.unique(np.concatenate([np.arange(0, Q, 61), [Q - 1]]))
    cols = np.unique(np.concatenate([np.arange(0, d, 37), [d - 1]]))
    sub = dict(inp, o=inp["o"][qs])
    ref = _oracle(sub, len(qs), H, c, g, d_g, d, cols=cols)
    # the bf16 intermediate adds a rounding: the bf16 output tolerance applies
    for i, q in enumerate(qs):
        U.check_out(O.dec_bf16(got[q, cols]), ref[i], "bf16", f"prefill {shape} q={q}")

