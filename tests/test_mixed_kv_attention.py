"""Attention over a mixed-precision KV cache (csa_sparse_mqa_mixed_kv, hca_dense_mqa_mixed_kv)
against the float64 oracle on the same bytes.

The workloads' bf16 caches are re-encoded by the input encoder as mixed rows (the first
c - r values as e4m3 with a row scale, the RoPE values as bf16); the oracle decodes those
bytes exactly, and the kernel widens code * scale to bf16 before its tensor-core products.
The outputs must meet the bf16 output tolerance.

These kernels have not yet run on a B200: the module runs only with
CSA_RUN_FIRST_GPU_CHECKS=1, so a first run is a deliberate, separate step.
"""
import os

import numpy as np
import pytest
import torch

import long_context_sparse_08_b200 as csa
from long_context_sparse_08_b200 import runner as R
from long_context_sparse_08_b200 import workloads as W
from oracle import pipeline as P
import tests.parity_util as U

pytestmark = [
    pytest.mark.gpu,
    pytest.mark.skipif(os.environ.get("CSA_RUN_FIRST_GPU_CHECKS") != "1",
                       reason="awaiting its first run on a B200 (CSA_RUN_FIRST_GPU_CHECKS=1)"),
]


def _mixed(name):
    s, inp = U.inputs(name)
    kv = W.bf16_bits_to_f32(inp["kv_cache"])
    codes, scale, rope = W.quant_mixed_kv(kv, s.rope_dims)
    rows = np.concatenate([codes, rope.view(np.uint8)], axis=-1)  # c + r bytes per row
    inp2 = {k: v for k, v in inp.items() if k != "kv_cache"}
    inp2.update(kv_codes=codes, kv_scale=scale, kv_rope=rope)
    return s, inp, inp2, torch.from_numpy(np.ascontiguousarray(rows)).cuda(), \
        torch.from_numpy(scale).cuda()


@pytest.mark.parametrize("name", ["mid_decode_fp8", "mid_decode_mxfp4", "edge_decode_bf16"])
def test_sparse_mqa_over_mixed_rows(name):
    s, inp, inp2, rows, scale = _mixed(name)
    res = P.run(s, inp2, want_scores=False)
    dev = R.upload(inp, s)
    idx = np.full((s.B, s.T, s.topk), -1, np.int32)
    for (b, ti), sel in res["idx"].items():
        idx[b, ti] = sel
    p = R.params_for(s)
    out = torch.empty((s.B, s.T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
    ws_bytes = csa.workspace_size(p, csa.CSA_WS_SPARSE_MQA, 0, s.B, s.T, s.n_cap)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device="cuda")
    csa.csa_sparse_mqa_mixed_kv(p, s.B, s.T, dev["q"], dev["q_pos"], rows, scale, s.n_cap,
                                torch.from_numpy(idx).cuda(), dev["win_kv"],
                                dev["win_kv"].shape[1], dev["win_pos0"], dev["sink"], None, out,
                                ws, ws_bytes)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    got = out.float().cpu().numpy()
    for (b, ti), ref in res["out"].items():
        U.check_out(got[b, ti], ref, "bf16", f"{name} mixed KV b={b} t={ti}")


@pytest.mark.parametrize("name", ["mid_hca_decode", "edge_hca_decode"])
def test_dense_mqa_over_mixed_rows(name):
    s, inp, inp2, rows, scale = _mixed(name)
    res = P.run(s, inp2)
    dev = R.upload(inp, s)
    p = R.params_for(s)
    out = torch.empty((s.B, s.T, s.n_heads, s.c), dtype=dev["q"].dtype, device="cuda")
    ws_bytes = csa.workspace_size(p, csa.CSA_WS_HCA_MQA, 0, s.B, s.T, s.n_cap)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device="cuda")
    csa.hca_dense_mqa_mixed_kv(p, s.B, s.T, dev["q"], dev["q_pos"], rows, scale, s.n_cap,
                               dev["win_kv"], dev["win_kv"].shape[1], dev["win_pos0"],
                               dev["sink"], None, out, ws, ws_bytes)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    got = out.float().cpu().numpy()
    for (b, ti), ref in res["out"].items():
        U.check_out(got[b, ti], ref, "bf16", f"{name} mixed KV b={b}")
