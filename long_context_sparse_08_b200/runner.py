"""One step of the hot path on a workload: upload its arrays and call the C ABI.

A step is the whole hot path over one batch:
  CSA decode   -> csa_forward (index scores -> top-k -> sparse MQA)
  CSA prefill  -> csa_forward with the chunk's compression first
  HCA decode   -> hca_dense_mqa
Everything here is argument marshalling: torch allocates device memory (inputs, outputs,
workspace) and the library's kernels do all the work.
"""
from __future__ import annotations

from typing import Dict

import numpy as np
import torch

from . import (CSA_BF16, CSA_F32, CSA_WS_FORWARD, CSA_WS_HCA_MQA, DTYPES, csa_forward,
               forward_args, hca_dense_mqa, make_params, workspace_size)

_BF16_KEYS = {"q", "kv_cache", "win_kv", "Ca", "Cb", "Za", "Zb", "bias", "prev_Cb", "prev_Zb"}


def to_torch(name: str, x: np.ndarray, io: str, idx: str) -> torch.Tensor:
    """Host tensor with the dtype the library expects for input `name`."""
    t = torch.from_numpy(np.ascontiguousarray(x))
    if x.dtype == np.uint16:  # bf16 bit patterns
        return t.view(torch.bfloat16)
    return t


def upload(inp: Dict[str, np.ndarray], s, device="cuda") -> Dict[str, torch.Tensor]:
    out = {}
    for k, v in inp.items():
        if k in ("KI_f32", "qI_f32"):
            continue
        out[k] = to_torch(k, v, s.io, s.idx).to(device)
    return out


def params_for(s):
    return make_params(m=s.m, overlap=s.overlap, c=s.c, rope_dims=s.rope_dims,
                       rope_base=s.rope_base, rms_eps=s.rms_eps, sm_scale=1.0 / np.sqrt(s.c),
                       n_heads=s.n_heads, n_idx_heads=max(s.n_idx_heads, 1),
                       d_idx=max(s.d_idx, 32), topk=max(s.topk, 1), n_win=s.n_win)


class Step:
    """Device buffers of one workload and the call that runs its hot path once."""

    def __init__(self, s, dev: Dict[str, torch.Tensor], want_scores: bool = False):
        self.s = s
        self.dev = dev
        self.p = params_for(s)
        self.io = CSA_BF16 if s.io == "bf16" else CSA_F32
        d = dev["q"].device
        odt = torch.bfloat16 if s.io == "bf16" else torch.float32
        B, T = s.B, s.T
        self.out = torch.empty((B, T, s.n_heads, s.c), dtype=odt, device=d)
        if s.kind == "hca_decode":
            self.ws_bytes = workspace_size(self.p, CSA_WS_HCA_MQA, 0, B, T, s.n_cap)
            self.out_idx = None
            self.scores = None
        else:
            self.kdt = DTYPES[s.idx]
            self.ws_bytes = workspace_size(self.p, CSA_WS_FORWARD, self.kdt, B, T, s.n_cap)
            self.out_idx = torch.empty((B, T, s.topk), dtype=torch.int32, device=d)
            self.scores = (torch.empty((B, T, s.n_cap), dtype=torch.float32, device=d)
                           if want_scores else None)
        self.ws = torch.empty((max(self.ws_bytes, 1),), dtype=torch.uint8, device=d)
        if s.kind != "hca_decode":
            self.args = self._forward_args()

    def _forward_args(self):
        s, D = self.s, self.dev
        kw = dict(idx_dtype=self.kdt, qI=D["qI"], qI_scale=D.get("qI_scale"), w=D["w"],
                  KI=D["KI"], KI_scale=D.get("KI_scale"), q=D["q"], q_pos=D["q_pos"],
                  kv_cache=D["kv_cache"], N_cap=s.n_cap, win_kv=D["win_kv"],
                  L_raw=D["win_kv"].shape[1], win_pos0=D["win_pos0"], sink=D["sink"],
                  out_idx=self.out_idx, out_scores=self.scores, out=self.out)
        if s.kind == "csa_prefill":
            kw.update(n_tok=s.n_tok, first_entry=s.ctx // s.m, Ca=D["Ca"], Cb=D["Cb"],
                      Za=D["Za"], Zb=D["Zb"], bias=D["bias"], prev_Cb=D.get("prev_Cb"),
                      prev_Zb=D.get("prev_Zb"))
        return forward_args(**kw)

    def __call__(self, stream=None):
        s, D = self.s, self.dev
        if s.kind == "hca_decode":
            hca_dense_mqa(self.p, self.io, s.B, s.T, D["q"], D["q_pos"], D["kv_cache"], s.n_cap,
                          D["win_kv"], D["win_kv"].shape[1], D["win_pos0"], D["sink"], None,
                          self.out, self.ws, self.ws_bytes, stream)
        else:
            csa_forward(self.p, self.io, s.B, s.T, self.args, self.ws, self.ws_bytes, stream)
        return self.out
