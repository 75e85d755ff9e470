"""Pure sliding-window attention (the first two layers of the Flash model, 【论文解读】
DeepSeek-V4 三(二) 模型配置; the window of 一(三)3(3) with the sink of 3(4) and no compressed
entries) is hca_dense_mqa with N_cap = 0: every query attends only its n_win most recent
tokens. Checked against the oracle's HCA query with no visible entry, at positions before,
at and past the first full window.
An empty cache with a NULL KV pointer takes the attention's window-only path for every
request.
"""
import math

import numpy as np
import pytest

from oracle import csa_oracle as O
from long_context_sparse_08_b200 import workloads as W
import tests.parity_util as U

pytestmark = [
    pytest.mark.gpu,
]

H, C, R, N_WIN, BASE, EPS = 64, 512, 64, 128, 10000.0, 1e-6


def test_window_only_attention():
    import torch
    import long_context_sparse_08_b200 as csa

    pos = np.array([[0], [5], [127], [128], [5000]], np.int64)
    B = pos.shape[0]
    g = np.random.default_rng(31)
    q = W.f32_to_bf16_bits(g.standard_normal((B, 1, H, C), np.float32))
    win = W.f32_to_bf16_bits(g.standard_normal((B, N_WIN, C), np.float32))
    pos0 = np.maximum(pos[:, 0] - N_WIN + 1, 0).astype(np.int64)
    sink = g.standard_normal((H,), np.float32)
    up = lambda a: torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).cuda()  # noqa
    p = csa.make_params(m=128, overlap=0, c=C, rope_dims=R, rope_base=BASE, rms_eps=EPS,
                        n_heads=H, n_win=N_WIN)
    need = csa.workspace_size(p, csa.CSA_WS_HCA_MQA, 0, B, 1, 0)
    ws = torch.empty((max(need, 1),), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, 1, H, C), dtype=torch.int16, device="cuda")
    torch.cuda.synchronize()
    csa.device_error()
    csa.hca_dense_mqa(p, csa.CSA_BF16, B, 1, up(q), up(pos), None, 0, up(win), N_WIN, up(pos0),
                      up(sink), None, out, ws, need)
    torch.cuda.synchronize()
    assert csa.device_error() == 0
    got = O.dec_bf16(out.cpu().numpy().view(np.uint16))
    for b in range(B):
        t = int(pos[b, 0])
        want = O.hca_query(O.dec_bf16(q[b, 0]), t, np.zeros((0, C)), 0, O.dec_bf16(win[b]),
                           int(pos0[b]), sink, r=R, base=BASE, eps=EPS,
                           scale=1.0 / math.sqrt(C), n_win=N_WIN)
        U.check_out(got[b, 0], want, "bf16", f"window-only request {b} (t = {t})")
