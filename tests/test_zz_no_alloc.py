"""csa_topk_noalloc (top-k with the library's own scratch array) against csa_topk with caller
scratch: identical indices on two calls in a row, for shapes that take the many-slice
selector (which needs scratch) and the one-CTA-per-row selector (which needs none), and the
size limit of the array is enforced. The file is named to be collected last, so that it
also runs after every other test has used the device."""
import numpy as np
import pytest
import torch

import long_context_sparse_08_b200 as csa

pytestmark = pytest.mark.gpu

# (B, T, N_cap, k): 4 x 262144 with k = 1024 is the 1M-context decode shape (about 8.5 MB of
# scratch); 8 x 32768 with k = 512 the 128K one; the last two need no scratch.
CASES = [(4, 1, 262144, 1024), (8, 1, 32768, 512), (2, 3, 9000, 2000), (3, 40, 700, 64)]


def _inputs(B, T, N, k, seed):
    g = np.random.default_rng(seed)
    sc = np.round(g.standard_normal((B, T, N)).astype(np.float32) * 4, 1)  # many exact ties
    sc[0, 0, : min(N, 300)] = -0.0
    # ragged visibility (m = 4): fewer than k visible, about half, all, and past N_cap
    pos = g.integers(0, 4 * N + 8, size=(B, T)).astype(np.int64)
    pos.flat[0] = 4 * (k // 2)
    pos.flat[-1] = 4 * N + 3
    return torch.from_numpy(sc).cuda(), torch.from_numpy(pos).cuda()


def _with_caller_scratch(p, B, T, N, sc, pos, k):
    ws_bytes = csa.workspace_size(p, csa.CSA_WS_TOPK, 0, B, T, N)
    ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device="cuda")
    out = torch.empty((B, T, k), dtype=torch.int32, device="cuda")
    csa.csa_topk(p, B, T, N, sc, pos, out, ws, ws_bytes)
    return out, ws_bytes


@pytest.mark.parametrize("B,T,N,k", CASES)
def test_noalloc_topk_matches_caller_scratch(B, T, N, k):
    p = csa.make_params(topk=k)
    sc, pos = _inputs(B, T, N, k, 300 + k)
    ref, ws_bytes = _with_caller_scratch(p, B, T, N, sc, pos, k)
    assert ws_bytes <= csa.TOPK_NOALLOC_SCRATCH_BYTES
    for call in range(2):  # the shared array is reused: its counters must restart at zero
        out = torch.full((B, T, k), -7, dtype=torch.int32, device="cuda")
        csa.csa_topk_noalloc(p, B, T, N, sc, pos, out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {call}: indices differ from csa_topk"
    assert csa.device_error() == 0


def test_noalloc_topk_interleaved_shapes():
    # a call of another shape in between leaves stale counters and lists behind it
    (B1, T1, N1, k1), (B2, T2, N2, k2) = CASES[0], CASES[1]
    p1, p2 = csa.make_params(topk=k1), csa.make_params(topk=k2)
    sc1, pos1 = _inputs(B1, T1, N1, k1, 41)
    sc2, pos2 = _inputs(B2, T2, N2, k2, 42)
    ref1, _ = _with_caller_scratch(p1, B1, T1, N1, sc1, pos1, k1)
    ref2, _ = _with_caller_scratch(p2, B2, T2, N2, sc2, pos2, k2)
    o1 = torch.empty_like(ref1)
    o2 = torch.empty_like(ref2)
    for _ in range(2):
        csa.csa_topk_noalloc(p1, B1, T1, N1, sc1, pos1, o1)
        csa.csa_topk_noalloc(p2, B2, T2, N2, sc2, pos2, o2)
        torch.cuda.synchronize()
        assert torch.equal(o1, ref1) and torch.equal(o2, ref2)


def test_noalloc_topk_rejects_sizes_beyond_the_array():
    B, T, N, k = 64, 1, 65536, 1024  # 64 rows x 65536 candidates x 8 B of lists alone: 32 MB
    p = csa.make_params(topk=k)
    assert csa.workspace_size(p, csa.CSA_WS_TOPK, 0, B, T, N) > csa.TOPK_NOALLOC_SCRATCH_BYTES
    sc = torch.zeros((B, T, N), dtype=torch.float32, device="cuda")
    pos = torch.full((B, T), 4 * N, dtype=torch.int64, device="cuda")
    out = torch.full((B, T, k), -7, dtype=torch.int32, device="cuda")
    with pytest.raises(csa.CsaError) as e:
        csa.csa_topk_noalloc(p, B, T, N, sc, pos, out)
    assert e.value.status == csa.CSA_ERR_WORKSPACE
    assert "scratch" in str(e.value)
    torch.cuda.synchronize()
    assert int((out != -7).sum()) == 0  # nothing was launched
