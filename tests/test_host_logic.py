"""Host-side arithmetic behind the bench line and the FP8 tensor-core path, on CPU.

- Algorithmic bytes per decode query and the prefill flop count, against the closed forms
  built from the workload shapes (keys scanned x bytes per key, rows attended x row bytes,
  visible (t, s) pairs x 2 H_I d_I flops, attended rows x 4 c H flops).
- Every OCP e4m3 code is exactly a bf16 value: the FP8 indexer widens codes to bf16 for the
  tensor cores, which is exact only because of this.
"""
import importlib.util
import os

import numpy as np
import pytest
import torch

from long_context_sparse_08_b200 import workloads as W
from oracle import csa_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,expected", [
    # keys x (FP8 row 128 B + fp32 scale) + (k + window) x 1 KB rows + q + qI + w + out
    ("flash_decode_131k", 32768 * 132 + 640 * 1024 + 65536 + 16384 + 256 + 65536),
    # keys x (64 B e2m1 + 4 B e8m0) + 1152 rows + q (128 heads) + MXFP4 qI + w + out
    ("pro_decode_1m", 262144 * 68 + 1152 * 1024 + 131072 + 4352 + 256 + 131072),
    # every visible entry and the window, q and out (64 heads)
    ("hca_decode_1m", 8320 * 1024 + 65536 + 65536),
])
def test_algorithmic_bytes_per_query(bench, name, expected):
    s = W.SHAPES[name]
    n_vis = min(s.ctx // s.m, s.n_cap)
    assert bench.algorithmic_bytes_per_query(s, n_vis)["total"] == expected


def test_prefill_flops(bench):
    s = W.SHAPES["flash_prefill_8k"]
    fl = bench.prefill_flops(s)
    # visible (t, s) pairs of queries 57344 .. 65535 at m = 4, N_cap = 16384
    pairs = sum(min((57344 + i) // 4, 16384) for i in range(8192))
    assert pairs == 125_825_024
    assert fl["index"] == 2 * 64 * 128 * pairs
    # every query attends k = 512 selected rows and a full 128-token window
    assert fl["attention"] == 8192 * 64 * 640 * 512 * 4
    assert fl["total"] == fl["index"] + fl["attention"]


def test_every_e4m3_code_is_a_bf16_value():
    codes = np.arange(256, dtype=np.uint8)
    vals = O.dec_e4m3(codes)  # float64, NaN for the two NaN codes
    finite = np.isfinite(vals)
    as_bf16 = torch.from_numpy(vals[finite]).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(as_bf16, vals[finite])


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the oracle on the host cores) prints one JSON line with
    the keys the bench contract names, on the configuration the GPU arm uses."""
    import json
    import subprocess
    import sys

    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_prefill_f32", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, cwd=ROOT, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 1
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["config"]["workload"] == "tiny_prefill_f32"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_extension_bytes(bench):
    # grouped projection, Pro decode: 16 groups of 4096 x 1024 and 16384 x 7168 bf16 weights,
    # 4 queries of 128 x 512 bf16 in, 7168 bf16 out
    assert bench.out_proj_bytes(4, 128, 512, 16, 1024, 7168) == \
        2 * (16 * 4096 * 1024 + 16384 * 7168) + 2 * 4 * 128 * 512 + 2 * 4 * 7168
    # one CSA append, c = 512: 4 raw rows read and stored, the window row read and stored;
    # every 4th token reads back 4 x 4 rows and writes one entry
    kv = 2 * 512 * (4 + 4 + 1 + 1) + (16 * 512 * 2 + 512 * 2) // 4
    keys = 2 * 128 * (4 + 4) + (16 * 128 * 2 + 68) // 4
    assert bench.state_append_bytes(512, 4, 1) == {"kv": kv, "keys": keys, "total": kv + keys}


def test_parts_refuse_workloads_they_cannot_run(bench):
    # the checks run before any GPU work, so they can be exercised here
    for part in ("bf16_scores", "forward_paged"):
        bench.check_part_workload(part, W.SHAPES["flash_decode_131k"])
        bench.check_part_workload(part, W.SHAPES["pro_decode_1m"])
    with pytest.raises(SystemExit, match="MXFP4, FP8 or bf16 indexer keys"):
        bench.check_part_workload("bf16_scores", W.SHAPES["hca_decode_1m"])
    bench.check_part_workload("forward_paged", W.SHAPES["hca_decode_1m"])  # the HCA layer
    with pytest.raises(SystemExit, match="a CSA or HCA decode step"):
        bench.check_part_workload("forward_paged", W.SHAPES["flash_prefill_8k"])
    bench.check_part_workload("bf16_scores", W.SHAPES["flash_prefill_8k"])
    with pytest.raises(SystemExit, match="a CSA or HCA decode step"):
        bench.check_part_workload("kv_layouts", W.SHAPES["flash_prefill_8k"])
    bench.check_part_workload("kv_layouts", W.SHAPES["hca_decode_1m"])
    bench.check_part_workload("out_proj", W.SHAPES["pro_decode_1m"])
