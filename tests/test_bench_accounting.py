"""The benchmark's accounting on CPU: algorithmic work per workload and the profile lookup.

* the chunk form's tensor-core FLOPs per token and value head, 6 Dk Dv + 2 C (3 Dk + 2 Dv)
  (180,224 for D = 128 and C = 64, the figure the roofline uses);
* the prefill's algorithmic HBM bytes, counted term by term here (q, k, v, out in the
  activations' type, g and beta in fp32 -- g with Dk values per token and head in the
  per-key-dimension spelling --, states in fp32, cu_seqlens);
* the DRAM traffic read from a committed ncu summary only while the kernel source, with the csrc
  headers it includes, still has the digest the summary records;
* the oracle arm (`--impl reference`) printing one line with the contract's keys, its warm-up
  steps run untimed.
"""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    sys.path.insert(0, ROOT)
    import bench as b
    return b


def test_flops_per_token_head(bench):
    assert bench.prefill_flops_per_token_head(128, 128) == 180224
    Dk, Dv, C = 64, 32, 64
    assert bench.prefill_flops_per_token_head(Dk, Dv) == 6 * Dk * Dv + 2 * C * (3 * Dk + 2 * Dv)


@pytest.mark.parametrize("per_key", [False, True])
def test_prefill_bytes(bench, per_key):
    from gated_deltanet_state_gdn_b200 import workloads as W
    lengths = [5, 0, 70]
    Hq, Hv, Dk, Dv = 2, 4, 32, 16
    c = W.make_prefill(3, lengths, Hq, Hv, Dk, Dv, init_std=0.02, decay_per_key=per_key)
    N, B = sum(lengths), len(lengths)
    qkvo = N * (2 * Hq * Dk + 2 * Hv * Dv) * 2          # bf16
    g = N * Hv * (Dk if per_key else 1) * 4
    beta = N * Hv * 4
    states = 2 * B * Hv * Dv * Dk * 4                    # initial and final
    cu = (B + 1) * 4
    assert bench.prefill_bytes(c) == qkvo + g + beta + states + cu


def test_profile_traffic_follows_the_source_hash(bench):
    # the committed summaries carry the hash of the source they were captured on
    t = bench.ncu_traffic("prefill_kd_ragged_per_key.md", "prefill_kd.cu")
    assert t is None or t > 0
    # a different source file never matches a summary's hash
    assert bench.ncu_traffic("prefill_kd_ragged_per_key.md", "decode.cu") is None
    assert bench.ncu_traffic("no_such_profile.md", "prefill_kd.cu") is None


def test_source_digest_covers_included_headers(bench):
    import hashlib
    csrc = os.path.join(ROOT, "gated_deltanet_state_gdn_b200", "csrc")

    def raw(name):
        return open(os.path.join(csrc, name), "rb").read()

    # prefill_kd.cu includes common.cuh, sm100.cuh and tile16.cuh (which includes the first two
    # again); each header enters the digest once, depth first, after the file that includes it
    want = hashlib.sha256(raw("prefill_kd.cu") + raw("common.cuh") + raw("sm100.cuh")
                          + raw("tile16.cuh")).hexdigest()[:16]
    assert bench.source_digest("prefill_kd.cu") == want
    assert bench.source_digest("prefill_kd.cu") != hashlib.sha256(raw("prefill_kd.cu")).hexdigest()[:16]
    assert bench.source_digest("no_such_kernel.cu") is None


def test_profile_traffic_keys(bench):
    # the long-context summary records DRAM bytes per call (three launches), not per launch
    assert bench.ncu_traffic("prefill_chunk_long_split.md", "prefill_chunk.cu") is None
    t = bench.ncu_traffic("prefill_chunk_long_split.md", "prefill_chunk.cu", "traffic_bytes_per_call")
    assert t is None or t > 0


def test_reference_arm_prints_one_contract_line():
    # the oracle arm runs on the host cores alone: W untimed and K timed steps, one JSON line
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "3"], cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["runs"] == 2 and d["cpu_baseline"]["warmup_runs"] == 3
