"""The benchmark's accounting on CPU: algorithmic work per workload and the profile lookup.

* the chunk form's tensor-core FLOPs per token and value head, 6 Dk Dv + 2 C (3 Dk + 2 Dv)
  (180,224 for D = 128 and C = 64, the figure the roofline uses);
* the prefill's algorithmic HBM bytes, counted term by term here (q, k, v, out in the
  activations' type, g and beta in fp32 -- g with Dk values per token and head in the
  per-key-dimension spelling --, states in fp32, cu_seqlens);
* the DRAM traffic read from a committed ncu summary only while the kernel source, with the csrc
  headers it includes, still has the digest the summary records.
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
