"""Host-side FLOP accounting of bench.py against brute-force counts (CPU)."""

import numpy as np
import pytest

import bench


def _brute_executed(lists, M, d, causal, b=64):
    """Count multiply-adds pair by pair: every visible (query, key) token pair of a
    listed block, and every (query, unlisted candidate block) pseudo-key, at 4 d FLOPs."""
    pairs = 0
    r = 0
    for I in range(M):
        listed = set(lists[r])
        cand = range(I + 1) if causal else range(M)
        for J in cand:
            if J in listed:
                for i in range(b):
                    for j in range(b):
                        if not causal or J < I or j <= i:
                            pairs += 1
            elif not (causal and J == I):
                pairs += b  # one pseudo-key per query of the block
        r += 1
    return 4.0 * d * pairs


@pytest.mark.parametrize("causal", [False, True])
def test_executed_flops_matches_pair_count(causal):
    rng = np.random.default_rng(3)
    M, d = 6, 8
    lists = []
    for I in range(M):
        n = I + 1 if causal else M
        keep = rng.random(n) < 0.5
        if causal:
            keep[I] = True  # the routers always list the causal diagonal
        lists.append(np.nonzero(keep)[0])
    rp = np.concatenate([[0], np.cumsum([len(x) for x in lists])])
    got = bench.executed_flops(rp, None, 1, 1, M, d, causal)
    assert got == _brute_executed(lists, M, d, causal)


def test_issued_flops_counts_tiles():
    # M = 4 non-causal, list sizes 0, 1, 4, 3: tiles 1 (pooled only), 1 + 1,
    # 2 (everything listed: no pooled tile), 1 + 2 -> 8 tiles
    rp = np.array([0, 0, 1, 5, 8])
    per_tile = 2.0 * 128 * 64 * 128 + 2.0 * 128 * 64 * 128
    assert bench.issued_flops(rp, 1, 1, 4, 128, False) == 8 * per_tile
    # dense: every candidate listed, no pooled tiles; causal row I lists I + 1 blocks
    rp_dense = np.concatenate([[0], np.cumsum(np.arange(1, 5))])
    assert bench.issued_flops(rp_dense, 1, 1, 4, 64, True, dense=True) == \
        (1 + 1 + 2 + 2) * (2.0 * 128 * 64 * 64 + 2.0 * 64 * 64 * 128)


def test_dense_flops_formula():
    assert bench.dense_flops(2, 3, 128, 64, False) == 4.0 * 2 * 3 * 128 * 128 * 64
    assert bench.dense_flops(2, 3, 128, 64, True) == 2.0 * 2 * 3 * 128 * 128 * 64


def test_launches_per_step_matches_the_launch_lists():
    # launch lists of one step (pool; route: header, score_tc, selection; attention:
    # header, stats_to_bf16, the sweep, its rerun of flagged blocks, fixup; + scan and
    # compaction for the threshold routers)
    assert bench.launches_per_step(1, 12, 512, "topk", False) == 9
    assert bench.launches_per_step(1, 12, 512, "thresh", False) == 11
    assert bench.launches_per_step(1, 8, 2048, "thresh", False) == 11      # 8 x 16 MB of scores: one batch
    assert bench.launches_per_step(1, 1, 16384, "topk", False) == 9
    assert bench.launches_per_step(1, 2, 16384, "topk", False) == 11       # 1 GB per head: two batches
    assert bench.launches_per_step(1, 12, 512, "topk", True) == 5
    assert bench.launches_per_step(1, 12, 512, "topk", False, hyd=True) == 13


def test_reference_arm_prints_its_line_on_the_host():
    """bench.py --impl reference: the fp64 oracle on the host cores, one JSON
    line with the fields the reference arm must carry (no GPU needed)."""
    import json
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3",
                        "--workload", "tiny_iid_n1k"], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["config"]["workload"] == "tiny_iid_n1k"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]


def test_recorded_traffic_matches_workload_and_density():
    # the ncu record is used only for the workload, routing override and kernel
    # source it was captured with
    assert bench.recorded_traffic("no_such_workload") is None
    assert bench.recorded_traffic("sweep_n64k", None) is None      # captured with --density 0.15
    assert bench.recorded_traffic("dit_video_n32k", 0.5) is None    # captured with its own routing
    for name, dens in (("dit_video_n32k", None), ("sweep_n64k", 0.15)):
        v = bench.recorded_traffic(name, dens)
        assert v is None or v > 0
