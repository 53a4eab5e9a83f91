"""The seeded generators are deterministic and have the documented shapes."""

import numpy as np
import torch

from block_sparse_attention_psa_b200.inputs import WORKLOADS, make_qkv


def test_deterministic_and_bf16():
    a = make_qkv(1, 2, 256, 64, "clustered", seed=0)
    b = make_qkv(1, 2, 256, 64, "clustered", seed=0)
    c = make_qkv(1, 2, 256, 64, "clustered", seed=1)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.shape == (1, 2, 256, 64)
        assert torch.equal(x, y)
    assert not torch.equal(a[0], c[0])


def test_clustered_structure():
    q, k, v = make_qkv(1, 1, 64 * 32, 64, "clustered", seed=0)
    kb = k.float().reshape(32, 64, 64)
    # within-block spread ~0.3, centroid norms ~sqrt(d) (x3 for 4 heavy blocks)
    spread = (kb - kb.mean(1, keepdim=True)).std().item()
    assert 0.25 < spread < 0.35
    norms = kb.mean(1).norm(dim=-1)
    assert (norms > 2 * np.sqrt(64)).sum().item() == 4


def test_workload_table():
    assert WORKLOADS["dit_video_n32k"]["N"] == 32768
    for w in WORKLOADS.values():
        assert w["N"] % 64 == 0 and w["d"] in (64, 128)


def test_wide_structure():
    q, k, v = make_qkv(1, 1, 64 * 32, 64, "clustered_wide", seed=0)
    kb = k.float().reshape(32, 64, 64)
    spread = (kb - kb.mean(1, keepdim=True)).std().item()
    assert 0.9 < spread < 1.1
    norms = kb.mean(1).norm(dim=-1)
    assert (norms > 2 * 4 * np.sqrt(64)).sum().item() == 4
