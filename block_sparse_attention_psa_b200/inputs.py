"""Seeded synthetic inputs shaped like the workloads the pages describe.

This module holds no arithmetic of the attention method itself: it only draws
Q, K, V.  Both the CUDA path and the fp64 oracle consume what it returns.

Generators (numpy ``PCG64`` streams, float32 draws, rounded once to bf16 with
round-to-nearest-even):

* ``iid``: every element of Q, K, V ~ N(0, 1).
* ``clustered`` (DiT-video-like, PISA summary: video Diffusion Transformers;
  FlashPrefill summary: vertical / block-sparse attention patterns): per
  (batch, head) and per 64-token block, a query centroid cQ_I and a key
  centroid cK_J ~ N(0, I_d), drawn independently; token rows are
  centroid + 0.3 * N(0, I_d); four distinct key blocks per head, chosen
  uniformly, have their key centroid scaled by 3 (vertical stripes);
  V ~ N(0, 1).
* ``clustered_wide``: as ``clustered`` with both centroids scaled by 4 and
  token noise N(0, 1): block scores reach ~170 and a query's logits spread
  ~+-50 around its block's score, so the per-block softmax stabiliser of the
  attention kernel is far from some rows' largest terms (a stress input for
  its exact fixup path).
* ``clustered_slash``: as ``clustered``, and before the x3 scaling each query
  centroid I >= 8 gets (2 / sqrt(d)) * cK_{I-8} added, which raises the
  expected block score of the pair (I, I-8) by about 2 (a slash pattern).

Draw order per (b, h), row-major over (b, h): [clustered] cQ (M x d),
cK (M x d), the 4 heavy block ids, Q noise (N x d), K noise (N x d),
V (N x d); [iid] Q, K, V (N x d each).
"""

from __future__ import annotations

import math

import numpy as np
import torch

BLOCK = 64

# Workloads by what they are.  ``routing`` is (mode, parameter).
WORKLOADS = {
    # tiny i.i.d. case the oracle finishes in a blink; also run at density 1
    "tiny_iid_n1k": dict(B=1, H=2, N=1024, d=64, gen="iid", causal=False,
                         routing=("topk", 0.25), keep_first=False),
    # DiT-video shaped, top-k density 0.15 (the headline workload, N = 32K)
    "dit_video_n32k": dict(B=1, H=12, N=32768, d=128, gen="clustered",
                           causal=False, routing=("topk", 0.15), keep_first=False),
    # same tensors, sorting-free threshold alpha = 0.5 (+ diagonal block)
    "dit_video_n32k_thresh": dict(B=1, H=12, N=32768, d=128, gen="clustered",
                                  causal=False, routing=("thresh", 0.5),
                                  keep_first=False),
    # same tensors, threshold alpha = 0.5 read in the probability domain: keep
    # blocks whose softmax weight is at least half the row's largest
    # (s >= max + ln 0.5)
    "dit_video_n32k_thresh_prob": dict(B=1, H=12, N=32768, d=128, gen="clustered",
                                       causal=False, routing=("thresh_prob", 0.5),
                                       keep_first=False),
    # DiT-video shaped with wide logits (centroids x4, token noise 1): the
    # fixed per-block softmax stabiliser misses some rows by > 2^60
    "dit_video_n32k_wide": dict(B=1, H=12, N=32768, d=128, gen="clustered_wide",
                                causal=False, routing=("topk", 0.15), keep_first=False),
    # long causal prefill, threshold 0.5, block 0 and diagonal always kept
    "long_causal_n128k": dict(B=1, H=8, N=131072, d=128, gen="clustered_slash",
                              causal=True, routing=("thresh", 0.5), keep_first=True),
    # density sweep, d = 64; 1.0 is the dense baseline
    "sweep_n64k": dict(B=1, H=24, N=65536, d=64, gen="clustered", causal=False,
                       routing=("topk", (0.05, 0.10, 0.15, 0.30, 1.0)),
                       keep_first=False),
}


def _to_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def make_qkv(B: int, H: int, N: int, d: int, gen: str = "iid", seed: int = 0,
             block: int = BLOCK):
    """Return bf16 CPU tensors ``(q, k, v)`` of shape ``[B, H, N, d]``."""
    if N % block:
        raise ValueError("N must be a multiple of the block size")
    M = N // block
    rng = np.random.Generator(np.random.PCG64(seed))
    q = torch.empty((B, H, N, d), dtype=torch.bfloat16)
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    for b in range(B):
        for h in range(H):
            if gen == "iid":
                qh = rng.standard_normal((N, d), dtype=np.float32)
                kh = rng.standard_normal((N, d), dtype=np.float32)
                vh = rng.standard_normal((N, d), dtype=np.float32)
            elif gen in ("clustered", "clustered_slash", "clustered_wide"):
                wide = gen == "clustered_wide"
                cscale, noise = (np.float32(4.0), np.float32(1.0)) if wide else (np.float32(1.0), np.float32(0.3))
                cq = rng.standard_normal((M, d), dtype=np.float32)
                ck = rng.standard_normal((M, d), dtype=np.float32)
                if wide:
                    cq *= cscale
                    ck *= cscale
                heavy = rng.choice(M, size=min(4, M), replace=False)
                if gen == "clustered_slash" and M > 8:
                    cq[8:] += np.float32(2.0 / math.sqrt(d)) * ck[:-8]
                ck[heavy] *= np.float32(3.0)
                qh = np.repeat(cq, block, axis=0)
                qh += noise * rng.standard_normal((N, d), dtype=np.float32)
                kh = np.repeat(ck, block, axis=0)
                kh += noise * rng.standard_normal((N, d), dtype=np.float32)
                vh = rng.standard_normal((N, d), dtype=np.float32)
            else:
                raise ValueError(f"unknown generator {gen!r}")
            q[b, h] = _to_bf16(qh)
            k[b, h] = _to_bf16(kh)
            v[b, h] = _to_bf16(vh)
    return q, k, v


def workload_inputs(name: str, seed: int = 0):
    """Q, K, V for a named workload (bf16, CPU)."""
    w = WORKLOADS[name]
    return make_qkv(w["B"], w["H"], w["N"], w["d"], w["gen"], seed)
