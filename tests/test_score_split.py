"""The block scores' three-way bf16 split (PISA summary, "How are candidate
blocks narrowed": s_IJ = qbar_I . kbar_J / sqrt(d) in fp32).

The GPU computes each score as six bf16 x bf16 products of the parts
x0 = bf16(x), x1 = bf16(x - x0), x2 = bf16(x - x0 - x1) accumulated in fp32.
Here the split is emulated on the host (round-to-nearest-even to bf16 by bit
arithmetic) and the six-product sum, taken exactly in fp64, is held against
the exact fp64 product: the dropped terms must stay within a few 2^-24 of
sum |q_i k_i|, the error of an fp32 dot product.  Host-only arithmetic; the
oracle is not involved."""
import numpy as np
import pytest


def bf16_rn(x):
    """Round fp32 values to bf16 (nearest, ties to even), returned as fp32."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return (r & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def split3(x):
    x = np.asarray(x, dtype=np.float32)
    p0 = bf16_rn(x)
    r1 = (x - p0).astype(np.float32)
    p1 = bf16_rn(r1)
    r2 = (r1 - p1).astype(np.float32)
    p2 = bf16_rn(r2)
    return p0, p1, p2


def test_bf16_rounding_emulation():
    # values exactly halfway between two bf16 numbers go to the even one
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 1.0 + 2 ** -9], dtype=np.float32)
    assert bf16_rn(x).tolist() == [1.0, 1.0 + 2 ** -6, -1.0, 1.0]


@pytest.mark.parametrize("scale", [1e-3, 1.0, 37.0])
def test_split_parts_are_exact_differences(scale):
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(100000) * scale).astype(np.float32)
    p0, p1, p2 = split3(x)
    # each part is a bf16 value, and x - (p0 + p1 + p2) is far below fp32's own rounding
    for p in (p0, p1, p2):
        assert np.array_equal(bf16_rn(p), p)
    rest = x.astype(np.float64) - (p0.astype(np.float64) + p1 + p2)
    assert np.all(np.abs(rest) <= 2.0 ** -24 * np.abs(x.astype(np.float64)))


@pytest.mark.parametrize("d", [64, 128])
def test_six_products_reach_fp32_accuracy(d):
    rng = np.random.default_rng(2)
    # pooled statistics of the workloads: centroids plus noise, some large rows
    q = (rng.standard_normal((256, d)) * rng.choice([0.1, 1.0, 3.0], size=(256, 1))).astype(np.float32)
    k = (rng.standard_normal((256, d)) * rng.choice([0.1, 1.0, 3.0], size=(256, 1))).astype(np.float32)
    q0, q1, q2 = (p.astype(np.float64) for p in split3(q))
    k0, k1, k2 = (p.astype(np.float64) for p in split3(k))
    six = q2 @ k0.T + q1 @ k1.T + q0 @ k2.T + q1 @ k0.T + q0 @ k1.T + q0 @ k0.T
    exact = q.astype(np.float64) @ k.astype(np.float64).T
    mag = np.abs(q.astype(np.float64)) @ np.abs(k.astype(np.float64)).T
    assert np.max(np.abs(six - exact) / mag) <= 4 * 2.0 ** -24
    # one part alone (a plain bf16 product) is far from it
    assert np.max(np.abs(q0 @ k0.T - exact) / mag) > 2.0 ** -12
