"""Pins of the oracle's first-order term and of the token-pooled scoring
reading (PISA summary, "Why approximating unselected blocks keeps softmax
intact" and the FAQ on the global first-order correction; FlashPrefill
summary, 2.a "Block approximation").

The first-order term is the expansion of e^{q.k/sqrt(d)} to first order
around the block-mean key.  What fixes it independently of its own formula:

* the order of the error: with the keys of every block spread by eps around
  their mean, the 0th-order output misses the exact attention by O(eps) and
  the first-order output by O(eps^2), so halving eps halves the first error
  and quarters the second (a wrong sign, a transposed statistic, a missing
  1/sqrt(d) or a wrong block all leave an O(eps) error behind);
* keys constant over each block: the deviations vanish and the term is zero;
* blocks that share one deviation pattern: every per-block statistic is the
  same closed-form matrix, so the global statistic (their mean) gives the
  per-block result exactly.
"""
import math

import numpy as np
import pytest

import oracle.psa_oracle as O

BS = 64


def _spread_keys(eps, seed=0, H=1, M=4, d=8):
    """Block centres plus eps times a zero-mean deviation per block."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, H, M * BS, d))
    c = rng.standard_normal((1, H, M, 1, d))
    u = rng.standard_normal((1, H, M, BS, d))
    u -= u.mean(axis=3, keepdims=True)
    k = (c + eps * u).reshape(1, H, M * BS, d)
    v = rng.standard_normal((1, H, M * BS, d))
    return q, k, v


def _outputs(q, k, v, lists, causal=False):
    H, N = q.shape[1], q.shape[2]
    M = N // BS
    rp, ci = O._to_csr(lists * H)
    _, kbar, vsum = O.pool(q, k, v, BS)
    HJ = O.block_deviation_stats(k, v, BS)
    zeroth, _ = O.attention(q, k, v, kbar, vsum, rp, ci, causal, BS)
    first, _ = O.attention_first_order(q, k, v, kbar, vsum, rp, ci, causal, HJ, BS)
    # exact: every candidate listed
    rp_all, ci_all = O._to_csr([np.arange(I + 1 if causal else M) for _ in range(H) for I in range(M)])
    exact, _ = O.attention(q, k, v, kbar, vsum, rp_all, ci_all, causal, BS)
    return zeroth, first, exact


@pytest.mark.parametrize("causal", [False, True])
def test_first_order_error_is_second_order(causal):
    M = 4
    # row I lists only its own block: every other candidate is approximated
    lists = [np.array([I]) for I in range(M)]
    e0, e1 = [], []
    for eps in (0.04, 0.02, 0.01):
        q, k, v = _spread_keys(eps, seed=3, M=M)
        zeroth, first, exact = _outputs(q, k, v, lists, causal)
        e0.append(np.abs(zeroth - exact).max())
        e1.append(np.abs(first - exact).max())
    for i in range(2):
        assert 1.7 < e0[i] / e0[i + 1] < 2.3, e0      # first-order error of the 0th-order term
        assert 3.4 < e1[i] / e1[i + 1] < 4.6, e1      # second-order error with the correction
        assert e1[i] < 0.2 * e0[i]


def test_first_order_term_vanishes_for_blockwise_constant_keys():
    q, k, v = _spread_keys(0.0, seed=4)
    HJ = O.block_deviation_stats(k, v, BS)
    assert np.abs(HJ).max() < 1e-12      # only the rounding of the block means
    lists = [np.array([I]) for I in range(4)]
    zeroth, first, exact = _outputs(q, k, v, lists)
    assert np.abs(first - zeroth).max() < 1e-12
    assert np.abs(first - exact).max() < 1e-12      # the 0th-order term is exact here


def test_first_order_with_everything_listed_is_plain_attention():
    q, k, v = _spread_keys(0.3, seed=5)
    lists = [np.arange(4) for _ in range(4)]
    zeroth, first, exact = _outputs(q, k, v, lists)
    assert np.abs(first - exact).max() < 1e-13


def test_deviation_stats_closed_form_and_global_reading():
    # k_j = c_J + u_t, v_j = w_J + y_t (t = position in the block), sum_t u_t = 0:
    # H_J = sum_t u_t (w_J + y_t)^T = sum_t u_t y_t^T for every block
    rng = np.random.default_rng(6)
    M, d = 4, 8
    u = rng.standard_normal((BS, d))
    u -= u.mean(axis=0)
    y = rng.standard_normal((BS, d))
    c = rng.standard_normal((M, d))
    w = rng.standard_normal((M, d))
    k = (c[:, None, :] + u[None]).reshape(1, 1, M * BS, d)
    v = (w[:, None, :] + y[None]).reshape(1, 1, M * BS, d)
    q = rng.standard_normal((1, 1, M * BS, d))
    HJ = O.block_deviation_stats(k, v, BS)
    closed = sum(np.outer(u[t], y[t]) for t in range(BS))
    for J in range(M):
        assert np.abs(HJ[0, 0, J] - closed).max() < 1e-12
    Hg = O.global_deviation_stat(HJ)
    assert np.abs(Hg[0, 0] - closed).max() < 1e-12
    _, kbar, vsum = O.pool(q, k, v, BS)
    rp, ci = O._to_csr([np.array([I]) for I in range(M)])
    per_block, _ = O.attention_first_order(q, k, v, kbar, vsum, rp, ci, False, HJ, BS)
    global_h, _ = O.attention_first_order(q, k, v, kbar, vsum, rp, ci, False, Hg, BS)
    assert np.abs(per_block - global_h).max() < 1e-13


def test_planted_first_order_mistakes_are_caught(monkeypatch):
    real = O._first_order_numerator
    plants = {
        "sign": lambda ea, Qi, Hs, d: -real(ea, Qi, Hs, d),
        "transposed": lambda ea, Qi, Hs, d: real(ea, Qi, np.swapaxes(Hs, -1, -2), d),
        "unscaled": lambda ea, Qi, Hs, d: real(ea, Qi, Hs, d) * math.sqrt(d),
    }
    for name, fn in plants.items():
        monkeypatch.setattr(O, "_first_order_numerator", fn)
        with pytest.raises(AssertionError):
            test_first_order_error_is_second_order(False)
        monkeypatch.undo()
    # a statistic of the raw keys (not their deviations from the block mean)
    real_stats = O.block_deviation_stats

    def raw_keys(k, v, block_size=64):
        B, H, N, d = k.shape
        kb = np.asarray(k, dtype=np.float64).reshape(B, H, N // block_size, block_size, d)
        vb = np.asarray(v, dtype=np.float64).reshape(B, H, N // block_size, block_size, d)
        return np.einsum("bhmtk,bhmtv->bhmkv", kb, vb)

    monkeypatch.setattr(O, "block_deviation_stats", raw_keys)
    with pytest.raises(AssertionError):
        test_first_order_error_is_second_order(False)
    monkeypatch.undo()
    assert O.block_deviation_stats is real_stats


def test_token_pooled_scores_equal_pooled_query_scores():
    # FlashPrefill's score-then-pool with mean pooling over the query block is
    # the block score of the pooled query (linearity of the dot product)
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 2, 8 * BS, 16))
    k = rng.standard_normal((1, 2, 8 * BS, 16))
    qbar, kbar, _ = O.pool(q, k, k, BS)
    fused = O.token_pooled_block_scores(q, kbar, BS)
    direct = O.block_scores(qbar, kbar)
    assert np.abs(fused - direct).max() < 1e-13
    # and it is not the max-pooled token score (a different reading)
    tok = np.matmul(q, np.swapaxes(kbar, -1, -2)) / 4.0
    maxpool = tok.reshape(1, 2, 8, BS, 8).max(axis=3)
    assert np.abs(maxpool - direct).max() > 0.1
