"""Pins of the fp64 oracle to things other than itself.

Each test checks the oracle against a hand-derived worked example, a closed
form, a library routine the method reduces to in a special case, an
invariant, or brute force on tiny inputs.  None of them re-types the
oracle's own formula.  A final group plants plausible mistakes in a copy of
the oracle and checks that some pin catches each one.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.psa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_inputs(B, H, N, d, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    t = [(torch.randn(B, H, N, d, generator=g) * scale).to(torch.bfloat16) for _ in range(3)]
    return [x.double().numpy() for x in t]


def _all_selected(B, H, M, causal):
    lists = []
    for _ in range(B * H):
        for I in range(M):
            lists.append(np.arange(I + 1 if causal else M))
    return O._to_csr(lists)


def _random_csr(B, H, M, causal, rng, p=0.4):
    lists = []
    for _ in range(B * H):
        for I in range(M):
            n = I + 1 if causal else M
            keep = rng.random(n) < p
            if causal:
                keep[I] = True   # both routers always list the causal diagonal
            lists.append(np.nonzero(keep)[0])
    return O._to_csr(lists)


def _units_all(q, bs):
    B, H, N, _ = q.shape
    return O.unit_rows(B, H, N // bs)


def _assemble(out_units, q, bs):
    B, H, N, d = q.shape
    return out_units.reshape(B, H, N, d)


# ---------------------------------------------------------------- pool
def test_pool_matches_bruteforce_sums():
    q, k, v = _bf16_inputs(1, 2, 128, 8, seed=1)
    qbar, kbar, vsum = O.pool(q, k, v, block_size=32)
    for h in range(2):
        for J in range(4):
            for c in range(8):
                col = [q[0, h, J * 32 + t, c] for t in range(32)]
                assert qbar[0, h, J, c] == math.fsum(col) / 32
                col = [k[0, h, J * 32 + t, c] for t in range(32)]
                assert kbar[0, h, J, c] == math.fsum(col) / 32
                col = [v[0, h, J * 32 + t, c] for t in range(32)]
                assert vsum[0, h, J, c] == math.fsum(col)


def test_pool_rejects_ragged_n():
    q, k, v = _bf16_inputs(1, 1, 96, 4, seed=2)
    with pytest.raises(ValueError):
        O.pool(q, k, v, block_size=64)


# ---------------------------------------------------------------- scores
def test_block_scores_bruteforce():
    rng = np.random.default_rng(3)
    qbar = rng.standard_normal((1, 2, 5, 6))
    kbar = rng.standard_normal((1, 2, 5, 6))
    s = O.block_scores(qbar, kbar)
    for h in range(2):
        for I in range(5):
            for J in range(5):
                ref = math.fsum(qbar[0, h, I, c] * kbar[0, h, J, c] for c in range(6))
                assert abs(s[0, h, I, J] - ref / math.sqrt(6)) < 1e-14


# ---------------------------------------------------------------- top-k
def _bruteforce_topk(vals, k):
    """The unique k-subset whose every member beats every non-member
    (higher score, or equal score and smaller index)."""
    n = len(vals)
    winners = []
    for sub in itertools.combinations(range(n), k):
        rest = [j for j in range(n) if j not in sub]
        if all(vals[a] > vals[b] or (vals[a] == vals[b] and a < b)
               for a in sub for b in rest):
            winners.append(list(sub))
    assert len(winners) == 1
    return winners[0]


@pytest.mark.parametrize("causal", [False, True])
def test_topk_bruteforce_all_subsets(causal):
    rng = np.random.default_rng(4)
    M = 8
    for trial in range(4):
        # quantised scores so that ties occur
        s = np.round(rng.standard_normal((1, 1, M, M)) * 2) / 2
        for kk in range(1, M + 1):
            density = kk / M
            rp, ci = O.route_topk(s, density, causal)
            for I in range(M):
                n = I + 1 if causal else M
                k = min(kk, n)
                got = list(ci[rp[I]:rp[I + 1]])
                if causal:   # diagonal + the k-1 best earlier blocks
                    want = sorted(_bruteforce_topk(list(s[0, 0, I, :I]), k - 1) + [I])
                else:
                    want = _bruteforce_topk(list(s[0, 0, I, :n]), k)
                assert got == want


def test_topk_count_reading():
    # ceil of the single-precision product, clamped to [1, n_cand]
    assert O.topk_count(0.15, 512, 512) == 77
    assert O.topk_count(0.25, 16, 16) == 4
    assert [O.topk_count(x, 1024, 1024) for x in (0.05, 0.10, 0.15, 0.30, 1.0)] == \
        [52, 103, 154, 308, 1024]
    assert O.topk_count(0.3, 1000, 1000) == 300      # fl32(0.3f * 1000) == 300
    assert O.topk_count(0.0, 64, 64) == 1
    assert O.topk_count(0.9, 64, 3) == 3


def test_topk_density_one_selects_every_candidate():
    rng = np.random.default_rng(5)
    s = rng.standard_normal((1, 2, 6, 6))
    for causal in (False, True):
        rp, ci = O.route_topk(s, 1.0, causal)
        rp2, ci2 = _all_selected(1, 2, 6, causal)
        assert np.array_equal(rp, rp2) and np.array_equal(ci, ci2)


# ---------------------------------------------------------------- threshold
def test_threshold_hand_example():
    with open(os.path.join(GOLDEN, "flashprefill_threshold_hand.json")) as f:
        g = json.load(f)
    qbar = np.array(g["qbar"]).reshape(1, 1, 5, 1)
    kbar = np.array(g["kbar"]).reshape(1, 1, 5, 1)
    s = O.block_scores(qbar, kbar)
    for key, causal, kf in (("noncausal", False, False), ("causal", True, False),
                            ("causal_keep_first", True, True)):
        rp, ci = O.route_thresh(s, g["alpha"], causal, kf)
        got = [list(ci[rp[i]:rp[i + 1]]) for i in range(5)]
        assert got == g[key], key


def test_threshold_bruteforce_and_limits():
    rng = np.random.default_rng(6)
    s = rng.standard_normal((1, 2, 7, 7))
    for causal in (False, True):
        for kf in (False, True):
            rp, ci = O.route_thresh(s, 0.5, causal, kf)
            r = 0
            for h in range(2):
                for I in range(7):
                    n = I + 1 if causal else 7
                    m = max(s[0, h, I, :n])
                    want = [J for J in range(n) if s[0, h, I, J] >= 0.5 * m
                            or J == I or (kf and J == 0)]
                    assert list(ci[rp[r]:rp[r + 1]]) == want
                    r += 1
    # alpha > 1 with a positive row max keeps only the forced blocks
    s_pos = np.abs(s) + 0.1
    rp, ci = O.route_thresh(s_pos, 1.5, True, True)
    r = 0
    for h in range(2):
        for I in range(7):
            assert list(ci[rp[r]:rp[r + 1]]) == sorted({0, I})
            r += 1


def test_threshold_prob_is_the_softmax_ratio_rule():
    # probability reading: p_IJ >= alpha * max p, with p the softmax of the
    # row's candidate scores, written out here with the normaliser
    rng = np.random.default_rng(17)
    s = 3.0 * rng.standard_normal((1, 2, 9, 9))
    alpha = 0.25
    for causal in (False, True):
        for kf in (False, True):
            rp, ci = O.route_thresh_prob(s, alpha, causal, kf)
            r = 0
            for h in range(2):
                for I in range(9):
                    n = I + 1 if causal else 9
                    e = np.exp(s[0, h, I, :n] - s[0, h, I, :n].max())
                    p = e / e.sum()
                    want = [J for J in range(n) if p[J] >= np.float32(alpha) * p.max()
                            or J == I or (kf and J == 0)]
                    assert list(ci[rp[r]:rp[r + 1]]) == want
                    r += 1


def test_threshold_prob_limits_and_shift_invariance():
    rng = np.random.default_rng(18)
    s = rng.standard_normal((1, 1, 8, 8))
    # alpha = 1 keeps the row's best block (plus the forced ones); a tiny alpha keeps all
    rp, ci = O.route_thresh_prob(s, 1.0, False, False)
    for I in range(8):
        assert list(ci[rp[I]:rp[I + 1]]) == sorted({int(np.argmax(s[0, 0, I])), I})
    rp, ci = O.route_thresh_prob(s, 1e-30, True, False)
    for I in range(8):
        assert list(ci[rp[I]:rp[I + 1]]) == list(range(I + 1))
    # only score differences matter: a per-row shift keeps every list, while the
    # logit-domain rule (alpha times the max) moves
    shift = 5.0 * rng.standard_normal((1, 1, 8, 1))
    a = O.route_thresh_prob(s, 0.3, False, False)
    b = O.route_thresh_prob(s + shift, 0.3, False, False)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    c = O.route_thresh(s, 0.3, False, False)
    d = O.route_thresh(s + shift, 0.3, False, False)
    assert not all(np.array_equal(x, y) for x, y in zip(c, d))


def test_routing_invariant_to_positive_query_scale():
    rng = np.random.default_rng(7)
    qbar = rng.standard_normal((1, 2, 9, 4))
    kbar = rng.standard_normal((1, 2, 9, 4))
    for causal in (False, True):
        a = O.route_topk(O.block_scores(qbar, kbar), 0.3, causal)
        b = O.route_topk(O.block_scores(2.0 * qbar, kbar), 0.3, causal)
        assert all(np.array_equal(x, y) for x, y in zip(a, b))
        a = O.route_thresh(O.block_scores(qbar, kbar), 0.5, causal, True)
        b = O.route_thresh(O.block_scores(2.0 * qbar, kbar), 0.5, causal, True)
        assert all(np.array_equal(x, y) for x, y in zip(a, b))


# ---------------------------------------------------------------- attention
def test_hand_worked_two_block_example():
    with open(os.path.join(GOLDEN, "pisa_two_block_hand.json")) as f:
        g = json.load(f)
    q = np.array(g["q"]).reshape(1, 1, 4, 1)
    k = np.array(g["k"]).reshape(1, 1, 4, 1)
    v = np.array(g["v"]).reshape(1, 1, 4, 1)
    bs = g["block_size"]
    _, kbar, vsum = O.pool(q, k, v, bs)
    out, lse = O.attention(q, k, v, kbar, vsum, np.array(g["row_ptr"]),
                           np.array(g["col_idx"]), g["causal"], bs)
    assert np.allclose(out.reshape(-1), g["out"], rtol=0, atol=1e-14)
    assert np.allclose(lse.reshape(-1), g["lse"], rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_all_selected_equals_library_softmax_attention(causal):
    """density 1: every candidate exact -> textbook softmax(QK^T/sqrt d)V."""
    q, k, v = _bf16_inputs(2, 2, 256, 16, seed=8)
    bs = 64
    _, kbar, vsum = O.pool(q, k, v, bs)
    rp, ci = _all_selected(2, 2, 4, causal)
    out, lse = O.attention(q, k, v, kbar, vsum, rp, ci, causal, bs)
    # the textbook product in fp64 with library softmax / logsumexp (explicit ops:
    # no fused-attention backend whose choice could vary between runs)
    logits = torch.from_numpy(q) @ torch.from_numpy(k).transpose(-1, -2) / 4.0
    if causal:
        logits = logits.masked_fill(torch.ones(256, 256).triu(1).bool(), float("-inf"))
    ref = torch.softmax(logits, dim=-1) @ torch.from_numpy(v)
    err = np.abs(out.reshape(q.shape) - ref.numpy()).max()
    assert err < 1e-12, err
    ref_lse = torch.logsumexp(logits, dim=-1).numpy()
    err = np.abs(lse.reshape(2, 2, 256) - ref_lse).max()
    assert err < 1e-12, err


@pytest.mark.parametrize("causal", [False, True])
def test_zeroth_order_exact_for_blockwise_constant_keys(causal):
    """If every key of a block equals the block mean, e^{q.k_j} = e^{q.kbar}
    for each token, so the 0th-order term is exact for ANY selection."""
    q, k, v = _bf16_inputs(1, 2, 512, 8, seed=9)
    bs = 64
    k = np.repeat(k.reshape(1, 2, 8, bs, 8).mean(axis=3), bs, axis=2)
    _, kbar, vsum = O.pool(q, k, v, bs)
    rng = np.random.default_rng(10)
    rp, ci = _random_csr(1, 2, 8, causal, rng)
    out, _ = O.attention(q, k, v, kbar, vsum, rp, ci, causal, bs)
    # causal rows list their diagonal block (exact, token mask), every earlier
    # block is exact or 0th-order, and both agree for constant keys
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x) for x in (q, k, v)), is_causal=causal).numpy()
    assert np.abs(out.reshape(q.shape) - ref).max() < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_online_fold_equals_two_pass(causal):
    """FlashAttention blog, section 2: the online recurrence gives the same
    answer as the full softmax (the blog measured 2.4e-8 in fp32; fp64 here)."""
    q, k, v = _bf16_inputs(1, 2, 640, 16, seed=11, scale=2.0)
    bs = 64
    _, kbar, vsum = O.pool(q, k, v, bs)
    rng = np.random.default_rng(12)
    rp, ci = _random_csr(1, 2, 10, causal, rng, p=0.3)
    a, la = O.attention(q, k, v, kbar, vsum, rp, ci, causal, bs)
    b, lb = O.attention_online(q, k, v, kbar, vsum, rp, ci, causal, bs)
    assert np.abs(a - b).max() < 1e-12
    assert np.abs(la - lb).max() < 1e-12


def test_nothing_selected_is_softmax_over_pseudo_keys():
    """Empty lists: out_i = sum_J softmax_J(q_i.kbar_J/sqrt d) * vsum_J / b."""
    q, k, v = _bf16_inputs(1, 1, 384, 8, seed=13)
    bs = 64
    M = 6
    kbar_ref = torch.from_numpy(k).reshape(1, 1, M, bs, 8).mean(dim=3)
    vmean_ref = torch.from_numpy(v).reshape(1, 1, M, bs, 8).sum(dim=3) / bs
    _, kbar, vsum = O.pool(q, k, v, bs)
    rp = np.zeros(M + 1, dtype=np.int64)
    ci = np.zeros(0, dtype=np.int64)
    out, _ = O.attention(q, k, v, kbar, vsum, rp, ci, False, bs)
    a = torch.from_numpy(q)[0, 0] @ kbar_ref[0, 0].T / math.sqrt(8)
    ref = torch.softmax(a, dim=-1) @ vmean_ref[0, 0]
    assert np.abs(out.reshape(384, 8) - ref.numpy()).max() < 1e-13


def test_linear_in_v_and_convex():
    q, k, v = _bf16_inputs(1, 1, 512, 8, seed=14)
    _, _, v2 = _bf16_inputs(1, 1, 512, 8, seed=15)
    bs = 64
    rng = np.random.default_rng(16)
    rp, ci = _random_csr(1, 1, 8, False, rng)

    def run(vv):
        _, kbar, vsum = O.pool(q, k, vv, bs)
        return O.attention(q, k, vv, kbar, vsum, rp, ci, False, bs)[0]

    o1, o2, o12 = run(v), run(v2), run(2.0 * v - 3.0 * v2)
    assert np.abs(o12 - (2.0 * o1 - 3.0 * o2)).max() < 1e-12
    # each output row is a convex combination of the listed rows and the
    # block means of the unlisted blocks
    vmean = v.reshape(8, bs, 8).mean(axis=1)
    for I in range(8):
        lst = ci[rp[I]:rp[I + 1]]
        rows = [v[0, 0, J * bs:(J + 1) * bs] for J in lst]
        rows += [vmean[J:J + 1] for J in range(8) if J not in lst]
        allr = np.concatenate(rows)
        lo, hi = allr.min(axis=0), allr.max(axis=0)
        blk = o1[I]
        assert (blk >= lo - 1e-12).all() and (blk <= hi + 1e-12).all()


def test_causal_future_blocks_do_not_contribute():
    q, k, v = _bf16_inputs(1, 1, 512, 8, seed=17)
    bs = 64
    rng = np.random.default_rng(18)
    rp, ci = _random_csr(1, 1, 8, True, rng)
    _, kbar, vsum = O.pool(q, k, v, bs)
    base, _ = O.attention(q, k, v, kbar, vsum, rp, ci, True, bs)
    k2, v2 = k.copy(), v.copy()
    k2[0, 0, 320:] += 5.0
    v2[0, 0, 320:] -= 7.0
    _, kbar2, vsum2 = O.pool(q, k2, v2, bs)
    moved, _ = O.attention(q, k2, v2, kbar2, vsum2, rp, ci, True, bs)
    assert np.array_equal(base[:5], moved[:5])         # blocks 0..4 see only J <= I
    assert not np.allclose(base[5:], moved[5:])


def _scalar_bruteforce(q, k, v, lists, causal, bs):
    """Independent scalar restatement on tiny inputs: plain Python loops."""
    _, _, N, d = q.shape
    M = N // bs
    tau = 1.0 / math.sqrt(d)
    out = np.zeros((N, d))
    for i in range(N):
        I = i // bs
        terms = []  # (log-weight, value row)
        for J in range(I + 1 if causal else M):
            if causal and J == I and J not in lists[I]:
                continue      # a causal diagonal block is never approximated
            if J in lists[I]:
                for j in range(J * bs, J * bs + bs):
                    if causal and j > i:
                        continue
                    z = tau * sum(q[0, 0, i, c] * k[0, 0, j, c] for c in range(d))
                    terms.append((z, [v[0, 0, j, c] for c in range(d)]))
            else:
                kb = [sum(k[0, 0, j, c] for j in range(J * bs, J * bs + bs)) / bs
                      for c in range(d)]
                vs = [sum(v[0, 0, j, c] for j in range(J * bs, J * bs + bs))
                      for c in range(d)]
                a = tau * sum(q[0, 0, i, c] * kb[c] for c in range(d))
                terms.append((a + math.log(bs), [x / bs for x in vs]))
        mx = max(t[0] for t in terms)
        den = sum(math.exp(t[0] - mx) for t in terms)
        for c in range(d):
            out[i, c] = sum(math.exp(t[0] - mx) * t[1][c] for t in terms) / den
    return out


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_scalar_bruteforce(causal):
    q, k, v = _bf16_inputs(1, 1, 128, 8, seed=19)
    bs = 16
    M = 8
    rng = np.random.default_rng(20)
    rp, ci = _random_csr(1, 1, M, causal, rng)
    lists = [list(ci[rp[I]:rp[I + 1]]) for I in range(M)]
    _, kbar, vsum = O.pool(q, k, v, bs)
    out, _ = O.attention(q, k, v, kbar, vsum, rp, ci, causal, bs)
    ref = _scalar_bruteforce(q, k, v, lists, causal, bs)
    assert np.abs(out.reshape(128, 8) - ref).max() < 1e-12


def test_invalid_lists_rejected():
    q, k, v = _bf16_inputs(1, 1, 256, 4, seed=21)
    _, kbar, vsum = O.pool(q, k, v, 64)
    rp = np.array([0, 1, 2, 3, 4])
    with pytest.raises(ValueError):   # future block in a causal row
        O.attention(q, k, v, kbar, vsum, rp, np.array([1, 0, 0, 0]), True, 64)
    rp = np.array([0, 2, 2, 2, 2])
    with pytest.raises(ValueError):   # repeated block
        O.attention(q, k, v, kbar, vsum, rp, np.array([1, 1]), False, 64)


# ---------------------------------------------------------------- planted mistakes
def _pins_fail(monkeypatch, name, fn):
    """Replace one oracle internal with a plausible mistake and report whether
    any of the attention / routing pins above fails."""
    monkeypatch.setattr(O, name, fn)
    checks = [
        test_hand_worked_two_block_example,
        lambda: test_all_selected_equals_library_softmax_attention(True),
        lambda: test_zeroth_order_exact_for_blockwise_constant_keys(False),
        test_nothing_selected_is_softmax_over_pseudo_keys,
        lambda: test_tiny_scalar_bruteforce(True),
        lambda: test_tiny_scalar_bruteforce(False),
        lambda: test_topk_bruteforce_all_subsets(True),
        test_threshold_hand_example,
        test_causal_future_blocks_do_not_contribute,
    ]
    failed = 0
    for c in checks:
        try:
            c()
        except (AssertionError, ValueError, IndexError):
            failed += 1
    return failed


def test_planted_mistakes_are_caught(monkeypatch):
    real_pool, real_terms = O.pool, O._unit_terms
    real_scores, real_topk_count = O.block_scores, O.topk_count

    def pool_vmean(q, k, v, block_size=64):          # value MEAN instead of sum
        a, b, c = real_pool(q, k, v, block_size)
        return a, b, c / block_size

    def pool_ksum(q, k, v, block_size=64):           # key SUM instead of mean
        a, b, c = real_pool(q, k, v, block_size)
        return a, b * block_size, c

    def terms_no_mask(q, k, v, kbar, vsum, sel, b, h, I, causal, bs):
        return real_terms(q, k, v, kbar, vsum, sel, b, h, I, False, bs)

    def terms_swap(q, k, v, kbar, vsum, sel, b, h, I, causal, bs):  # K <-> Q
        return real_terms(k, q, v, kbar, vsum, sel, b, h, I, causal, bs)

    def scores_unscaled(qbar, kbar):                 # dropped 1/sqrt(d)
        return real_scores(qbar, kbar) * math.sqrt(qbar.shape[-1])

    def scores_negated(qbar, kbar):                  # wrong sign
        return -real_scores(qbar, kbar)

    def topk_floor(density, M, n):                   # floor instead of ceil
        return max(1, min(int(math.floor(np.float32(density) * np.float32(M))), n))

    for name, fn in (("pool", pool_vmean), ("pool", pool_ksum),
                     ("_unit_terms", terms_no_mask), ("_unit_terms", terms_swap),
                     ("block_scores", scores_negated)):
        assert _pins_fail(monkeypatch, name, fn) > 0, (name, fn.__name__)
        monkeypatch.undo()
    # the threshold example has d = 1, so the unscaled score is caught by the
    # scale-free hand example only through sqrt(d) != 1 cases: check directly
    monkeypatch.setattr(O, "block_scores", scores_unscaled)
    with pytest.raises(AssertionError):
        test_block_scores_bruteforce()
    monkeypatch.undo()
    monkeypatch.setattr(O, "topk_count", topk_floor)
    with pytest.raises(AssertionError):
        test_topk_count_reading()
    monkeypatch.undo()
