"""Pins of the oracle's gradients of the 0th-order attention (the
training-support variant of the PISA summary, "Minimal usage").

* forward: the differentiable torch forward reproduces ``psa_oracle.attention``;
* central finite differences in fp64 on tiny inputs (directional derivatives);
* density one: the gradients of textbook softmax attention, written out here
  with explicit ops;
* keys constant over each block: the 0th-order term is exact for any query,
  so dq and dv equal dense attention's; dk reaches a block through its mean
  key, so only its block sums (not each row) equal dense attention's.
"""
import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
import oracle.psa_oracle_grad as G

BS = 16   # small blocks keep the pure-Python loops fast; the method has no fixed block size


def _inputs(seed, H=2, M=4, d=4, const_keys=False):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, H, M * BS, d))
    k = rng.standard_normal((1, H, M * BS, d))
    if const_keys:
        k = np.repeat(k.reshape(1, H, M, BS, d)[:, :, :, :1], BS, axis=3).reshape(1, H, M * BS, d)
    v = rng.standard_normal((1, H, M * BS, d))
    return q, k, v


def _random_lists(H, M, causal, rng):
    lists = []
    for _ in range(H):
        for I in range(M):
            n = I + 1 if causal else M
            keep = rng.random(n) < 0.4
            if causal:
                keep[I] = True
            lists.append(np.nonzero(keep)[0])
    return O._to_csr(lists)


def _dense_grads(q, k, v, causal, dout):
    t = [torch.tensor(x, requires_grad=True) for x in (q, k, v)]
    d = q.shape[-1]
    logits = t[0] @ t[1].transpose(-1, -2) / np.sqrt(d)
    if causal:
        n = q.shape[2]
        logits = logits.masked_fill(torch.ones(n, n).triu(1).bool(), float("-inf"))
    out = torch.softmax(logits, dim=-1) @ t[2]
    (out * torch.tensor(dout)).sum().backward()
    return [x.grad.numpy() for x in t]


@pytest.mark.parametrize("causal", [False, True])
def test_forward_matches_the_oracle(causal):
    q, k, v = _inputs(1)
    rp, ci = _random_lists(2, 4, causal, np.random.default_rng(2))
    _, kbar, vsum = O.pool(q, k, v, BS)
    ref, _ = O.attention(q, k, v, kbar, vsum, rp, ci, causal, BS)
    got = G.forward(*(torch.tensor(x) for x in (q, k, v)), rp, ci, causal, BS)
    assert np.abs(got.detach().numpy().reshape(ref.shape) - ref).max() < 1e-13


@pytest.mark.parametrize("causal", [False, True])
def test_gradients_match_central_differences(causal):
    rng = np.random.default_rng(3)
    q, k, v = _inputs(4, H=1, M=3, d=3)
    rp, ci = _random_lists(1, 3, causal, rng)
    dout = rng.standard_normal(q.shape)
    grads = G.backward(q, k, v, rp, ci, causal, dout, BS)

    def loss(qq, kk, vv):
        _, kbar, vsum = O.pool(qq, kk, vv, BS)
        out, _ = O.attention(qq, kk, vv, kbar, vsum, rp, ci, causal, BS)
        return float((out.reshape(q.shape) * dout).sum())

    h = 1e-5
    for which in range(3):
        for trial in range(3):
            dirn = rng.standard_normal(q.shape)
            args_p = [q, k, v]
            args_m = [q, k, v]
            args_p[which] = args_p[which] + h * dirn
            args_m[which] = args_m[which] - h * dirn
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            ad = float((grads[which] * dirn).sum())
            assert abs(fd - ad) <= 1e-7 * max(1.0, abs(ad)), (which, fd, ad)


@pytest.mark.parametrize("causal", [False, True])
def test_density_one_gradients_are_dense_attention_gradients(causal):
    q, k, v = _inputs(5)
    M = 4
    lists = [np.arange(I + 1 if causal else M) for _ in range(2) for I in range(M)]
    rp, ci = O._to_csr(lists)
    dout = np.random.default_rng(6).standard_normal(q.shape)
    got = G.backward(q, k, v, rp, ci, causal, dout, BS)
    want = _dense_grads(q, k, v, causal, dout)
    for g, w in zip(got, want):
        assert np.abs(g - w).max() < 1e-12


def test_blockwise_constant_keys_gradients():
    q, k, v = _inputs(7, const_keys=True)
    rp, ci = _random_lists(2, 4, False, np.random.default_rng(8))
    dout = np.random.default_rng(9).standard_normal(q.shape)
    dq, dk, dv = G.backward(q, k, v, rp, ci, False, dout, BS)
    dq_d, dk_d, dv_d = _dense_grads(q, k, v, False, dout)
    assert np.abs(dq - dq_d).max() < 1e-12
    assert np.abs(dv - dv_d).max() < 1e-12
    blk = lambda x: x.reshape(1, 2, 4, BS, -1).sum(axis=3)
    assert np.abs(blk(dk) - blk(dk_d)).max() < 1e-12
    # ... but not row by row: an approximated block's key rows share one gradient
    assert np.abs(dk - dk_d).max() > 1e-3


def test_planted_gradient_mistake_is_caught(monkeypatch):
    # gradients that stop at the pooled statistics (kbar, vsum treated as
    # constants) miss the 0th-order path into k and v
    real = G._unit
    monkeypatch.setattr(G, "_unit", lambda q, k, v, kbar, vsum, *rest: real(q, k, v, kbar.detach(),
                                                                            vsum.detach(), *rest))
    with pytest.raises(AssertionError):
        test_gradients_match_central_differences(False)


@pytest.mark.parametrize("causal", [False, True])
def test_given_output_backward(causal):
    # A backward pass forms D_i = dout_i . out_i from the output it is given.
    # With the exact output the oracle's given-output backward is the plain
    # gradient; with out + e it shifts dq_i by exactly -tau delta_i khat_i, where
    # delta_i = dout_i . e_i and khat_i = sum_j p_ij k_j + sum_J pi_iJ (b kbar_J)
    # is the softmax-weighted mean key (the attention of the oracle's plain
    # forward with the keys as values), and leaves dv unchanged.
    rng = np.random.default_rng(11)
    q, k, v = _inputs(12)
    H, N, d = q.shape[1], q.shape[2], q.shape[3]
    M = N // BS
    rp, ci = _random_lists(H, M, causal, rng)
    dout = rng.standard_normal(q.shape)
    _, kbar, vsum = O.pool(q, k, v, BS)
    out, _ = O.attention(q, k, v, kbar, vsum, rp, ci, causal, BS)
    out = out.reshape(q.shape)
    plain = G.backward(q, k, v, rp, ci, causal, dout, BS)
    same = G.backward(q, k, v, rp, ci, causal, dout, BS, out_for_delta=out)
    for a, b in zip(plain, same):
        assert np.abs(a - b).max() < 1e-12
    e = 1e-3 * rng.standard_normal(q.shape)
    shifted = G.backward(q, k, v, rp, ci, causal, dout, BS, out_for_delta=out + e)
    delta = (dout * e).sum(-1)
    khat, _ = O.attention(q, k, k, kbar, BS * kbar, rp, ci, causal, BS)
    khat = khat.reshape(q.shape)
    want_dq = plain[0] - delta[..., None] * khat / np.sqrt(d)
    assert np.abs(shifted[0] - want_dq).max() < 1e-10
    assert np.abs(shifted[2] - plain[2]).max() < 1e-12
    assert np.abs(shifted[1] - plain[1]).max() > 1e-6  # dk moves too
