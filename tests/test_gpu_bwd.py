"""GPU parity of the backward of the 0th-order attention (f-4) against the
fp64 oracle's gradients (``oracle/psa_oracle_grad.py``: autograd of the
oracle's forward, pinned by central differences).

PISA summary, "Minimal usage": the simplified 0th-order version supports
training.  The block lists are the GPU router's (held fixed: routing is a
selection).  The backward takes the forward's bf16 output and forms
D_i = dout_i . out_i from it, so the oracle is asked for the gradients that
this given output defines (``out_for_delta``: the exact gradient plus the
shift of every score gradient by -p_ij dout_i . (out_given - out_exact)_i,
pinned in ``tests/test_oracle_grad.py``).  Tolerance, from the arithmetic:
every gradient is a sum of products with one bf16-rounded softmax weight (P
or the pseudo weight) and one bf16-rounded score gradient (dS or dA), 2^-9
relative each, plus the bf16 rounding of the result; with cancellation
between terms the element error is bounded relative to the tensor's scale,
not the element: max |err| <= 2e-2 max |ref| and mean |err| <= 2e-3 max
|ref|, per tensor."""

import ctypes

import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
import oracle.psa_oracle_grad as G
from block_sparse_attention_psa_b200 import psa
from block_sparse_attention_psa_b200.inputs import make_qkv
from tests.parity import f64

pytestmark = pytest.mark.gpu

MAX_REL = 2e-2
MEAN_REL = 2e-3


def _dout(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def _run(q, k, v, dout, causal, route=None, lists=None):
    dq_, dk_, dv_, do_ = (x.cuda() for x in (q, k, v, dout))
    B, H, N, d = q.shape
    ws = psa.workspace(B, H, N, d)
    qbar, kbar, vsum = psa.psa_pool(dq_, dk_, dv_)
    if lists is not None:
        rp_np, ci_np = O._to_csr(lists)
        rp = torch.tensor(rp_np, dtype=torch.int32, device="cuda")
        ci = torch.tensor(ci_np if ci_np.size else [0], dtype=torch.int32, device="cuda")
        n = int(rp_np[-1])
    else:
        mode, param = route
        if mode == "topk":
            rp, ci, nnz, _ = psa.psa_route_topk(qbar, kbar, param, causal, ws=ws)
        else:
            rp, ci, nnz, _ = psa.psa_route_thresh(qbar, kbar, param, causal, causal, ws=ws)
        n = int(nnz.item())
    out, lse = psa.psa_attn(dq_, dk_, dv_, kbar, vsum, rp, ci, causal, ws=ws, want_lse=True)
    fwd_status = psa.psa_read_status(ws)
    gq, gk, gv = psa.psa_attn_bwd(dq_, dk_, dv_, kbar, vsum, rp, ci, out, lse, do_, causal, ws=ws)
    status = psa.psa_read_status(ws)
    return dict(dq=gq.cpu(), dk=gk.cpu(), dv=gv.cpu(), out=out.cpu(), row_ptr=rp.cpu().long().numpy(),
                col_idx=ci[:n].cpu().long().numpy(), status=status, fwd_status=fwd_status)


def _check(g, q, k, v, dout, causal):
    assert g["fwd_status"] == psa.PSA_OK, psa.status_text(g["fwd_status"])
    assert g["status"] == psa.PSA_OK, psa.status_text(g["status"])
    ref = G.backward(f64(q), f64(k), f64(v), g["row_ptr"], g["col_idx"], causal, f64(dout),
                     out_for_delta=f64(g["out"]))
    for name, r in zip(("dq", "dk", "dv"), ref):
        got = f64(g[name])
        assert np.isfinite(got).all(), name
        scale = np.abs(r).max()
        err = np.abs(got - r)
        assert err.max() <= MAX_REL * scale, f"{name}: max err {err.max()} (scale {scale})"
        assert err.mean() <= MEAN_REL * scale, f"{name}: mean err {err.mean()} (scale {scale})"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_topk_gradients(d, causal):
    q, k, v = make_qkv(1, 2, 12 * 64, d, "clustered", seed=41)
    dout = _dout(q.shape, 42)
    g = _run(q, k, v, dout, causal, route=("topk", 0.25))
    _check(g, q, k, v, dout, causal)


@pytest.mark.parametrize("d", [64, 128])
def test_threshold_gradients_causal(d):
    # variable list lengths, block 0 and the diagonal forced, an odd count of
    # listing query blocks per key block (a pair with one block)
    q, k, v = make_qkv(1, 2, 13 * 64, d, "clustered_slash", seed=43)
    dout = _dout(q.shape, 44)
    g = _run(q, k, v, dout, True, route=("thresh", 0.5))
    _check(g, q, k, v, dout, True)


def test_empty_lists_and_full_lists():
    # nothing listed (every candidate through its pseudo-key) and everything
    # listed (dense softmax attention) on the same tensors
    q, k, v = make_qkv(1, 1, 10 * 64, 64, "iid", seed=45)
    dout = _dout(q.shape, 46)
    for lists in ([np.zeros(0, dtype=np.int64)] * 10, [np.arange(10)] * 10):
        g = _run(q, k, v, dout, False, lists=lists)
        _check(g, q, k, v, dout, False)


def test_dense_gradients_match_sdpa():
    # density 1: the gradients are those of textbook softmax attention
    q, k, v = make_qkv(1, 2, 9 * 64, 128, "iid", seed=47)
    dout = _dout(q.shape, 48)
    g = _run(q, k, v, dout, False, lists=[np.arange(9)] * 18)
    t = [torch.tensor(f64(x), requires_grad=True) for x in (q, k, v)]
    out = torch.nn.functional.scaled_dot_product_attention(*t)
    lse = torch.logsumexp(t[0] @ t[1].transpose(-1, -2) / np.sqrt(q.shape[-1]), dim=-1)
    # with D formed from the given (bf16) output, as the backward does
    delta = (torch.tensor(f64(dout)) * (torch.tensor(f64(g["out"])) - out.detach())).sum(-1)
    ((out * torch.tensor(f64(dout))).sum() - (delta * lse).sum()).backward()
    for name, x in zip(("dq", "dk", "dv"), t):
        r = x.grad.numpy()
        err = np.abs(f64(g[name]) - r)
        assert err.max() <= MAX_REL * np.abs(r).max(), (name, err.max())


def test_many_units_and_items_per_cta():
    # 3 heads x 100 blocks: several units and items per CTA, ragged pooled tiles
    q, k, v = make_qkv(1, 3, 100 * 64, 128, "clustered", seed=49)
    dout = _dout(q.shape, 50)
    g = _run(q, k, v, dout, False, route=("topk", 0.1))
    _check(g, q, k, v, dout, False)


def test_repeated_entry_is_reported():
    q, k, v = make_qkv(1, 1, 4 * 64, 64, "iid", seed=51)
    dout = _dout(q.shape, 52)
    lists = [np.array([0, 1])] * 3 + [np.array([2, 2])]
    g = _run(q, k, v, dout, False, lists=lists)
    assert g["status"] == psa.PSA_ERR_CSR


def test_full_dit_video_backward_conserves_dv_and_repeats():
    """The bench's backward configuration (DiT-video, 12 heads x 512 blocks,
    top-k 0.15): far too large for the fp64 oracle, so checked by a property
    that holds at any size and would fail for a missing or doubled term.  Each
    query's weights over its listed keys and its pooled blocks (64 tokens
    each) sum to 1, and d(vsum_J) reaches every token of block J, so per head
    and feature the sum of dv over all tokens equals the sum of dout over all
    queries.  Error budget: the bf16 weights (2^-9 relative) and the bf16 dv
    (2^-9 per element), random over 32768 tokens, give ~1e-3 of
    sqrt(sum dout^2); the bound is 2e-2 of it, while dropping the pooled
    blocks' share would miss by a large fraction of the sum itself.  A second
    call must give the same bytes (every unit's and item's arithmetic is
    fixed, whichever CTA draws it)."""
    from block_sparse_attention_psa_b200.inputs import workload_inputs

    q, k, v = (x.cuda() for x in workload_inputs("dit_video_n32k", seed=0))
    B, H, N, d = q.shape
    ws = psa.workspace(B, H, N, d)
    qbar, kbar, vsum = psa.psa_pool(q, k, v)
    rp, ci, nnz, row_max = psa.psa_route_topk(qbar, kbar, 0.15, False, ws=ws)
    out, lse = psa.psa_attn(q, k, v, kbar, vsum, rp, ci, False, ws=ws, want_lse=True, row_max=row_max)
    dout = _dout(q.shape, 53).cuda()
    first = psa.psa_attn_bwd(q, k, v, kbar, vsum, rp, ci, out, lse, dout, False, ws=ws)
    assert psa.psa_read_status(ws) == psa.PSA_OK
    first = tuple(t.clone() for t in first)
    second = psa.psa_attn_bwd(q, k, v, kbar, vsum, rp, ci, out, lse, dout, False, ws=ws)
    assert psa.psa_read_status(ws) == psa.PSA_OK
    for a, b in zip(first, second):
        assert torch.equal(a, b)
    dq, dk, dv = (t.double() for t in first)
    for t in (dq, dk, dv):
        assert torch.isfinite(t).all() and t.abs().max() > 0
    dsum = dout.double().sum(dim=2)       # [B, H, d]
    vsum_grad = dv.sum(dim=2)
    scale = dout.double().pow(2).sum(dim=2).sqrt()
    err = (vsum_grad - dsum).abs()
    assert (err <= 2e-2 * scale).all(), float((err / scale).max())
