"""GPU parity of the first-order ("hyd") correction against the fp64 oracle.

PISA summary, "Why approximating unselected blocks keeps softmax intact" and
the FAQ "Why a global first-order correction?": every unselected block adds
e^{a_iJ} H^T q_i / sqrt(d) to the numerator, with one global statistic H per
head (read as the mean over the head's blocks of H_J = sum_j (k_j - kbar_J)
v_j^T).  The statistic is compared with ``global_deviation_stat`` of the
oracle's ``block_deviation_stats``; the output with ``attention_first_order``
fed the GPU's own block lists and the oracle's own statistic, at the
tolerances of the 0th-order parity tests."""

import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
from block_sparse_attention_psa_b200 import psa
from block_sparse_attention_psa_b200.inputs import WORKLOADS, make_qkv, workload_inputs
from tests.parity import MAX_ABS, MEAN_ABS, check_pool, check_routing, f64, sample_units

pytestmark = pytest.mark.gpu


def _oracle_stat(k, v):
    return O.global_deviation_stat(O.block_deviation_stats(f64(k), f64(v)))


def _check_stat(got, k, v):
    ref = _oracle_stat(k, v)
    got = f64(got)
    err = np.abs(got - ref).max()
    assert err <= 1e-4 * max(1.0, np.abs(ref).max()), f"statistic: max err {err}, scale {np.abs(ref).max()}"
    return ref


def _run(q, k, v, mode, param, causal=False, keep_first=False, lists=None):
    dq, dk, dv = (x.cuda() for x in (q, k, v))
    B, H, N, d = q.shape
    ws = psa.workspace(B, H, N, d)
    qbar, kbar, vsum = psa.psa_pool(dq, dk, dv)
    row_max = None
    if lists is not None:
        rp_np, ci_np = O._to_csr(lists)
        rp = torch.tensor(rp_np, dtype=torch.int32, device="cuda")
        ci = torch.tensor(ci_np if ci_np.size else [0], dtype=torch.int32, device="cuda")
        n = int(rp_np[-1])
    else:
        route = {"topk": psa.psa_route_topk, "thresh": psa.psa_route_thresh}[mode]
        args = (qbar, kbar, param, causal) if mode == "topk" else (qbar, kbar, param, causal, keep_first)
        rp, ci, nnz, row_max = route(*args, ws=ws)
        n = int(nnz.item())
    hstat = psa.psa_hyd_stat(dk, dv, kbar, vsum, ws=ws)
    out, lse = psa.psa_attn_hyd(dq, dk, dv, kbar, vsum, hstat, rp, ci, causal, ws=ws, want_lse=True,
                                row_max=row_max)
    out0, lse0 = psa.psa_attn(dq, dk, dv, kbar, vsum, rp, ci, causal, ws=psa.workspace(B, H, N, d),
                              want_lse=True, row_max=row_max)
    status = psa.psa_read_status(ws)
    torch.cuda.synchronize()
    return dict(qbar=qbar.cpu(), kbar=kbar.cpu(), vsum=vsum.cpu(), hstat=hstat.cpu(), out=out.cpu(), lse=lse.cpu(),
                out0=out0.cpu(), lse0=lse0.cpu(), row_ptr=rp.cpu().long().numpy(),
                col_idx=ci[:n].cpu().long().numpy(), nnz=n, status=status)


def _check_hyd(g, q, k, v, causal, units=None):
    assert g["status"] == psa.PSA_OK, psa.status_text(g["status"])
    B, H, N, d = q.shape
    M = N // 64
    if units is None:
        units = O.unit_rows(B, H, M)
    units = list(units)
    Href = _check_stat(g["hstat"], k, v)
    _, kbar, vsum = O.pool(f64(q), f64(k), f64(v))
    ref, ref_lse = O.attention_first_order(f64(q), f64(k), f64(v), kbar, vsum, g["row_ptr"], g["col_idx"], causal,
                                           Href, 64, units)
    out, lse = f64(g["out"]), f64(g["lse"])
    got = np.stack([out[b, h, I * 64:(I + 1) * 64] for (b, h, I) in units])
    got_lse = np.stack([lse[b, h, I * 64:(I + 1) * 64] for (b, h, I) in units])
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert err.max() <= MAX_ABS, f"max abs err {err.max()}"
    assert err.mean() <= MEAN_ABS, f"mean abs err {err.mean()}"
    lerr = np.abs(got_lse - ref_lse).max()
    assert lerr <= 1e-3 * max(1.0, np.abs(ref_lse).max()), f"lse err {lerr}"
    # the lse is the 0th-order one (the correction adds nothing to the denominator)
    assert torch.equal(g["lse"], g["lse0"])
    return err


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_statistic_and_output_ragged(d, causal):
    # M = 37: ragged query tiles of the correction (128 rows) and odd block counts
    q, k, v = make_qkv(2, 2, 37 * 64, d, "clustered", seed=31)
    g = _run(q, k, v, "topk", 0.15, causal)
    qbar, kbar, vsum = check_pool(g, q, k, v)
    check_routing(g, O.block_scores(qbar, kbar), "topk", 0.15, causal)
    _check_hyd(g, q, k, v, causal)


@pytest.mark.parametrize("d", [64, 128])
def test_threshold_routing(d):
    q, k, v = make_qkv(1, 3, 45 * 64, d, "clustered_slash", seed=32)
    g = _run(q, k, v, "thresh", 0.5, True, True)
    _check_hyd(g, q, k, v, True)


def test_correction_changes_the_output():
    # the correction is not a no-op: on keys spread around their block means
    # the 0th-order output misses the first-order oracle by more than the
    # tolerance, while the corrected output meets it
    q, k, v = make_qkv(1, 2, 40 * 64, 128, "iid", seed=33)
    g = _run(q, k, v, "topk", 0.1)
    _check_hyd(g, q, k, v, False)
    _, kbar, vsum = O.pool(f64(q), f64(k), f64(v))
    ref, _ = O.attention_first_order(f64(q), f64(k), f64(v), kbar, vsum, g["row_ptr"], g["col_idx"], False,
                                     _oracle_stat(k, v), 64)
    out0 = f64(g["out0"]).reshape(ref.shape)
    assert np.abs(out0 - ref).max() > MAX_ABS


def test_every_block_listed_leaves_the_output_unchanged():
    # density 1: no unselected block, w = 0 everywhere, out == psa_attn's
    q, k, v = make_qkv(1, 2, 20 * 64, 64, "clustered", seed=34)
    g = _run(q, k, v, "topk", 1.0)
    _check_hyd(g, q, k, v, False)
    assert torch.equal(g["out"], g["out0"])


def test_empty_lists_first_order_everywhere():
    # nothing listed: every candidate through the 0th- and first-order terms
    q, k, v = make_qkv(1, 2, 12 * 64, 128, "clustered", seed=35)
    lists = [np.zeros(0, dtype=np.int64) for _ in range(2 * 12)]
    g = _run(q, k, v, None, None, lists=lists)
    _check_hyd(g, q, k, v, False)


def test_statistic_many_chunks():
    # M = 1024 blocks over 4 heads: each head's blocks split over many CTAs and
    # summed in a fixed order
    q, k, v = make_qkv(1, 4, 1024 * 64, 64, "clustered", seed=36)
    dk, dv = k.cuda(), v.cuda()
    _, kbar, vsum = psa.psa_pool(q.cuda(), dk, dv)
    h1 = psa.psa_hyd_stat(dk, dv, kbar, vsum)
    h2 = psa.psa_hyd_stat(dk, dv, kbar, vsum)
    assert torch.equal(h1, h2)  # deterministic
    _check_stat(h1.cpu(), k, v)


def test_full_dit_video_hyd_sampled():
    w = WORKLOADS["dit_video_n32k"]
    q, k, v = workload_inputs("dit_video_n32k")
    g = _run(q, k, v, "topk", 0.15)
    qbar, kbar, vsum = check_pool(g, q, k, v)
    check_routing(g, O.block_scores(qbar, kbar), "topk", 0.15, False)
    _check_hyd(g, q, k, v, False, sample_units(w["B"], w["H"], w["N"] // 64, 40, seed=11, g=g))
