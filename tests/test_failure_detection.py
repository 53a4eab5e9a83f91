"""Failure detection without a GPU fault: a bounded device wait that runs out.

The library's test hook makes the next attention launch withhold one
internal hand-off in its first block; every wait in the kernel is bounded and
abort-aware, so the launch must end by itself with PSA_ERR_TIMEOUT in the
status word, and the context must stay usable for the next call."""

import time

import numpy as np
import pytest
import torch

import oracle.psa_oracle as O
from block_sparse_attention_psa_b200 import psa
from block_sparse_attention_psa_b200.inputs import make_qkv
from tests.parity import check_output, f64


def test_stall_hook_arguments():
    L = psa.lib()
    assert L.psa_test_stall_next_attn(2) == psa.PSA_ERR_ARG
    assert L.psa_test_stall_next_attn(0) == psa.PSA_OK   # cancels nothing pending: fine


@pytest.mark.gpu
def test_bounded_wait_runs_out_and_context_survives():
    q, k, v = make_qkv(1, 2, 12 * 64, 64, "clustered", seed=20)
    dq, dk, dv = (x.cuda() for x in (q, k, v))
    B, H, N, d = q.shape
    qbar, kbar, vsum = psa.psa_pool(dq, dk, dv)
    rp, ci, nnz, row_max = psa.psa_route_topk(qbar, kbar, 0.25)
    ws = psa.workspace(B, H, N, d)
    psa.psa_test_stall_next_attn(True)
    t0 = time.perf_counter()
    psa.psa_attn(dq, dk, dv, kbar, vsum, rp, ci, ws=ws, row_max=row_max)
    status = psa.psa_read_status(ws)          # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert status == psa.PSA_ERR_TIMEOUT, psa.status_text(status)
    assert elapsed < 60.0, elapsed
    # the next call on the same context runs normally and is right
    out, lse = psa.psa_attn(dq, dk, dv, kbar, vsum, rp, ci, ws=ws, row_max=row_max, want_lse=True)
    status = psa.psa_read_status(ws)
    assert status == psa.PSA_OK, psa.status_text(status)
    n = int(nnz.item())
    g = dict(out=out.cpu(), lse=lse.cpu(), row_ptr=rp.cpu().long().numpy(), col_idx=ci[:n].cpu().long().numpy(),
             status=status)
    _, kb, vs = O.pool(f64(q), f64(k), f64(v))
    check_output(g, q, k, v, kb, vs, False)
