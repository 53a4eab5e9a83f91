"""psa_attn_noalloc: attention for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: plugins inside frameworks
whose device memory all comes from the framework's own pool, and real-time or
safety-critical loops that forbid any allocation after start-up.  The
no-allocation entry point keeps its scratch in a fixed array inside the
library instead.  These tests call it through the C ABI twice in a row and
check each result against the workspace entry point psa_attn on the same
inputs: both run the same kernels on the same data, so the outputs, the lse
and the device status must be bit-identical.  The file sorts last so that a
run that stops at the first failure has already run every other test.
"""

import ctypes

import pytest
import torch

from block_sparse_attention_psa_b200 import psa
from block_sparse_attention_psa_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(q, k, v, kbar, vsum, row_ptr, col_idx, col_cap, row_max, causal):
    B, H, N, d = q.shape
    out = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    rc = psa.lib().psa_attn_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(kbar), _ptr(vsum), _ptr(row_ptr), _ptr(col_idx), col_cap, _ptr(row_max),
        B, H, N, d, 64, int(causal), _ptr(out), _ptr(lse), _ptr(status),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == psa.PSA_OK, psa.status_text(rc)
    torch.cuda.synchronize()
    return out, lse, int(status.item())


def _workspace_call(q, k, v, kbar, vsum, row_ptr, col_idx, col_cap, row_max, causal):
    B, H, N, d = q.shape
    ws = psa.workspace(B, H, N, d)
    out = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    rc = psa.lib().psa_attn(
        _ptr(q), _ptr(k), _ptr(v), _ptr(kbar), _ptr(vsum), _ptr(row_ptr), _ptr(col_idx), col_cap, _ptr(row_max),
        B, H, N, d, 64, int(causal), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == psa.PSA_OK, psa.status_text(rc)
    return out, lse, psa.psa_read_status(ws)


def _problem(causal, d):
    q, k, v = (x.cuda() for x in make_qkv(1, 4, 96 * 64, d, "clustered", seed=21))
    qbar, kbar, vsum = psa.psa_pool(q, k, v)
    row_ptr, col_idx, nnz, row_max = psa.psa_route_topk(qbar, kbar, 0.15, causal)
    return q, k, v, kbar, vsum, row_ptr, col_idx, int(nnz.item()), row_max


@pytest.mark.parametrize("use_row_max", [False, True])
@pytest.mark.parametrize("causal,d", [(False, 128), (True, 64)])
def test_no_alloc_matches_workspace_entry_point(causal, d, use_row_max):
    # with and without the router's row maxima as the softmax stabiliser
    q, k, v, kbar, vsum, row_ptr, col_idx, nnz, row_max = _problem(causal, d)
    rm = row_max if use_row_max else None
    ref, ref_lse, ref_status = _workspace_call(q, k, v, kbar, vsum, row_ptr, col_idx, col_idx.numel(), rm, causal)
    assert ref_status == psa.PSA_OK
    for call in range(2):
        out, lse, status = _noalloc(q, k, v, kbar, vsum, row_ptr, col_idx, col_idx.numel(), rm, causal)
        assert status == psa.PSA_OK, f"call {call}: device status {status}"
        assert torch.equal(out, ref), f"call {call}: output differs from psa_attn"
        assert torch.equal(lse, ref_lse), f"call {call}: lse differs from psa_attn"


def test_no_alloc_reports_a_cut_block_list():
    # col_capacity below the lists' total: rows whose row_ptr range leaves the
    # buffer are treated as empty, PSA_ERR_CSR reaches the caller's status
    # word, and the other rows are as psa_attn computes them with the same cut
    q, k, v, kbar, vsum, row_ptr, col_idx, nnz, row_max = _problem(False, 128)
    cap = nnz // 2
    ref, ref_lse, ref_status = _workspace_call(q, k, v, kbar, vsum, row_ptr, col_idx, cap, row_max, False)
    assert ref_status == psa.PSA_ERR_CSR
    for call in range(2):
        out, lse, status = _noalloc(q, k, v, kbar, vsum, row_ptr, col_idx, cap, row_max, False)
        assert status == psa.PSA_ERR_CSR, f"call {call}: device status {status}"
        assert torch.equal(out, ref) and torch.equal(lse, ref_lse), f"call {call}"
    # and a call with the whole list afterwards is clean again (the status word
    # of the shared array starts at zero on every call)
    out, lse, status = _noalloc(q, k, v, kbar, vsum, row_ptr, col_idx, col_idx.numel(), row_max, False)
    assert status == psa.PSA_OK


def test_no_alloc_rejects_shapes_beyond_its_scratch():
    # B*H*M*d bf16 pairs beyond 16 MiB: rejected on the host, nothing launched
    L = psa.lib()
    fake = ctypes.c_void_p(1 << 20)
    rc = L.psa_attn_noalloc(fake, fake, fake, fake, fake, fake, fake, 1 << 20, None, 1, 64, 65536, 128, 64, 0,
                            fake, None, None, None)
    assert rc == psa.PSA_ERR_CAPACITY
