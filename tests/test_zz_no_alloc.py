"""psa_attn_noalloc: attention for callers that cannot allocate device memory.

Such callers (plugins inside frameworks whose device memory all comes from
the framework's own pool, real-time and safety-critical loops that forbid
allocation after start-up) cannot hand the library a workspace.  The no-allocation entry point keeps its scratch in a
fixed array inside the library instead.  This test calls it through the C
ABI twice in a row and checks each result against the workspace entry point
psa_attn on the same inputs, within the tolerance the other parity tests use.
The file sorts last so that a failing run has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_psa_b200 import psa
from block_sparse_attention_psa_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


@pytest.mark.parametrize("causal,d", [(False, 128), (True, 64)])
def test_no_alloc_matches_workspace_entry_point(causal, d):
    q, k, v = (x.cuda() for x in make_qkv(1, 4, 96 * 64, d, "clustered", seed=21))
    B, H, N, _ = q.shape
    qbar, kbar, vsum = psa.psa_pool(q, k, v)
    row_ptr, col_idx, _, row_max = psa.psa_route_topk(qbar, kbar, 0.15, causal)
    ws = psa.workspace(B, H, N, d)
    ref, ref_lse = psa.psa_attn(q, k, v, kbar, vsum, row_ptr, col_idx, causal, ws=ws, want_lse=True)
    assert psa.psa_read_status(ws) == psa.PSA_OK
    L = psa.lib()
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
        status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        rc = L.psa_attn_noalloc(
            ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
            ctypes.c_void_p(kbar.data_ptr()), ctypes.c_void_p(vsum.data_ptr()),
            ctypes.c_void_p(row_ptr.data_ptr()), ctypes.c_void_p(col_idx.data_ptr()), col_idx.numel(),
            None, B, H, N, d, 64, int(causal), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
            ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == psa.PSA_OK, psa.status_text(rc)
        torch.cuda.synchronize()
        assert int(status.item()) == psa.PSA_OK, f"call {call}: device status {int(status.item())}"
        err = (out.double() - ref.double()).abs()
        assert torch.isfinite(out).all(), f"call {call}: non-finite output"
        assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS, (call, err.max().item())
        lerr = (lse.double() - ref_lse.double()).abs().max().item()
        assert lerr <= 1e-3 * max(1.0, ref_lse.abs().max().item()), (call, lerr)


def test_no_alloc_rejects_shapes_beyond_its_scratch():
    # B*H*M*d bf16 pairs beyond 16 MiB: rejected on the host, nothing launched
    L = psa.lib()
    fake = ctypes.c_void_p(1 << 20)
    rc = L.psa_attn_noalloc(fake, fake, fake, fake, fake, fake, fake, 1 << 20, None, 1, 64, 65536, 128, 64, 0,
                            fake, None, None, None)
    assert rc == psa.PSA_ERR_CAPACITY
