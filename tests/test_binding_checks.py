"""The Python binding checks every tensor against the problem's dimensions
before a pointer crosses the C ABI (which takes plain pointers and sizes
them from B, H, N, d): a smaller or differently typed buffer would otherwise
be read or written past its end on the device.  Host-only: the checks fire
on CPU tensors before the device check."""
import pytest
import torch

from block_sparse_attention_psa_b200 import psa

B, H, N, d = 1, 2, 256, 64
M = N // 64


def _qkv():
    return [torch.zeros(B, H, N, d, dtype=torch.bfloat16) for _ in range(3)]


def _stats():
    return [torch.zeros(B, H, M, d, dtype=torch.float32) for _ in range(3)]


def _lists():
    return torch.zeros(B * H * M + 1, dtype=torch.int32), torch.zeros(B * H * M, dtype=torch.int32)


def test_pool_inputs_and_outputs():
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="k must have shape"):
        psa.psa_pool(q, torch.zeros(B, H, N // 2, d, dtype=torch.bfloat16), v)
    with pytest.raises(ValueError, match="v must be torch.bfloat16"):
        psa.psa_pool(q, k, v.float())
    with pytest.raises(ValueError, match="vsum must have shape"):
        psa.psa_pool(q, k, v, out=(*_stats()[:2], torch.zeros(B, H, M - 1, d)))
    with pytest.raises(ValueError, match="CUDA device"):
        psa.psa_pool(q, k, v)   # well formed: only the device is wrong here


def test_router_inputs_and_outputs():
    qbar, kbar, _ = _stats()
    with pytest.raises(ValueError, match="kbar must have shape"):
        psa.psa_route_topk(qbar, torch.zeros(B, H, M + 1, d), 0.5)
    with pytest.raises(ValueError, match="float32"):
        psa.psa_route_thresh(qbar.double(), kbar, 0.5)
    out = (torch.zeros(B * H * M, dtype=torch.int32), torch.zeros(64, dtype=torch.int32),
           torch.zeros(1, dtype=torch.int32), torch.zeros(B * H * M))
    with pytest.raises(ValueError, match="row_ptr needs at least"):
        psa.psa_route_topk(qbar, kbar, 0.5, out=out)
    small_ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="ws needs at least"):
        psa.psa_route_thresh_prob(qbar, kbar, 0.5, ws=small_ws)
    with pytest.raises(ValueError, match="ws must be torch.uint8"):
        psa.psa_route_topk(qbar, kbar, 0.5, ws=torch.zeros(1 << 20, dtype=torch.int32))


def test_attention_inputs_and_outputs():
    q, k, v = _qkv()
    _, kbar, vsum = _stats()
    rp, ci = _lists()
    with pytest.raises(ValueError, match="kbar must have shape"):
        psa.psa_attn(q, k, v, kbar[:, :1], vsum, rp, ci)
    with pytest.raises(ValueError, match="col_idx must be torch.int32"):
        psa.psa_attn(q, k, v, kbar, vsum, rp, ci.long())
    with pytest.raises(ValueError, match="row_max needs at least"):
        psa.psa_attn(q, k, v, kbar, vsum, rp, ci, row_max=torch.zeros(3))
    with pytest.raises(ValueError, match="lse must have shape"):
        psa.psa_attn(q, k, v, kbar, vsum, rp, ci, lse=torch.zeros(B, H, N - 1))
    with pytest.raises(ValueError, match="out must be torch.bfloat16"):
        psa.psa_dense(q, k, v, out=torch.zeros(B, H, N, d))
    with pytest.raises(ValueError, match="status must be torch.int32"):
        psa.psa_attn_noalloc(q, k, v, kbar, vsum, rp, ci, status=torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError, match="ws needs at least"):
        psa.psa_read_status(torch.zeros(8, dtype=torch.uint8))
