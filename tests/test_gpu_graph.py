"""One whole step inside a CUDA graph.

The library launches every kernel of the forward path with programmatic
stream serialization, so a kernel may start while the one before it drains
and waits on the device for its inputs.  Captured into a CUDA graph those
launches become programmatic edges.  These tests capture pool, routing and
attention once and replay the graph: the output, the lse and the device status
must be bit-identical to the same calls made eagerly, and a replay on new
inputs copied into the captured buffers must match the eager calls on those
inputs.
"""

import pytest
import torch

from block_sparse_attention_psa_b200 import psa
from block_sparse_attention_psa_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


class _Step:
    def __init__(self, B, H, N, d, causal, density):
        dev = torch.device("cuda", 0)
        self.q = torch.empty(B, H, N, d, dtype=torch.bfloat16, device=dev)
        self.k = torch.empty_like(self.q)
        self.v = torch.empty_like(self.q)
        self.causal, self.density = causal, density
        self.ws = psa.workspace(B, H, N, d)
        M = N // 64
        self.stats = tuple(torch.empty(B, H, M, d, dtype=torch.float32, device=dev) for _ in range(3))
        cap = psa.psa_route_capacity(B, H, M, causal)
        self.csr = (torch.empty(B * H * M + 1, dtype=torch.int32, device=dev),
                    torch.empty(cap, dtype=torch.int32, device=dev),
                    torch.empty(1, dtype=torch.int32, device=dev),
                    torch.empty(B * H * M, dtype=torch.float32, device=dev))
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)

    def load(self, seed):
        q, k, v = make_qkv(*self.q.shape, gen="clustered", seed=seed)
        self.q.copy_(q)
        self.k.copy_(k)
        self.v.copy_(v)

    def run(self):
        qbar, kbar, vsum = psa.psa_pool(self.q, self.k, self.v, out=self.stats)
        psa.psa_route_topk(qbar, kbar, self.density, self.causal, out=self.csr, ws=self.ws)
        psa.psa_attn(self.q, self.k, self.v, kbar, vsum, self.csr[0], self.csr[1], self.causal, ws=self.ws,
                     out=self.out, lse=self.lse, row_max=self.csr[3])


@pytest.mark.parametrize("d,causal", [(128, False), (64, True)])
def test_step_replayed_from_a_cuda_graph_is_bit_identical(d, causal):
    st = _Step(1, 3, 64 * 96, d, causal, 0.2)
    expect = []
    for seed in (0, 1):
        st.load(seed)
        st.run()
        torch.cuda.synchronize()
        assert psa.psa_read_status(st.ws) == 0
        expect.append((st.out.clone(), st.lse.clone(), st.csr[0].clone()))
    st.load(0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        st.run()  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st.run()
    for seed in (0, 1):
        st.load(seed)
        st.out.zero_()
        st.lse.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert psa.psa_read_status(st.ws) == 0
        out, lse, rp = expect[seed]
        assert torch.equal(st.csr[0], rp)
        assert torch.equal(st.out, out)
        assert torch.equal(st.lse, lse)
    del g
