"""Gradients of the 0th-order block-sparse attention, fp64, on the CPU.

TEST INFRASTRUCTURE ONLY, like ``psa_oracle``: nothing on the product path
imports it, and it shares no code with the CUDA library.

The backward of the 0th-order version is the training-support variant the
PISA summary names (section "Minimal usage": the simplified 0th-order
version supports training).  With the block lists held fixed (routing is a
selection, not a differentiable function), the output of query i is

    out_i = num_i / den_i
    num_i = sum_{J in S_I} sum_{j in J, visible} e^{z_ij} v_j + sum_{J in U_I} e^{a_iJ} vsum_J
    den_i = sum_{J in S_I} sum_{j in J, visible} e^{z_ij}     + sum_{J in U_I} b e^{a_iJ}

with z_ij = q_i.k_j/sqrt(d), a_iJ = q_i.kbar_J/sqrt(d), kbar_J the mean of
the block's keys and vsum_J the sum of its values (the same definition as
``psa_oracle.attention``).  This module writes that forward with plain
PyTorch fp64 ops, pooling included, and takes dq, dk, dv by autograd: the
gradients reach k and v both through the exact terms and through kbar and
vsum.  A library primitive (autograd) serves as the differentiation step;
the pins in ``tests/test_oracle_grad.py`` hold it against central finite
differences and closed forms.
"""

from __future__ import annotations

import math

import numpy as np
import torch

__all__ = ["forward", "backward"]


def _unit(q, k, v, kbar, vsum, sel, b, h, I, causal, bs):
    """Output rows of query block I of head (b, h) (differentiable)."""
    M = q.shape[2] // bs
    d = q.shape[3]
    tau = 1.0 / math.sqrt(d)
    n_cand = I + 1 if causal else M
    sel = [int(J) for J in sel]
    Qi = q[b, h, I * bs:(I + 1) * bs]
    tok = [J * bs + t for J in sel for t in range(bs)]
    Kx, Vx = k[b, h, tok], v[b, h, tok]
    z = tau * (Qi @ Kx.T)
    if causal and tok:
        qi = torch.arange(bs)[:, None] + I * bs
        z = torch.where(torch.tensor(tok)[None, :] <= qi, z, torch.full_like(z, -math.inf))
    n_pseudo = I if causal else n_cand
    unsel = [J for J in range(n_pseudo) if J not in set(sel)]
    a = tau * (Qi @ kbar[b, h, unsel].T)
    VS = vsum[b, h, unsel]
    m = torch.cat([z, a], dim=1).max(dim=1, keepdim=True).values.detach()
    ez, ea = torch.exp(z - m), torch.exp(a - m)
    num = ez @ Vx + ea @ VS
    den = ez.sum(dim=1, keepdim=True) + bs * ea.sum(dim=1, keepdim=True)
    return num / den


def forward(q, k, v, row_ptr, col_idx, causal: bool, block_size: int = 64):
    """The 0th-order output [B, H, N, d] as a differentiable function of
    torch fp64 tensors q, k, v (the block lists fixed)."""
    B, H, N, d = q.shape
    bs = block_size
    M = N // bs
    kbar = k.reshape(B, H, M, bs, d).mean(dim=3)
    vsum = v.reshape(B, H, M, bs, d).sum(dim=3)
    rows = []
    for b in range(B):
        for h in range(H):
            for I in range(M):
                r = (b * H + h) * M + I
                rows.append(_unit(q, k, v, kbar, vsum, col_idx[row_ptr[r]:row_ptr[r + 1]], b, h, I, causal, bs))
    return torch.stack(rows).reshape(B, H, N, d)


def backward(q, k, v, row_ptr, col_idx, causal: bool, dout, block_size: int = 64):
    """(dq, dk, dv) = the gradient of sum(out * dout), as float64 numpy arrays."""
    t = [torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=True) for x in (q, k, v)]
    out = forward(*t, row_ptr, col_idx, causal, block_size)
    (out * torch.tensor(np.asarray(dout, dtype=np.float64))).sum().backward()
    return tuple(x.grad.numpy() for x in t)
