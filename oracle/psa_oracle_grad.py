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
    return num / den, (m + torch.log(den)).squeeze(1)


def forward(q, k, v, row_ptr, col_idx, causal: bool, block_size: int = 64, with_lse: bool = False):
    """The 0th-order output [B, H, N, d] as a differentiable function of
    torch fp64 tensors q, k, v (the block lists fixed); with ``with_lse``
    also its lse [B, H, N] (natural log of the denominator)."""
    B, H, N, d = q.shape
    bs = block_size
    M = N // bs
    kbar = k.reshape(B, H, M, bs, d).mean(dim=3)
    vsum = v.reshape(B, H, M, bs, d).sum(dim=3)
    rows, lses = [], []
    for b in range(B):
        for h in range(H):
            for I in range(M):
                r = (b * H + h) * M + I
                o, l = _unit(q, k, v, kbar, vsum, col_idx[row_ptr[r]:row_ptr[r + 1]], b, h, I, causal, bs)
                rows.append(o)
                lses.append(l)
    out = torch.stack(rows).reshape(B, H, N, d)
    if with_lse:
        return out, torch.stack(lses).reshape(B, H, N)
    return out


def backward(q, k, v, row_ptr, col_idx, causal: bool, dout, block_size: int = 64, out_for_delta=None):
    """(dq, dk, dv) = the gradient of sum(out * dout), as float64 numpy arrays.

    ``out_for_delta``: the output a backward pass is given in place of the
    exact one.  Softmax backward passes form D_i = dout_i . out_i from that
    given output; with out' = out + e, D shifts by delta_i = dout_i . e_i, which
    moves every score gradient by -p_ij delta_i (-b pi_iJ delta_i for a
    pseudo-key).  Since d lse_i / d z_ij = p_ij (and b pi_iJ for a pseudo-key),
    those gradients are exactly the gradient of
    sum(out * dout) - sum_i delta_i lse_i with delta held constant, which is
    what is returned then."""
    t = [torch.tensor(np.asarray(x, dtype=np.float64), requires_grad=True) for x in (q, k, v)]
    out, lse = forward(*t, row_ptr, col_idx, causal, block_size, with_lse=True)
    g = torch.tensor(np.asarray(dout, dtype=np.float64))
    loss = (out * g).sum()
    if out_for_delta is not None:
        delta = (g * (torch.tensor(np.asarray(out_for_delta, dtype=np.float64)) - out.detach())).sum(dim=-1)
        loss = loss - (delta * lse).sum()
    loss.backward()
    return tuple(x.grad.numpy() for x in t)
