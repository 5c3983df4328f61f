"""float64 reference gradients of the gated local-global graph-attention layer.

TEST INFRASTRUCTURE ONLY (like the rest of `oracle/`): used by `tests/` and the bench's
CPU leg, never by the library.

The forward of the method page ("Gated Local-Global Graph Attention", Key formulas) is
written out once more with torch float64 tensor operations over the edge list (per edge
and head: score, max-shifted exponential, segment sums by target), and its gradients are
taken with torch's autograd (a library primitive).  The segment maximum is held constant
(it cancels in the softmax; tinymesh "Target softmax" detaches it too).  This forward is
tied to the C oracle (`oracle.forward`) by the tests, and the gradients are pinned by
central finite differences of the C oracle itself.
"""
from __future__ import annotations

import numpy as np
import torch


def _t(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float64))


def forward_torch(X, W_Q, W_K, W_V, w_g, b_g, eps, row_ptr, col_idx, H, r):
    """Y [N, H*r] as a torch float64 function of the given tensors (which may require
    grad)."""
    N = X.shape[0]
    row_ptr = np.asarray(row_ptr, dtype=np.int64)
    dst = torch.as_tensor(np.repeat(np.arange(N), np.diff(row_ptr)))
    src = torch.as_tensor(np.asarray(col_idx, dtype=np.int64)[: row_ptr[-1]])
    Q = (X @ W_Q).view(N, H, r)
    K = (X @ W_K).view(N, H, r)
    V = (X @ W_V).view(N, H, r)
    t = X @ w_g
    # local branch: softmax of q_i . k_j / sqrt(r) over the CSR row, weights on v_j
    s = (Q[dst] * K[src]).sum(-1) / np.sqrt(r)                       # [E, H]
    m = torch.full((N, H), -np.inf, dtype=torch.float64)
    if s.shape[0]:
        m = m.scatter_reduce(0, dst[:, None].expand(-1, H), s.detach(), "amax", include_self=True)
    p = torch.exp(s - m[dst])
    l = torch.zeros(N, H, dtype=torch.float64).index_add(0, dst, p)
    w = p / l[dst]
    L = torch.zeros(N, H, r, dtype=torch.float64).index_add(0, dst, w[..., None] * V[src])
    # global branch: phi = elu + 1 linear attention over all nodes
    phiQ = torch.nn.functional.elu(Q) + 1.0
    phiK = torch.nn.functional.elu(K) + 1.0
    S = torch.einsum("jha,jhc->hac", phiK, V)
    z = phiK.sum(0)
    G = torch.einsum("iha,hac->ihc", phiQ, S) / (torch.einsum("iha,ha->ih", phiQ, z) + eps)[..., None]
    # gate and blend
    g = torch.sigmoid(t + b_g)[:, None, None]
    return (g * L + (1.0 - g) * G).reshape(N, H * r)


def backward(X, W_Q, W_K, W_V, w_g, b_g, eps, row_ptr, col_idx, H, r, dY):
    """Gradients of sum(Y * dY) with respect to X, W_Q, W_K, W_V, w_g, b_g (float64)."""
    params = [_t(a).requires_grad_(True) for a in (X, W_Q, W_K, W_V, w_g)]
    bg = torch.tensor(float(b_g), dtype=torch.float64, requires_grad=True)
    Y = forward_torch(*params, bg, float(eps), row_ptr, col_idx, H, r)
    grads = torch.autograd.grad(Y, params + [bg], _t(dY))
    names = ("dX", "dW_Q", "dW_K", "dW_V", "dw_g", "db_g")
    out = {k: g.numpy() for k, g in zip(names, grads)}
    out["Y"] = Y.detach().numpy()
    return out
