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

`backward_chunked` takes the same gradients with bounded memory for full-size graphs: the
target rows are visited in groups whose edge lists fit a budget, each group's outputs are
differentiated with respect to Q, K, V, the gate logits and S, z held as leaves, and the
chain rule is then finished by autograd through the statistics and the projections.  It
runs the very same formula code (`rows_output`) and is tied to `backward` by a CPU test.
"""
from __future__ import annotations

import numpy as np
import torch


def _t(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float64))


def statistics(K, V):
    """S_h = sum_j phi(k_j) v_j^T and z_h = sum_j phi(k_j) over all rows, phi = elu + 1
    (Key formulas); K, V [N, H, r]."""
    phiK = torch.nn.functional.elu(K) + 1.0
    return torch.einsum("jha,jhc->hac", phiK, V), phiK.sum(0)


def rows_output(Q, K, V, t, S, z, b_g, eps, dst, src, r):
    """Y of a group of target rows ([n, H*r]): Q [n, H, r] and t [n] are the group's rows,
    K, V [N, H, r] every node's, dst [E'] the group-local target of each edge and src [E']
    its source node.  Local branch: softmax of q_i . k_j / sqrt(r) over the row's edges,
    weights on v_j; global branch phi(q_i)^T S / (phi(q_i)^T z + eps); gate
    sigmoid(t_i + b_g); blend."""
    n, H = Q.shape[0], Q.shape[1]
    s = (Q[dst] * K[src]).sum(-1) / np.sqrt(r)                       # [E', H]
    m = torch.full((n, H), -np.inf, dtype=torch.float64)
    if s.shape[0]:
        m = m.scatter_reduce(0, dst[:, None].expand(-1, H), s.detach(), "amax", include_self=True)
    p = torch.exp(s - m[dst])
    l = torch.zeros(n, H, dtype=torch.float64).index_add(0, dst, p)
    w = p / l[dst]
    L = torch.zeros(n, H, r, dtype=torch.float64).index_add(0, dst, w[..., None] * V[src])
    phiQ = torch.nn.functional.elu(Q) + 1.0
    G = torch.einsum("iha,hac->ihc", phiQ, S) / (torch.einsum("iha,ha->ih", phiQ, z) + eps)[..., None]
    g = torch.sigmoid(t + b_g)[:, None, None]
    return (g * L + (1.0 - g) * G).reshape(n, H * r)


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
    S, z = statistics(K, V)
    return rows_output(Q, K, V, t, S, z, b_g, eps, dst, src, r)


NAMES = ("dX", "dW_Q", "dW_K", "dW_V", "dw_g", "db_g")


def backward(X, W_Q, W_K, W_V, w_g, b_g, eps, row_ptr, col_idx, H, r, dY):
    """Gradients of sum(Y * dY) with respect to X, W_Q, W_K, W_V, w_g, b_g (float64)."""
    params = [_t(a).requires_grad_(True) for a in (X, W_Q, W_K, W_V, w_g)]
    bg = torch.tensor(float(b_g), dtype=torch.float64, requires_grad=True)
    Y = forward_torch(*params, bg, float(eps), row_ptr, col_idx, H, r)
    grads = torch.autograd.grad(Y, params + [bg], _t(dY))
    out = {k: g.numpy() for k, g in zip(NAMES, grads)}
    out["Y"] = Y.detach().numpy()
    return out


def _groups(row_ptr, max_edges, max_rows):
    """Consecutive row ranges [a, b) holding at most max_edges CSR entries and max_rows rows
    each (a single heavier row forms a group of its own)."""
    N = row_ptr.shape[0] - 1
    a = 0
    while a < N:
        b = int(np.searchsorted(row_ptr, row_ptr[a] + max_edges, side="right")) - 1
        b = min(max(b, a + 1), a + max_rows, N)
        yield a, b
        a = b


def backward_chunked(X, W_Q, W_K, W_V, w_g, b_g, eps, row_ptr, col_idx, H, r, dY,
                     max_edges=1 << 18, max_rows=1 << 16):
    """The gradients of `backward` (same names, float64) with the edge-level work done one
    group of target rows at a time, so memory stays bounded on full-size graphs."""
    params = [_t(a).requires_grad_(True) for a in (X, W_Q, W_K, W_V, w_g)]
    Xp, WQ, WK, WV, wg = params
    bg = torch.tensor(float(b_g), dtype=torch.float64, requires_grad=True)
    N = Xp.shape[0]
    proj = [Xp @ WQ, Xp @ WK, Xp @ WV, Xp @ wg]
    Q, K, V, t = (p.detach().requires_grad_(True) for p in proj)
    Sf, zf = statistics(K.view(N, H, r), V.view(N, H, r))
    S, z = Sf.detach().requires_grad_(True), zf.detach().requires_grad_(True)
    rp = np.asarray(row_ptr, dtype=np.int64)
    col = np.asarray(col_idx, dtype=np.int64)
    dYt = _t(dY)
    for a, b in _groups(rp, max_edges, max_rows):
        dst = torch.as_tensor(np.repeat(np.arange(b - a), np.diff(rp[a:b + 1])))
        src = torch.as_tensor(col[rp[a]:rp[b]])
        Yc = rows_output(Q.view(N, H, r)[a:b], K.view(N, H, r), V.view(N, H, r), t[a:b], S, z, bg,
                         float(eps), dst, src, r)
        (Yc * dYt[a:b]).sum().backward()
    zero = torch.zeros
    gS = S.grad if S.grad is not None else zero(S.shape, dtype=torch.float64)
    gz = z.grad if z.grad is not None else zero(z.shape, dtype=torch.float64)
    torch.autograd.backward([Sf, zf], [gS, gz])       # adds the global terms into K.grad, V.grad
    leaf_grads = [x.grad if x.grad is not None else zero(x.shape, dtype=torch.float64) for x in (Q, K, V, t)]
    torch.autograd.backward(proj, leaf_grads)
    out = {k: (p.grad if p.grad is not None else zero(p.shape, dtype=torch.float64)).numpy()
           for k, p in zip(NAMES, params + [bg])}
    return out
