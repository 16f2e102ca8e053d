"""Oracle: gradients of the block-sparse attention output with respect to Q, K and V (fp64).

The backward pass of the fine stage. The pages train through the sparse backend (the
``video_sparse_attn_h3`` page's ``tile()`` gives a grad-tracking forward its own buffer, and training
compiles keep the Triton route) but print no backward formulas; what is computed here is the
derivative of the forward definition in ``attention``. For a valid query row ``r`` of query tile
``i`` with kept keys ``C_i`` (the valid keys of its kept key tiles) the forward is::

    s_c = scale * q_r . k_c,    p = softmax over c in C_i of s,    o_r = sum_c p_c v_c

Given ``dO`` (the gradient of a scalar loss with respect to the output) the chain rule gives::

    dV_c += p_c dO_r
    dP_c  = dO_r . v_c
    dS_c  = p_c (dP_c - sum_c' p_c' dP_c')     (the softmax Jacobian; the sum equals dO_r . o_r)
    dQ_r  = scale * sum_c dS_c k_c
    dK_c += scale * dS_c q_r

Readings: the kept sets come from the coarse stage and are piecewise constant in Q and K, so no
gradient flows through the selection (or the pooling that feeds it). Pad query rows and pad keys
receive zero gradient (pad rows output zero whatever their inputs; pad keys have zero weight). In the
pruned-query variant a pruned row's output is a copy of its source row's, so its ``dO`` is added to
the source row's and its own ``q`` receives no gradient.

Test infrastructure, not the product: only the test suite may call it.
"""
from __future__ import annotations

import numpy as np

from .attention import TILE_ELEMS, _key_rows


def attend_rows_bwd(q_rows, k_rows, v_rows, do_rows, scale: float):
    """Gradients of dense softmax attention of ``q_rows [m, D]`` over ``k_rows, v_rows [n, D]``
    for the output gradient ``do_rows [m, D]``. Returns ``(dq [m, D], dk [n, D], dv [n, D])``."""
    q = q_rows.astype(np.float64)
    k = k_rows.astype(np.float64)
    v = v_rows.astype(np.float64)
    do = do_rows.astype(np.float64)
    logits = scale * (q @ k.T)
    e = np.exp(logits - logits.max(axis=1, keepdims=True))
    p = e / e.sum(axis=1, keepdims=True)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    delta = (do * o).sum(axis=1, keepdims=True)
    ds = p * (dp - delta)
    dq = scale * (ds @ k)
    dk = scale * (ds.T @ q)
    return dq, dk, dv


def block_sparse_attention_bwd(qt, kt, vt, vc, sets, scale: float, do, keep=None, src=None):
    """Gradients of ``attention.block_sparse_attention`` on padded tile-ordered tensors.

    Same arguments as the forward plus ``do`` (``[B, 64*nT, heads, D]``, the output gradient).
    Returns fp64 ``(dq, dk, dv)``, each ``[B, 64*nT, heads, D]``."""
    B, Lp, nh, D = qt.shape
    nT = Lp // TILE_ELEMS
    dq = np.zeros((B, Lp, nh, D), dtype=np.float64)
    dk = np.zeros((B, Lp, nh, D), dtype=np.float64)
    dv = np.zeros((B, Lp, nh, D), dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    for b in range(B):
        for h in range(nh):
            for i in range(nT):
                rows_k = _key_rows(sets[b][h][i], vc)
                n_q = int(vc[i])
                base = TILE_ELEMS * i
                if rows_k.size == 0 or n_q == 0:
                    continue
                if keep is None:
                    rows_q = base + np.arange(n_q)
                    g_out = do[b, rows_q, h]
                else:
                    # Output row rr is attended row src(rr): gather the gradients back onto them.
                    s = np.asarray(src[b, h, i][:n_q], dtype=np.int64)
                    g_blk = np.zeros((n_q, D), dtype=np.float64)
                    np.add.at(g_blk, s, do[b, base:base + n_q, h])
                    kk = np.nonzero(keep[b, h, i][:n_q])[0]
                    rows_q = base + kk
                    g_out = g_blk[kk]
                if rows_q.size == 0:
                    continue
                gq, gk, gv = attend_rows_bwd(qt[b, rows_q, h], kt[b, rows_k, h], vt[b, rows_k, h],
                                             g_out, scale)
                dq[b, rows_q, h] = gq
                dk[b, rows_k, h] += gk
                dv[b, rows_k, h] += gv
    return dq, dk, dv
