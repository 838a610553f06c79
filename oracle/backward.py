"""Float64 CPU oracle of the backward pass of HiLS attention (gradients through a fixed selection).

TEST INFRASTRUCTURE: imported only by the tests.  The product library has no backward pass yet.

"Hierarchical Sparse Attention Done Right" (arXiv 2607.02980v1), Sec. 3 Methodology, "Hierarchical
softmax": because the chunk retrieval scores enter the forward computation as fusion weights, the
language-model loss trains the landmarks and the retrieval through them; a chunk that is not selected
receives no gradient.  The selection itself is a discrete choice and is held fixed (taken from the
forward oracle).  Per head h of kv-group g and query i at position p, over the slots c of its
selection (the retrieved chunks and the own chunk):

    s_c   = scale * <q, L_c>                    w = softmax_c(s)
    l_j   = scale * <q, k_j>  (j in chunk c, j <= p)   P^c = softmax_j(l) inside chunk c
    o_c   = sum_j P^c_j v_j                     o = sum_c w_c o_c

and for an upstream gradient dO = dLoss/do the chain rule, step by step:

    dw_c  = <dO, o_c>                           ds_c = w_c (dw_c - sum_c' w_c' dw_c')
    dq   += scale * sum_c ds_c L_c              dL_c += scale * ds_c q
    do_c  = w_c dO
    dP_j  = <do_c, v_j>                         dl_j = P^c_j (dP_j - sum_j' P^c_j' dP_j')
    dq   += scale * sum_j dl_j k_j              dk_j += scale * dl_j q      dv_j += P^c_j do_c

Gradients of K, V and L accumulate over every (query, head) that touches the row.  Plain loops, no
blocking: a reader can check each line against the list above.
"""
import numpy as np

from . import oracle as orc

_MUTANT = 0


def set_mutant(m):
    """Test hook: plant mistake m (0 = none) so that the pins can be shown to catch it."""
    global _MUTANT
    _MUTANT = int(m)


def backward(Q, K, V, L, dO, C, k, q_offset=0, scale=None, sel=None):
    """Gradients (dQ, dK, dV, dL) of sum(O * dO) for the HiLS forward pass, float64.

    Q [B,H,N,d], K/V [B,Hkv,T,d], L [B,Hkv,ceil(T/C),d], dO [B,H,N,d].  sel [B,Hkv,N,k+1] (the
    forward oracle's selection, own chunk last) is computed when not given."""
    Q, K, V, L, dO = (np.asarray(a, dtype=np.float64) for a in (Q, K, V, L, dO))
    B, H, N, d = Q.shape
    Hkv, T = K.shape[1], K.shape[2]
    G = H // Hkv
    scale = orc.default_scale(d) if scale is None else scale
    if sel is None:
        sel = orc.forward(Q, K, V, L, C, k, q_offset=q_offset, scale=scale)["sel"]
    dQ, dK, dV, dL = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V), np.zeros_like(L)
    for b in range(B):
        for g in range(Hkv):
            for i in range(N):
                pos = q_offset + i
                slots = [int(c) for c in sel[b, g, i] if c >= 0]
                for h in range(g * G, (g + 1) * G):
                    q = Q[b, h, i]
                    # forward quantities of this (head, query)
                    s = np.array([scale * q @ L[b, g, c] for c in slots])
                    w = np.exp(s - s.max())
                    w /= w.sum()
                    rows, P, oc = [], [], []
                    for c in slots:
                        j0, j1 = c * C, min(c * C + C, pos + 1, T)
                        l = scale * (K[b, g, j0:j1] @ q)
                        pc = np.exp(l - l.max())
                        pc /= pc.sum()
                        rows.append((j0, j1))
                        P.append(pc)
                        oc.append(pc @ V[b, g, j0:j1])
                    g_o = dO[b, h, i]
                    # fusion weights
                    dw = np.array([g_o @ o for o in oc])
                    if _MUTANT == 21:      # planted: softmax backward without the weighted mean
                        ds = w * dw
                    elif _MUTANT == 22:    # planted: no gradient through the fusion weights
                        ds = np.zeros_like(w)
                    else:
                        ds = w * (dw - w @ dw)
                    for a, c in enumerate(slots):
                        dQ[b, h, i] += scale * ds[a] * L[b, g, c]
                        dL[b, g, c] += scale * ds[a] * q
                    # inside each chunk
                    for a, c in enumerate(slots):
                        j0, j1 = rows[a]
                        do_c = w[a] * g_o
                        dP = V[b, g, j0:j1] @ do_c
                        if _MUTANT == 23:  # planted: chunk softmax backward without the weighted mean
                            dl = P[a] * dP
                        else:
                            dl = P[a] * (dP - P[a] @ dP)
                        dQ[b, h, i] += scale * (dl @ K[b, g, j0:j1])
                        kscale = 1.0 if _MUTANT == 24 else scale   # planted: scale dropped on dK
                        dK[b, g, j0:j1] += kscale * np.outer(dl, q)
                        pv = P[a] if _MUTANT != 25 else P[a] / max(w[a], 1e-300)   # planted: w missing in dV
                        dV[b, g, j0:j1] += np.outer(pv, do_c)
    return dQ, dK, dV, dL
