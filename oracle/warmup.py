"""fp64 oracle of the indexer's sparse warm-up objective and its gradients.

TEST INFRASTRUCTURE ONLY (see the package docstring): no product code calls it.

The pages (arXiv abstract "A.X K2 Technical Report"; archdb "A.X K2", stage
notes of the SGA adaptation) say the indexer is trained in a warm-up stage with
the backbone frozen, against its own sparse top-k selection rather than the
dense attention distribution, and later jointly with its loss down-weighted.
They print no formula.  The reading taken here, in the DSA style the token-
selection field names, for one query t with selection S_t (the indexer's own
top-k, ties to the lower position):

    p_t(s) = (1/H) sum_h softmax_{s in S_t}(z_{t,h,s}),   z = (q_h . kv_s) * 192^-0.5
             the frozen attention's distribution over the selected rows,
             averaged over the 64 heads (a target: no gradient flows into it)
    r_t(s) = softmax_{s in S_t}(score_t(s))
             the indexer's distribution over the same rows
    L      = sum_t KL(p_t || r_t) = sum_t sum_{s in S_t} p_t(s) (log p_t(s) - log r_t(s))

The selection itself is discrete and carries no gradient.  With
score_t(s) = sum_j w_tj ReLU(a_tjs), a_tjs = q_idx[t,j,:] . k_idx[s,:],
and g_ts = dL/dscore_t(s) = r_t(s) - p_t(s):

    dL/dw_tj         = sum_{s in S_t} g_ts ReLU(a_tjs)
    dL/dq_idx[t,j,:] = sum_{s in S_t} g_ts w_tj [a_tjs > 0] k_idx[s,:]
    dL/dk_idx[s,:]   = sum_t [s in S_t] sum_j g_ts w_tj [a_tjs > 0] q_idx[t,j,:]

(the ReLU passes no gradient at a_tjs = 0).  Everything is exact fp64 on the
bf16 input values; the selection comes from the pinned path oracle.
"""
from __future__ import annotations

import numpy as np

from . import SCALE, index_scores, topk
from .layer import to_f64


def attention_target(q, kv, idx_row, scale: float = SCALE) -> np.ndarray:
    """p over the selected rows of one query: q [H,576], kv [L,576], idx_row [k] (-1 = empty).
    Returns p [n_valid] in the order of the valid slots."""
    sel = idx_row[idx_row >= 0]
    z = (q @ kv[sel].T) * scale                      # [H, n]
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return (e / e.sum(axis=1, keepdims=True)).mean(axis=0)


def kl_to_softmax(p: np.ndarray, scores: np.ndarray) -> float:
    """KL(p || softmax(scores)) for one query, with 0 log 0 = 0."""
    s = scores - scores.max()
    log_r = s - np.log(np.exp(s).sum())
    nz = p > 0
    return float(np.sum(p[nz] * (np.log(p[nz]) - log_r[nz])))


def loss_on_selection(QI, Wt, KI, Q, KV, idx) -> dict:
    """The objective and its gradients for a given selection, on float64 values:
    QI [B,T,Hi,Di], Wt [B,T,Hi], KI [B,L,Di], Q [B,T,H,576], KV [B,L,576], idx [B,T,k]
    (-1 = empty slot)."""
    B, T = idx.shape[:2]
    per_query = np.zeros((B, T))
    g_qi, g_w, g_ki = np.zeros_like(QI), np.zeros_like(Wt), np.zeros_like(KI)
    for b in range(B):
        for t in range(T):
            sel = idx[b, t][idx[b, t] >= 0]
            if sel.size == 0:
                continue
            ks = KI[b, sel]                                   # [n, Di]
            a = QI[b, t] @ ks.T                               # [Hi, n]
            relu = np.maximum(a, 0.0)
            sc = Wt[b, t] @ relu                              # [n]
            p = attention_target(Q[b, t], KV[b], idx[b, t])
            per_query[b, t] = kl_to_softmax(p, sc)
            s = sc - sc.max()
            r = np.exp(s) / np.exp(s).sum()
            g = r - p                                         # dL/dscore over the selection
            g_w[b, t] = relu @ g
            act = (a > 0) * Wt[b, t][:, None] * g[None, :]    # [Hi, n]: g_s w_j [a_js > 0]
            g_qi[b, t] = act @ ks
            np.add.at(g_ki[b], sel, act.T @ QI[b, t])
    return {"loss": float(per_query.sum()), "per_query": per_query, "grad_q_idx": g_qi, "grad_w": g_w,
            "grad_k_idx": g_ki}


def warmup_loss(q_idx, w, k_idx, q, kv, q_pos, k: int = 2048, n_threads: int = 0) -> dict:
    """The warm-up objective and its gradients for queries [B,T] (bf16 inputs as in the path).

    The selection is the indexer's own top-k from the path oracle.  Returns loss
    (sum over queries), per_query [B,T], idx [B,T,k], and grad_q_idx [B,T,64,128],
    grad_w [B,T,64], grad_k_idx [B,L,128]."""
    pos = np.asarray(q_pos.cpu() if hasattr(q_pos, "cpu") else q_pos, dtype=np.int32)
    scores = index_scores(q_idx, w, k_idx, pos, n_threads=n_threads)
    idx = topk(scores, pos, k=k, n_threads=n_threads)
    res = loss_on_selection(to_f64(q_idx), to_f64(w), to_f64(k_idx), to_f64(q), to_f64(kv), idx)
    res["idx"] = idx
    return res
