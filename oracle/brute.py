"""Dense brute-force HSA in numpy, for tiny inputs only -- TEST INFRASTRUCTURE ONLY.

A second, structurally different formulation of the same definition as ``hsa_oracle.c``, used to pin
the C oracle on tiny shapes: it builds the full masked score matrix, ranks every row with numpy's
stable argsort, attends every query to EVERY chunk (dense, whether selected or not) and fuses with a
dense weight matrix that is zero off the selection. Source: explainer page of "Every Token Counts",
"How It Works (Technically)", Steps 2-4, and "The algorithm, simplified".
"""
import itertools

import numpy as np


def forward(Q, K, V, L, chunk, topk, scale, Qs=None, qk_norm=False, eps=1e-6):
    """Q [B, H, T, D], K, V [B, Hkv, T, D], L [B, Hkv, N, D] -> (out [B,H,T,D], sel_idx [B,H,T,topk],
    sel_w [B,H,T,topk]).

    Qs: separate retrieval queries (scores Qs . L), or None when Q also retrieves. Fewer key heads than
    query heads: each key head is repeated for its H // Hkv consecutive query heads. qk_norm: Step 3
    uses x / max(||x||, eps) for the query and the keys."""
    Q, K, V, L = (np.asarray(x, np.float64) for x in (Q, K, V, L))
    Qs = Q if Qs is None else np.asarray(Qs, np.float64)
    B, H, T, D = Q.shape
    G = H // K.shape[1]
    K, V, L = (np.repeat(x, G, axis=1) for x in (K, V, L))
    Qa = Q
    if qk_norm:
        Qa = Q / np.maximum(np.linalg.norm(Q, axis=-1, keepdims=True), eps)
        K = K / np.maximum(np.linalg.norm(K, axis=-1, keepdims=True), eps)
    N = T // chunk
    t = np.arange(T)
    admissible = (np.arange(N)[None, :] + 1) * chunk - 1 <= t[:, None]           # [T, N]
    S = scale * np.einsum("bhtd,bhnd->bhtn", Qs, L)                                # [B,H,T,N]
    S_masked = np.where(admissible, S, -np.inf)
    order = np.argsort(-S_masked, axis=-1, kind="stable")                         # ties -> lower index
    n_t = admissible.sum(-1)                                                       # [T]
    k_t = np.minimum(n_t, topk)
    sel_idx = np.full((B, H, T, topk), -1, np.int32)
    Wd = np.zeros((B, H, T, N))
    for i in range(T):
        k = int(k_t[i])
        if k == 0:
            continue
        sel = order[:, :, i, :k]                                                   # [B,H,k]
        sel_idx[:, :, i, :k] = sel
        s_sel = np.take_along_axis(S[:, :, i, :], sel, axis=-1)
        e = np.exp(s_sel - s_sel.max(-1, keepdims=True))
        np.put_along_axis(Wd[:, :, i, :], sel, e / e.sum(-1, keepdims=True), axis=-1)
    Kc = K[:, :, : N * chunk].reshape(B, H, N, chunk, D)
    Vc = V[:, :, : N * chunk].reshape(B, H, N, chunk, D)
    A = scale * np.einsum("bhtd,bhnud->bhtnu", Qa, Kc)                              # every query x every chunk
    P = np.exp(A - A.max(-1, keepdims=True))
    P /= P.sum(-1, keepdims=True)
    Obar = np.einsum("bhtnu,bhnud->bhtnd", P, Vc)
    out = np.einsum("bhtn,bhtnd->bhtd", Wd, Obar)
    sel_w = np.zeros((B, H, T, topk))
    valid = sel_idx >= 0
    sel_w[valid] = np.take_along_axis(Wd, np.where(valid, sel_idx, 0), axis=-1)[valid]
    return out, sel_idx, sel_w


def scores(Qs, L, chunk, scale):
    """Dense masked score matrix of Step 2: Qs [B, H, T, D], L [B, Hkv, N, D] -> [B, H, T, N] float64 with
    NaN where chunk c has not ended at or before token t (the same einsum as ``forward``)."""
    Qs, L = (np.asarray(x, np.float64) for x in (Qs, L))
    B, H, T, D = Qs.shape
    L = np.repeat(L, H // L.shape[1], axis=1)
    N = L.shape[2]
    t = np.arange(T)
    admissible = (np.arange(N)[None, :] + 1) * chunk - 1 <= t[:, None]
    S = scale * np.einsum("bhtd,bhnd->bhtn", Qs, L)
    return np.where(admissible, S, np.nan)


def best_subset(scores, k):
    """Top-k by exhaustive search: the k-subset with the largest score sum (distinct scores only)."""
    best, best_sum = None, -np.inf
    for comb in itertools.combinations(range(len(scores)), k):
        s = sum(scores[i] for i in comb)
        if s > best_sum:
            best, best_sum = comb, s
    return set(best)
