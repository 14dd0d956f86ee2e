"""Comparison rules between the CUDA path and the CPU oracle.

Selection: the kept chunk SETS must be identical, except on rows where the oracle's K-th and
(K+1)-th scores differ by less than 1e-3; there the GPU's set is accepted when every chunk it kept
has an oracle score within 1e-3 of the oracle's K-th score (several answers are correct), and that
row's output is compared with the oracle evaluated on the GPU's (valid) set.
Outputs (bf16 from fp32 accumulation): max-abs <= 2e-2 and mean-abs <= 2e-3.
Fusion weights: max-abs <= 1e-3, matched by chunk id.
"""
import numpy as np

TIE = 1e-3
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
W_MAX_ABS = 1e-3


def compare_forward_rows(oracle_mod, gpu_out, gpu_idx, gpu_w, orc, Q, K, V, L, rows, chunk, scale, Qs=None,
                         qk_norm=False):
    """gpu_* and orc[...] are per-row arrays aligned with ``rows`` (flat (b*H+h)*T+t ids).

    Q, K, V, L: float32 host arrays [B, H, T, D] / [B, H, N, D] (needed for tie rows only); Qs: the
    separate retrieval queries when there are any (they decide the ties); qk_norm as in the oracle.
    Returns a dict of statistics; raises AssertionError on a violation.
    """
    gpu_out = np.asarray(gpu_out, np.float64)
    R = len(rows)
    same = np.zeros(R, bool)
    tie_rows = []
    for i in range(R):
        gs = set(int(c) for c in gpu_idx[i] if c >= 0)
        os_ = set(int(c) for c in orc["sel_idx"][i] if c >= 0)
        if gs == os_:
            same[i] = True
            continue
        assert len(gs) == len(os_), f"row {rows[i]}: {len(gs)} chunks kept, oracle keeps {len(os_)}"
        k = len(os_)
        s_k = orc["sel_s"][i, k - 1]
        gap = s_k - orc["next_s"][i]
        assert gap < TIE, f"row {rows[i]}: selection differs but the oracle's K/K+1 gap is {gap:.3g}"
        tie_rows.append(i)
    stats = dict(rows=R, tie_rows=len(tie_rows))
    # rows with identical sets: outputs and weights against the oracle
    d = np.abs(gpu_out[same] - orc["out"][same])
    if d.size:
        assert d.max() <= OUT_MAX_ABS, f"max-abs {d.max():.4g}"
        assert d.mean() <= OUT_MEAN_ABS, f"mean-abs {d.mean():.4g}"
        stats.update(max_abs=float(d.max()), mean_abs=float(d.mean()))
    wmax = 0.0
    for i in np.nonzero(same)[0]:
        og = {int(c): w for c, w in zip(orc["sel_idx"][i], orc["sel_w"][i]) if c >= 0}
        for c, w in zip(gpu_idx[i], gpu_w[i]):
            if c >= 0:
                wmax = max(wmax, abs(float(w) - og[int(c)]))
            else:
                assert w == 0.0
    assert wmax <= W_MAX_ABS, f"sel_w max-abs {wmax:.3g}"
    stats["w_max_abs"] = wmax
    # tie rows: validity of the GPU set, then its output against the oracle on that set
    if tie_rows:
        B, H, T, D = Q.shape
        G = H // K.shape[1]  # query heads per key head
        rr = np.asarray([rows[i] for i in tie_rows])
        S = oracle_mod.scores(Q if Qs is None else Qs, L, rr, chunk=chunk, scale=scale)
        topk = gpu_idx.shape[1]
        Lg = np.zeros((len(rr), topk, D), np.float32)
        Kg = np.zeros((len(rr), topk, chunk, D), np.float32)
        Vg = np.zeros_like(Kg)
        nsel = np.zeros(len(rr), np.int32)
        Qr = Q.reshape(-1, D)[rr]
        for n, i in enumerate(tie_rows):
            bh = rows[i] // T
            b, hk = bh // H, (bh % H) // G
            k = len([c for c in orc["sel_idx"][i] if c >= 0])
            s_k = orc["sel_s"][i, k - 1]
            kept = [int(c) for c in gpu_idx[i] if c >= 0]
            for j, c in enumerate(kept):
                assert S[n, c] >= s_k - TIE, f"row {rows[i]}: chunk {c} is not a near-tie choice"
                Lg[n, j] = L[b, hk, c]
                Kg[n, j] = K[b, hk, c * chunk:(c + 1) * chunk]
                Vg[n, j] = V[b, hk, c * chunk:(c + 1) * chunk]
            nsel[n] = len(kept)
        Qsr = None if Qs is None else Qs.reshape(-1, D)[rr]
        o, _ = oracle_mod.attend_gathered(Qr, Lg, Kg, Vg, nsel, scale=scale, qs=Qsr, qk_norm=qk_norm)
        dt = np.abs(gpu_out[tie_rows] - o)
        assert dt.max() <= OUT_MAX_ABS, f"tie rows max-abs {dt.max():.4g}"
    return stats


def grad_close(g, ref, name):
    """Backward tolerance: max-abs <= 2e-2 * max(1, |ref|max) and sum|g - ref| / sum|ref| <= 1e-2 (the
    relative part only where the reference is not identically zero)."""
    g = np.asarray(g, np.float64)
    err = np.abs(g - ref)
    scale = max(1.0, float(np.abs(ref).max()))
    assert err.max() <= 2e-2 * scale, f"{name}: max-abs {err.max():.4g} (scale {scale:.3g})"
    if not np.any(ref):
        return  # an exactly zero reference (e.g. dL where every fusion softmax has one chunk): max-abs only
    rel = err.sum() / np.abs(ref).sum()
    assert rel <= 1e-2, f"{name}: relative L1 {rel:.4g}"
    return float(err.max()), float(rel)
