"""Pins for the CPU oracle: every check compares it with something other than itself.

Source of the definitions: explainer page of "Every Token Counts: Generalizing 16M Ultra-Long Context
in Large Language Models", "How It Works (Technically)" Steps 1-4 and "The algorithm, simplified".
The pages print no worked numeric example, so the pins are: a dense brute force and an exhaustive
subset search on tiny inputs, closed forms worked by hand, reductions to torch's scaled-dot-product
attention, invariants (causality, weights summing to one, independence from unselected chunks,
chunk-permutation equivariance, decode = last prefill row) and, for the backward, central finite
differences and torch autograd through a dense masked formulation.
"""
import math

import numpy as np
import pytest
import torch

from oracle import brute
from ultra_long_context_b200 import inputs


def bf16_arrays(B, H, T, D, chunk, seed, landmarks="iid"):
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, seed, chunk=chunk, landmarks=landmarks)
    return tuple(x.float().numpy() for x in (Q, K, V, L))


# ---------------------------------------------------------------------------------------------
# Step 2 + 3 + 4 against the dense brute force


@pytest.mark.parametrize("B,H,T,D,chunk,topk", [
    (1, 2, 48, 8, 4, 3),
    (2, 1, 70, 16, 8, 2),      # ragged: 70 = 8*8 + 6, the trailing partial chunk has no landmark
    (1, 1, 256, 16, 64, 2),
    (1, 2, 40, 4, 4, 20),      # topk larger than every n_t
    (1, 1, 24, 4, 4, 1),
])
def test_oracle_matches_dense_brute_force(oracle_mod, B, H, T, D, chunk, topk):
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=7 + T + D)
    scale = 1.0 / math.sqrt(D)
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, scale=scale)
    out_b, idx_b, w_b = brute.forward(Q, K, V, L, chunk, topk, scale)
    np.testing.assert_array_equal(r["sel_idx"].reshape(idx_b.shape), idx_b)
    np.testing.assert_allclose(r["out"].reshape(out_b.shape), out_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["sel_w"].reshape(w_b.shape), w_b, rtol=0, atol=1e-13)


def test_topk_is_the_best_subset(oracle_mod):
    """For distinct scores the top-K set is the K-subset with the largest score sum."""
    B, H, T, D, chunk, topk = 1, 2, 36, 8, 4, 3
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=11)
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk)
    rows = np.arange(B * H * T)
    S = oracle_mod.scores(Q, L, rows, chunk=chunk)
    checked = 0
    for i in rows:
        t = i % T
        n = (t + 1) // chunk
        if n <= topk:
            continue
        s = S[i, :n]
        assert len(set(s.tolist())) == n
        assert set(r["sel_idx"][i].tolist()) == brute.best_subset(list(s), topk)
        checked += 1
    assert checked > 20


def test_equal_scores_tie_to_lower_index(oracle_mod):
    """All landmarks equal: every admissible chunk ties; the stable sort keeps 0..k-1, weights 1/k."""
    B, H, T, D, chunk, topk = 1, 1, 64, 4, 8, 3
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=3)
    L[:] = L[:, :, :1, :]
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk)
    for t in range(T):
        n = (t + 1) // chunk
        k = min(n, topk)
        assert r["sel_idx"][t].tolist() == list(range(k)) + [-1] * (topk - k)
        if k:
            assert r["sel_w"][t, :k].tolist() == [1.0 / k] * k


def test_topk_one_is_argmax_and_plain_attention(oracle_mod):
    B, H, T, D, chunk = 1, 1, 32, 8, 4
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=5)
    scale = 1.0 / math.sqrt(D)
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=1)
    S = oracle_mod.scores(Q, L, np.arange(T), chunk=chunk)
    for t in range(chunk - 1, T):
        n = (t + 1) // chunk
        c = int(np.argmax(S[t, :n]))
        assert r["sel_idx"][t, 0] == c and r["sel_w"][t, 0] == 1.0
        q = torch.tensor(Q[0, 0, t], dtype=torch.float64).view(1, 1, D)
        kc = torch.tensor(K[0, 0, c * chunk:(c + 1) * chunk], dtype=torch.float64).view(1, chunk, D)
        vc = torch.tensor(V[0, 0, c * chunk:(c + 1) * chunk], dtype=torch.float64).view(1, chunk, D)
        ref = torch.nn.functional.scaled_dot_product_attention(q, kc, vc, scale=scale).view(D).numpy()
        np.testing.assert_allclose(r["out"][t], ref, rtol=0, atol=1e-13)


def test_single_chunk_reduces_to_sdpa(oracle_mod):
    """T = 64: rows 0..62 see no complete chunk (output 0); row 63 is exact attention over the chunk."""
    B, H, T, D, chunk = 1, 2, 64, 16, 64
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=9)
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=4)
    out = r["out"].reshape(B, H, T, D)
    idx = r["sel_idx"].reshape(B, H, T, 4)
    assert np.all(out[:, :, :63] == 0.0) and np.all(idx[:, :, :63] == -1)
    assert np.all(idx[:, :, 63] == np.array([0, -1, -1, -1]))
    q = torch.tensor(Q[:, :, 63:64], dtype=torch.float64)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, torch.tensor(K, dtype=torch.float64), torch.tensor(V, dtype=torch.float64), scale=1 / math.sqrt(D))
    np.testing.assert_allclose(out[:, :, 63], ref[:, :, 0].numpy(), rtol=0, atol=1e-12)


def test_all_chunks_selected_is_sdpa_mixture(oracle_mod):
    """topk >= N: O[t] = sum_c softmax_c(s[t, c]) * SDPA(q_t, K_c, V_c) over the admissible chunks."""
    B, H, T, D, chunk = 1, 1, 8 * 16, 16, 16
    N = T // chunk
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=13)
    scale = 1.0 / math.sqrt(D)
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=N)
    q = torch.tensor(Q[0, 0], dtype=torch.float64)                                  # [T, D]
    Kc = torch.tensor(K[0, 0], dtype=torch.float64).view(N, chunk, D)
    Vc = torch.tensor(V[0, 0], dtype=torch.float64).view(N, chunk, D)
    per_chunk = torch.nn.functional.scaled_dot_product_attention(
        q.unsqueeze(0).expand(N, T, D), Kc, Vc, scale=scale)                         # [N, T, D]
    s = scale * q @ torch.tensor(L[0, 0], dtype=torch.float64).T                     # [T, N]
    t = torch.arange(T)
    adm = (torch.arange(N)[None, :] + 1) * chunk - 1 <= t[:, None]
    w = torch.softmax(s.masked_fill(~adm, -math.inf), dim=-1).nan_to_num(0.0)
    ref = torch.einsum("tn,ntd->td", w, per_chunk).numpy()
    np.testing.assert_allclose(r["out"], ref, rtol=0, atol=1e-12)


def test_constant_values_per_chunk_give_weighted_sum(oracle_mod):
    """If V is constant inside every chunk, each chunk output is that constant: O = sum_j w_j v_j."""
    B, H, T, D, chunk, topk = 1, 1, 96, 8, 8, 4
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=17)
    N = T // chunk
    vconst = V[0, 0, ::chunk].copy()                                                # [N, D]
    V[0, 0] = np.repeat(vconst, chunk, axis=0)
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk)
    for t in range(T):
        k = min((t + 1) // chunk, topk)
        w = r["sel_w"][t, :k]
        if k:
            assert abs(w.sum() - 1.0) < 1e-15
        ref = (w[:, None] * vconst[r["sel_idx"][t, :k]]).sum(0) if k else np.zeros(D)
        np.testing.assert_allclose(r["out"][t], ref, rtol=0, atol=1e-14)
    assert N == 12


def test_hand_worked_example(oracle_mod):
    """A 4-token, D = 1, chunk = 2 example worked by hand (scale 1).

    Chunk 0 holds tokens 0-1 with keys (1, 2), values (1, 3); chunk 1 holds tokens 2-3 with keys
    (0, 1), values (2, 6). Landmarks: 1/2 and -1/2. Queries: 0.25, 1, 0.5, 1.
      t = 0: no chunk has ended -> 0.            t = 1, 2: only chunk 0 -> its attention output.
      t = 3: both chunks; top-1 picks chunk 0 (1/2 > -1/2); top-2 blends with w = softmax(1/2, -1/2).
    """
    Q = np.array([0.25, 1.0, 0.5, 1.0], np.float32).reshape(1, 1, 4, 1)
    K = np.array([1.0, 2.0, 0.0, 1.0], np.float32).reshape(1, 1, 4, 1)
    V = np.array([1.0, 3.0, 2.0, 6.0], np.float32).reshape(1, 1, 4, 1)
    L = np.array([0.5, -0.5], np.float32).reshape(1, 1, 2, 1)
    e = math.exp

    def o0(q):  # attention of query q inside chunk 0
        return (e(q * 1) * 1 + e(q * 2) * 3) / (e(q * 1) + e(q * 2))

    o1 = (e(0) * 2 + e(1) * 6) / (e(0) + e(1))  # chunk 1 with q = 1
    w0 = 1 / (1 + e(-1))
    expect_top1 = [0.0, o0(1.0), o0(0.5), o0(1.0)]
    expect_top2 = [0.0, o0(1.0), o0(0.5), w0 * o0(1.0) + (1 - w0) * o1]
    r1 = oracle_mod.forward(Q, K, V, L, chunk=2, topk=1, scale=1.0)
    r2 = oracle_mod.forward(Q, K, V, L, chunk=2, topk=2, scale=1.0)
    np.testing.assert_allclose(r1["out"][:, 0], expect_top1, rtol=1e-15, atol=0)
    np.testing.assert_allclose(r2["out"][:, 0], expect_top2, rtol=1e-15, atol=0)
    assert r2["sel_idx"].tolist() == [[-1, -1], [0, -1], [0, -1], [0, 1]]
    np.testing.assert_allclose(r2["sel_w"][3], [w0, 1 - w0], rtol=1e-15)
    assert r1["next_s"][3] == -0.5 and r2["next_s"][3] == -math.inf


# ---------------------------------------------------------------------------------------------
# Invariants


def test_future_positions_do_not_matter(oracle_mod):
    B, H, T, D, chunk, topk = 1, 2, 80, 8, 8, 3
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=19)
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk)
    cut = 43
    Q2, K2, V2, L2 = (x.copy() for x in (Q, K, V, L))
    rng = np.random.default_rng(0)
    for X in (Q2, K2, V2):
        X[:, :, cut:] = rng.standard_normal(X[:, :, cut:].shape).astype(np.float32)
    first_future_chunk = (cut + 1) // chunk          # chunks ending at or after the cut
    L2[:, :, first_future_chunk:] = rng.standard_normal(L2[:, :, first_future_chunk:].shape).astype(np.float32)
    r2 = oracle_mod.forward(Q2, K2, V2, L2, chunk=chunk, topk=topk)
    rows = np.array([bh * T + t for bh in range(B * H) for t in range(cut)])
    np.testing.assert_array_equal(r2["out"][rows], r["out"][rows])
    np.testing.assert_array_equal(r2["sel_idx"][rows], r["sel_idx"][rows])
    t_of = np.tile(np.arange(T), B * H)
    n_t = (t_of + 1) // chunk
    assert np.all(r["sel_idx"] < n_t[:, None])


def test_unselected_chunks_do_not_matter(oracle_mod):
    B, H, T, D, chunk, topk = 1, 1, 128, 8, 8, 4
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=23)
    t = T - 1
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, rows=[t])
    sel = set(r["sel_idx"][0].tolist())
    rng = np.random.default_rng(1)
    K2, V2, L2 = K.copy(), V.copy(), L.copy()
    q = Q[0, 0, t].astype(np.float64)
    for c in range(T // chunk):
        if c in sel:
            continue
        K2[0, 0, c * chunk:(c + 1) * chunk] = rng.standard_normal((chunk, D))
        V2[0, 0, c * chunk:(c + 1) * chunk] = rng.standard_normal((chunk, D))
        L2[0, 0, c] = (L[0, 0, c] - 4.0 * q / (q @ q)).astype(np.float32)   # lowers its score
    r2 = oracle_mod.forward(Q, K2, V2, L2, chunk=chunk, topk=topk, rows=[t])
    assert set(r2["sel_idx"][0].tolist()) == sel
    np.testing.assert_allclose(r2["out"], r["out"], rtol=0, atol=1e-14)


def test_chunk_permutation_equivariance(oracle_mod):
    """Permuting whole chunks (keys, values and landmark together) permutes the selection of the last
    token, which sees every chunk, and leaves its output unchanged."""
    B, H, T, D, chunk, topk = 1, 1, 96, 8, 8, 5
    N = T // chunk
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=29)
    perm = np.random.default_rng(2).permutation(N)
    Kp = K.reshape(1, 1, N, chunk, D)[:, :, perm].reshape(K.shape).copy()
    Vp = V.reshape(1, 1, N, chunk, D)[:, :, perm].reshape(V.shape).copy()
    Lp = L[:, :, perm].copy()
    t = T - 1
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, rows=[t])
    rp = oracle_mod.forward(Q, Kp, Vp, Lp, chunk=chunk, topk=topk, rows=[t])
    assert [int(perm[c]) for c in rp["sel_idx"][0]] == r["sel_idx"][0].tolist()
    np.testing.assert_allclose(rp["out"], r["out"], rtol=0, atol=1e-14)


def gather_chunks(X, sel, chunk):
    """X [B,H,T,D], sel [B,H,k] (-1 = none) -> [B*H, k, chunk, D] (zeros where empty)."""
    B, H, T, D = X.shape
    k = sel.shape[-1]
    out = np.zeros((B * H, k, chunk, D), np.float32)
    for bh in range(B * H):
        for j in range(k):
            c = sel.reshape(B * H, k)[bh, j]
            if c >= 0:
                out[bh, j] = X.reshape(B * H, T, D)[bh, c * chunk:(c + 1) * chunk]
    return out


def gather_landmarks(L, sel):
    BH, k = L.shape[0] * L.shape[1], sel.shape[-1]
    D = L.shape[-1]
    out = np.zeros((BH, k, D), np.float32)
    for bh in range(BH):
        for j in range(k):
            c = sel.reshape(BH, k)[bh, j]
            if c >= 0:
                out[bh, j] = L.reshape(BH, -1, D)[bh, c]
    return out


@pytest.mark.parametrize("T", [128, 130, 127])
def test_decode_equals_last_prefill_row(oracle_mod, T):
    """A decode step against a cache of T tokens is the prefill output of token T-1."""
    B, H, D, chunk, topk = 2, 2, 8, 8, 3
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=31)
    q = Q[:, :, T - 1].copy()
    sel = oracle_mod.decode_select(q, L, [T] * B, chunk=chunk, topk=topk)
    nsel = (sel["sel_idx"] >= 0).sum(-1).reshape(-1)
    out, w = oracle_mod.attend_gathered(q.reshape(B * H, D), gather_landmarks(L, sel["sel_idx"]),
                                        gather_chunks(K, sel["sel_idx"], chunk),
                                        gather_chunks(V, sel["sel_idx"], chunk), nsel)
    rows = [bh * T + T - 1 for bh in range(B * H)]
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, rows=rows)
    np.testing.assert_array_equal(sel["sel_idx"].reshape(B * H, topk), r["sel_idx"])
    np.testing.assert_allclose(out, r["out"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(w, r["sel_w"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(sel["sel_w"].reshape(B * H, topk), r["sel_w"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("lens,Hkv", [([128, 130], 2), ([127, 96], 1)])
def test_decode_all_scores_match_dense_scores(oracle_mod, lens, Hkv):
    """The decode's full score list (used to judge another selection on near-tie rows) is the dense
    score matrix's row of the token at cache_len - 1, NaN for chunks it does not see; its stable
    descending order starts with the selection."""
    B, H, D, chunk, topk, Tmax = 2, 2, 8, 8, 3, 136
    Q, K, V, L = bf16_arrays(B, H, Tmax, D, chunk, seed=33)
    L = L[:, :Hkv]
    q = np.stack([Q[b, :, lens[b] - 1] for b in range(B)])
    scale = 1 / math.sqrt(D)
    sel = oracle_mod.decode_select(q, L, lens, chunk=chunk, topk=topk, scale=scale, all_scores=True)
    S = brute.scores(Q, L, chunk, scale)
    for b in range(B):
        ref = S[b, :, lens[b] - 1]                                   # [H, N]
        np.testing.assert_allclose(sel["all_s"][b], ref, rtol=0, atol=1e-13)
        assert np.array_equal(np.isnan(sel["all_s"][b]), np.isnan(ref))
        for h in range(H):
            s = np.where(np.isnan(ref[h]), -np.inf, ref[h])
            n = int((~np.isnan(ref[h])).sum())
            order = np.argsort(-s, kind="stable")[:min(topk, n)]
            assert sel["sel_idx"][b, h, :len(order)].tolist() == order.tolist()


def test_decode_short_and_ragged_caches(oracle_mod):
    B, H, D, chunk, topk = 3, 1, 4, 8, 2
    q = np.random.default_rng(3).standard_normal((B, H, D)).astype(np.float32)
    Lc = np.random.default_rng(4).standard_normal((B, H, 4, D)).astype(np.float32)
    sel = oracle_mod.decode_select(q, Lc, [7, 8, 23], chunk=chunk, topk=topk)
    assert sel["sel_idx"][0, 0].tolist() == [-1, -1]           # no complete chunk
    assert sel["sel_idx"][1, 0].tolist() == [0, -1]            # one chunk: selected alone, w = 1
    assert sel["sel_w"][1, 0].tolist() == [1.0, 0.0]
    assert set(sel["sel_idx"][2, 0].tolist()) <= {0, 1}        # 23 tokens -> chunks 0 and 1 only
    assert (sel["sel_idx"][2, 0] >= 0).all()


def test_needle_is_retrieved(oracle_mod):
    q, Kc, Vc, Lc, lens, needle = inputs.decode_inputs(2, 4, 64 * 300, 128, seed=41)
    sel = oracle_mod.decode_select(q.float().numpy(), Lc.float().numpy(), lens.numpy(), topk=4)
    for b in range(2):
        assert (sel["sel_idx"][b, :, 0] == int(needle[b])).all()


# ---------------------------------------------------------------------------------------------
# Backward


def _grid_inputs(B, H, T, D, chunk, seed):
    """Values on a 1/8 grid in [-1, 1]: exact in float32, and x +- 2^-12 is exact as well."""
    rng = np.random.default_rng(seed)
    mk = lambda *s: (rng.integers(-8, 9, size=s) / 8.0).astype(np.float32)
    return mk(B, H, T, D), mk(B, H, T, D), mk(B, H, T, D), mk(B, H, T // chunk, D), mk(B, H, T, D)


def _loss_fixed_selection(oracle_mod, Q, K, V, L, G, sel_idx, chunk, scale):
    B, H, T, D = Q.shape
    k = sel_idx.shape[-1]
    si = sel_idx.reshape(B * H * T, k)
    rows_bh = np.repeat(np.arange(B * H), T)
    Kr = K.reshape(B * H, T, D)
    Vr = V.reshape(B * H, T, D)
    Lr = L.reshape(B * H, -1, D)
    Kg = np.zeros((B * H * T, k, chunk, D), np.float32)
    Vg = np.zeros_like(Kg)
    Lg = np.zeros((B * H * T, k, D), np.float32)
    for i in range(B * H * T):
        for j in range(k):
            c = si[i, j]
            if c >= 0:
                Kg[i, j] = Kr[rows_bh[i], c * chunk:(c + 1) * chunk]
                Vg[i, j] = Vr[rows_bh[i], c * chunk:(c + 1) * chunk]
                Lg[i, j] = Lr[rows_bh[i], c]
    out, _ = oracle_mod.attend_gathered(Q.reshape(-1, D), Lg, Kg, Vg, (si >= 0).sum(-1), scale=scale)
    return float((out * G.reshape(-1, D).astype(np.float64)).sum())


def test_backward_matches_central_differences(oracle_mod):
    B, H, T, D, chunk, topk = 1, 1, 16, 4, 4, 2
    scale = 0.5
    Q, K, V, L, G = _grid_inputs(B, H, T, D, chunk, seed=43)
    sel = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, scale=scale)["sel_idx"].reshape(B, H, T, topk)
    grads = oracle_mod.backward(Q, K, V, L, G, sel, chunk=chunk, scale=scale)
    h = 2.0 ** -12
    for X, g in zip((Q, K, V, L), grads):
        num = np.zeros(X.shape)
        for ix in np.ndindex(X.shape):
            x0 = X[ix]
            X[ix] = x0 + h
            fp = _loss_fixed_selection(oracle_mod, Q, K, V, L, G, sel, chunk, scale)
            X[ix] = x0 - h
            fm = _loss_fixed_selection(oracle_mod, Q, K, V, L, G, sel, chunk, scale)
            X[ix] = x0
            num[ix] = (fp - fm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=0, atol=2e-6 * max(1.0, np.abs(num).max()))
        assert np.abs(g).max() > 0


def dense_masked_hsa_torch(Q, K, V, L, sel_idx, chunk, scale, Qs=None, qk_norm=False):
    """HSA with a fixed selection as dense masked torch ops (every query x every chunk). Qs: separate
    retrieval queries (the fusion weights come from Qs . L), or None when Q also retrieves. K, V, L with
    fewer heads than Q are repeated over consecutive query heads (torch.repeat_interleave); qk_norm
    attends with torch.nn.functional.normalize(., eps=1e-6) of the query and the keys."""
    B, H, T, D = Q.shape
    G = H // K.shape[1]
    K, V, L = (x.repeat_interleave(G, dim=1) for x in (K, V, L))
    Qa = torch.nn.functional.normalize(Q, dim=-1, eps=1e-6) if qk_norm else Q
    if qk_norm:
        K = torch.nn.functional.normalize(K, dim=-1, eps=1e-6)
    N = L.shape[2]
    S = scale * torch.einsum("bhtd,bhnd->bhtn", Q if Qs is None else Qs, L)
    si = torch.as_tensor(sel_idx, dtype=torch.int64)
    hits = torch.zeros(B, H, T, N + 1, dtype=torch.int64)
    hits.scatter_add_(-1, torch.where(si >= 0, si, N), torch.ones_like(si))   # empty slots -> column N
    M = hits[..., :N] > 0
    W = torch.softmax(S.masked_fill(~M, -math.inf), dim=-1)
    W = torch.where(M.any(-1, keepdim=True), W, torch.zeros_like(W))
    Kc = K[:, :, : N * chunk].reshape(B, H, N, chunk, D)
    Vc = V[:, :, : N * chunk].reshape(B, H, N, chunk, D)
    P = torch.softmax(scale * torch.einsum("bhtd,bhnud->bhtnu", Qa, Kc), dim=-1)
    Obar = torch.einsum("bhtnu,bhnud->bhtnd", P, Vc)
    return torch.einsum("bhtn,bhtnd->bhtd", W, Obar)


@pytest.mark.parametrize("T,chunk,topk", [(96, 8, 3), (70, 8, 20)])
def test_backward_matches_torch_autograd(oracle_mod, T, chunk, topk):
    B, H, D = 2, 2, 8
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=47)
    G = np.random.default_rng(5).standard_normal((B, H, T, D)).astype(np.float32)
    scale = 1.0 / math.sqrt(D)
    sel = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk)["sel_idx"].reshape(B, H, T, topk)
    ts = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V, L)]
    out = dense_masked_hsa_torch(*ts, sel, chunk, scale)
    (out * torch.tensor(G, dtype=torch.float64)).sum().backward()
    grads = oracle_mod.backward(Q, K, V, L, G, sel, chunk=chunk, scale=scale)
    for t_, g in zip(ts, grads):
        np.testing.assert_allclose(g, t_.grad.numpy(), rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# Separate retrieval query (the pages' hsa_step takes a retrieval query q_slc and an attention query
# q_attn): Step 2 scores q_slc . L, Step 3 attends with q_attn, Step 4 weights by the retrieval scores


@pytest.mark.parametrize("B,H,T,D,chunk,topk", [(1, 2, 48, 8, 4, 3), (2, 1, 70, 16, 8, 2), (1, 2, 40, 4, 4, 20)])
def test_separate_retrieval_query_matches_dense_brute_force(oracle_mod, B, H, T, D, chunk, topk):
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=11 + T + D)
    Qs = bf16_arrays(B, H, T, D, chunk, seed=99 + T + D)[0]
    scale = 1.0 / math.sqrt(D)
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, scale=scale, Qs=Qs)
    out_b, idx_b, w_b = brute.forward(Q, K, V, L, chunk, topk, scale, Qs=Qs)
    np.testing.assert_array_equal(r["sel_idx"].reshape(idx_b.shape), idx_b)
    np.testing.assert_allclose(r["out"].reshape(out_b.shape), out_b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["sel_w"].reshape(w_b.shape), w_b, rtol=0, atol=1e-13)
    # and the retrieval query really decides: the selection differs from the one Q would make
    r_same = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, scale=scale)
    if topk < T // chunk:
        assert not np.array_equal(r["sel_idx"], r_same["sel_idx"])


def test_retrieval_query_equal_to_q_is_the_shared_path(oracle_mod):
    B, H, T, D, chunk, topk = 1, 2, 96, 8, 8, 3
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=5)
    G = np.random.default_rng(9).standard_normal((B, H, T, D)).astype(np.float32)
    a = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk)
    b = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, Qs=Q.copy())
    np.testing.assert_array_equal(a["sel_idx"], b["sel_idx"])
    np.testing.assert_array_equal(a["out"], b["out"])
    sel = a["sel_idx"].reshape(B, H, T, topk)
    dQ, dK, dV, dL = oracle_mod.backward(Q, K, V, L, G, sel, chunk=chunk)
    dQa, dK2, dV2, dL2, dQs = oracle_mod.backward(Q, K, V, L, G, sel, chunk=chunk, Qs=Q.copy())
    np.testing.assert_allclose(dQa + dQs, dQ, rtol=0, atol=1e-12)  # the two parts of one query's gradient
    for x, y in ((dK, dK2), (dV, dV2), (dL, dL2)):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("T,chunk,topk", [(96, 8, 3), (70, 8, 20)])
def test_separate_retrieval_query_backward_matches_torch_autograd(oracle_mod, T, chunk, topk):
    B, H, D = 2, 2, 8
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=53)
    Qs = bf16_arrays(B, H, T, D, chunk, seed=59)[0]
    G = np.random.default_rng(6).standard_normal((B, H, T, D)).astype(np.float32)
    scale = 1.0 / math.sqrt(D)
    sel = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, Qs=Qs)["sel_idx"].reshape(B, H, T, topk)
    ts = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V, L, Qs)]
    out = dense_masked_hsa_torch(*ts[:4], sel, chunk, scale, Qs=ts[4])
    (out * torch.tensor(G, dtype=torch.float64)).sum().backward()
    grads = oracle_mod.backward(Q, K, V, L, G, sel, chunk=chunk, scale=scale, Qs=Qs)
    for t_, g in zip(ts, grads):  # dQ (attention), dK, dV, dL, dQs (retrieval)
        np.testing.assert_allclose(g, t_.grad.numpy(), rtol=0, atol=1e-12)
        assert np.abs(g).max() > 0


# ---------------------------------------------------------------------------------------------
# Query-key normalisation (explainer, Step 3: the attention logits are norm(q_attn) . norm(K) / sqrt(d),
# norm = L2 normalisation, as in the per-token procedure's l2norm(q_attn), l2norm(K)). Reading: the
# retrieval scores of Step 2 stay unnormalised; norm(x) = x / max(||x||, 1e-6).


def normalized(x):
    return torch.nn.functional.normalize(torch.tensor(x, dtype=torch.float64), dim=-1, eps=1e-6).numpy()


@pytest.mark.parametrize("B,H,T,D,chunk,topk", [(1, 2, 48, 8, 4, 3), (2, 1, 70, 16, 8, 2), (1, 2, 40, 4, 4, 20)])
def test_qk_norm_matches_dense_brute_force(oracle_mod, B, H, T, D, chunk, topk):
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=13 + T + D)
    scale = 1.0 / math.sqrt(D)
    for Qs in (None, bf16_arrays(B, H, T, D, chunk, seed=17 + T)[0]):
        r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, scale=scale, Qs=Qs, qk_norm=True)
        out_b, idx_b, w_b = brute.forward(Q, K, V, L, chunk, topk, scale, Qs=Qs, qk_norm=True)
        np.testing.assert_array_equal(r["sel_idx"].reshape(idx_b.shape), idx_b)
        np.testing.assert_allclose(r["out"].reshape(out_b.shape), out_b, rtol=0, atol=1e-12)
        np.testing.assert_allclose(r["sel_w"].reshape(w_b.shape), w_b, rtol=0, atol=1e-13)


def test_qk_norm_is_attention_on_normalised_inputs(oracle_mod):
    """Normalising inside equals normalising the inputs first (torch's normalize) while the raw query
    still retrieves; the selection is the raw query's."""
    B, H, T, D, chunk, topk = 1, 2, 256, 16, 16, 4
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=23)
    a = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, qk_norm=True)
    b = oracle_mod.forward(normalized(Q), normalized(K), V, L, chunk=chunk, topk=topk, Qs=Q)
    np.testing.assert_array_equal(a["sel_idx"], b["sel_idx"])
    np.testing.assert_allclose(a["out"], b["out"], rtol=0, atol=2e-6)  # the normalised inputs pass as float32
    c = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk)
    np.testing.assert_array_equal(a["sel_idx"], c["sel_idx"])
    assert np.abs(a["out"] - c["out"]).max() > 1e-2


def test_qk_norm_ignores_query_and_key_lengths(oracle_mod):
    """Rescaling attention queries and keys by positive powers of two (exact in float) changes nothing
    once they are normalised; the retrieval query is held fixed."""
    B, H, T, D, chunk, topk = 1, 2, 128, 8, 8, 3
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=29)
    rng = np.random.default_rng(3)
    Q2 = Q * np.exp2(rng.integers(-3, 4, (B, H, T, 1))).astype(np.float32)
    K2 = K * np.exp2(rng.integers(-3, 4, (B, H, T, 1))).astype(np.float32)
    a = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, Qs=Q, qk_norm=True)
    b = oracle_mod.forward(Q2, K2, V, L, chunk=chunk, topk=topk, Qs=Q, qk_norm=True)
    np.testing.assert_array_equal(a["sel_idx"], b["sel_idx"])
    np.testing.assert_allclose(a["out"], b["out"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("separate", [False, True])
def test_qk_norm_backward_matches_torch_autograd(oracle_mod, separate):
    B, H, T, D, chunk, topk = 2, 2, 96, 8, 8, 3
    Q, K, V, L = bf16_arrays(B, H, T, D, chunk, seed=61)
    K[0, 1, 20] *= np.float32(2.0 ** -40)  # a key shorter than eps: the other branch of the norm's gradient
    Qs = bf16_arrays(B, H, T, D, chunk, seed=67)[0] if separate else None
    G = np.random.default_rng(8).standard_normal((B, H, T, D)).astype(np.float32)
    scale = 1.0 / math.sqrt(D)
    sel = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, Qs=Qs, qk_norm=True)["sel_idx"]
    sel = sel.reshape(B, H, T, topk)
    assert (sel == 2).any()  # chunk 2 holds the short key of head (0, 1)
    ts = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V, L)]
    qs_t = torch.tensor(Qs, dtype=torch.float64, requires_grad=True) if separate else None
    out = dense_masked_hsa_torch(*ts, sel, chunk, scale, Qs=qs_t, qk_norm=True)
    (out * torch.tensor(G, dtype=torch.float64)).sum().backward()
    grads = oracle_mod.backward(Q, K, V, L, G, sel, chunk=chunk, scale=scale, Qs=Qs, qk_norm=True)
    refs = ts + ([qs_t] if separate else [])
    for t_, g in zip(refs, grads):
        np.testing.assert_allclose(g, t_.grad.numpy(), rtol=1e-10, atol=1e-10)
        assert np.abs(g).max() > 0


# ---------------------------------------------------------------------------------------------
# Grouped heads ("How to Improve It" #2: several query heads per key/value head). Reading: consecutive
# query heads h share key head h // (H // Hkv), and each query head selects on its own.


def repeat_heads(x, G):
    return np.repeat(x, G, axis=1)


@pytest.mark.parametrize("H,Hkv", [(4, 2), (4, 1), (6, 3)])
def test_grouped_heads_equal_repeated_heads(oracle_mod, H, Hkv):
    B, T, D, chunk, topk = 2, 100, 8, 8, 3
    Q = bf16_arrays(B, H, T, D, chunk, seed=71)[0]
    _, K, V, L = bf16_arrays(B, Hkv, T, D, chunk, seed=73)
    G = H // Hkv
    Kr, Vr, Lr = repeat_heads(K, G), repeat_heads(V, G), repeat_heads(L, G)
    for qk_norm in (False, True):
        a = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, qk_norm=qk_norm)
        b = oracle_mod.forward(Q, Kr, Vr, Lr, chunk=chunk, topk=topk, qk_norm=qk_norm)
        for key in ("out", "sel_idx", "sel_w"):
            np.testing.assert_array_equal(a[key], b[key])
        dO = np.random.default_rng(4).standard_normal(Q.shape).astype(np.float32)
        sel = a["sel_idx"].reshape(B, H, T, topk)
        ga = oracle_mod.backward(Q, K, V, L, dO, sel, chunk=chunk, qk_norm=qk_norm)
        gb = oracle_mod.backward(Q, Kr, Vr, Lr, dO, sel, chunk=chunk, qk_norm=qk_norm)
        np.testing.assert_allclose(ga[0], gb[0], rtol=0, atol=1e-12)
        for x, y in zip(ga[1:], gb[1:]):  # a key head's gradient is the sum over its query heads
            np.testing.assert_allclose(x, y.reshape(B, Hkv, G, *y.shape[2:]).sum(2), rtol=0, atol=1e-12)
    q = Q[:, :, -1]
    lens = np.array([T, 37])
    s1 = oracle_mod.decode_select(q, L, lens, chunk=chunk, topk=topk)
    s2 = oracle_mod.decode_select(q, Lr, lens, chunk=chunk, topk=topk)
    for key in s1:
        np.testing.assert_array_equal(s1[key], s2[key])


@pytest.mark.parametrize("T,chunk,topk", [(96, 8, 3), (70, 8, 20)])
def test_grouped_heads_match_brute_force_and_autograd(oracle_mod, T, chunk, topk):
    B, H, Hkv, D = 1, 4, 2, 8
    Q = bf16_arrays(B, H, T, D, chunk, seed=79)[0]
    _, K, V, L = bf16_arrays(B, Hkv, T, D, chunk, seed=83)
    scale = 1.0 / math.sqrt(D)
    r = oracle_mod.forward(Q, K, V, L, chunk=chunk, topk=topk, scale=scale)
    out_b, idx_b, w_b = brute.forward(Q, K, V, L, chunk, topk, scale)
    np.testing.assert_array_equal(r["sel_idx"].reshape(idx_b.shape), idx_b)
    np.testing.assert_allclose(r["out"].reshape(out_b.shape), out_b, rtol=0, atol=1e-12)
    G = np.random.default_rng(10).standard_normal(Q.shape).astype(np.float32)
    sel = r["sel_idx"].reshape(B, H, T, topk)
    ts = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V, L)]
    out = dense_masked_hsa_torch(*ts, sel, chunk, scale)
    (out * torch.tensor(G, dtype=torch.float64)).sum().backward()
    for t_, g in zip(ts, oracle_mod.backward(Q, K, V, L, G, sel, chunk=chunk, scale=scale)):
        np.testing.assert_allclose(g, t_.grad.numpy(), rtol=0, atol=1e-12)
