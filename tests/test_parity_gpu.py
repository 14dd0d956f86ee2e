"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on seeded synthetic inputs."""
import ctypes
import math

import numpy as np
import pytest
import torch

from tests.parity import OUT_MAX_ABS, TIE, W_MAX_ABS, compare_forward_rows, grad_close
from ultra_long_context_b200 import hsa, inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def host(x):
    return x.float().cpu().numpy()


def run_forward_case(oracle_mod, B, H, T, D, topk, seed, landmarks="iid", rows=None):
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, seed, landmarks=landmarks, device=DEV)
    out, idx, w = hsa.hsa_forward(Q, K, V, L, topk)
    torch.cuda.synchronize()
    Qh, Kh, Vh, Lh = (host(x) for x in (Q, K, V, L))
    scale = 1.0 / math.sqrt(D)
    if rows is None:
        rows = np.arange(B * H * T)
    orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=scale, rows=rows)
    rr = torch.as_tensor(rows, device=DEV)
    g_out = host(out.reshape(-1, D)[rr])
    g_idx = idx.reshape(-1, topk)[rr].cpu().numpy()
    g_w = w.reshape(-1, topk)[rr].cpu().numpy()
    stats = compare_forward_rows(oracle_mod, g_out, g_idx, g_w, orc, Qh, Kh, Vh, Lh, rows, 64, scale)
    # invariants that hold for every row: causal selection, weights sum to one, padding
    t = rows % T
    n_t = np.minimum((t + 1) // 64, T // 64)
    assert np.all(g_idx < n_t[:, None])
    k_t = np.minimum(n_t, topk)
    assert np.all((g_idx >= 0).sum(1) == k_t)
    wsum = g_w.sum(1)
    assert np.allclose(wsum[k_t > 0], 1.0, atol=1e-5) and np.all(wsum[k_t == 0] == 0)
    assert np.all(g_out[k_t == 0] == 0)
    return stats, (Q, K, V, L, out, idx, w)


@pytest.mark.parametrize("B,H,T,D,topk,landmarks", [
    (1, 4, 4096, 64, 8, "iid"),            # the small benchmark workload, every row
    (2, 2, 4096 + 37, 128, 16, "chunk_mean"),  # ragged tail, several 128-row tiles
    (1, 2, 130, 64, 5, "iid"),             # topk above n_t; topk not a list length
    (1, 1, 50, 128, 4, "iid"),             # no complete chunk at all
    (1, 2, 1024, 128, 1, "iid"),
    (1, 2, 2048 + 64, 64, 32, "iid"),
    (1, 1, 64 * 40 + 63, 128, 3, "chunk_mean"),
    (1, 2, 2048 + 64, 128, 32, "chunk_mean"),  # the 32-wide selection list at head dim 128
    (1, 1, 3000, 128, 24, "iid"),              # kout below the list length, ragged tail
    # topk up to 64 (the per-token procedure's default): rows with n_t below and above topk, ragged tails
    (1, 2, 4096 + 640 + 37, 64, 64, "iid"),
    (1, 2, 4096 + 1000, 128, 48, "chunk_mean"),
    (2, 1, 64 * 70 + 11, 128, 64, "chunk_mean"),
    (1, 1, 3000, 64, 64, "iid"),               # n_t < topk on every row
])
def test_forward_matches_oracle(oracle_mod, B, H, T, D, topk, landmarks):
    stats, _ = run_forward_case(oracle_mod, B, H, T, D, topk, seed=100 + T + topk, landmarks=landmarks)
    assert stats["rows"] == B * H * T


@pytest.mark.parametrize("T,D,topk", [(640, 64, 4), (64 * 90 + 5, 128, 64), (64 * 70, 64, 48)])
def test_forward_equal_scores_keep_lowest_chunks(oracle_mod, T, D, topk):
    B, H = 1, 2
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, 7, device=DEV)
    L[:] = L[:, :, :1, :]
    out, idx, w = hsa.hsa_forward(Q, K, V, L, topk)
    idx = idx.cpu().numpy().reshape(-1, topk)
    w = w.cpu().numpy().reshape(-1, topk)
    for r in range(B * H * T):
        n = min((r % T + 1) // 64, T // 64)
        k = min(n, topk)
        assert idx[r].tolist() == list(range(k)) + [-1] * (topk - k)
        if k:
            assert np.allclose(w[r, :k], 1.0 / k, atol=1e-6)


def test_forward_full_size_32k_sampled_rows(oracle_mod):
    """B2 T32768 H8 D128 topk16 with chunk-mean landmarks, checked on 1024 sampled rows plus edges."""
    w = inputs.WORKLOADS["fwd_t32k_h8_d128_k16"]
    rng = np.random.default_rng(5)
    BH, T = w.B * w.H, w.T
    edges = [bh * T + t for bh in (0, BH - 1) for t in (0, 62, 63, 64, 127, 128, 4095, T - 65, T - 1)]
    rows = np.unique(np.concatenate([rng.integers(0, BH * T, 1024), edges]))
    stats, _ = run_forward_case(oracle_mod, w.B, w.H, w.T, w.D, w.topk, w.seed, w.landmarks, rows=rows)
    assert stats["rows"] == len(rows)


def test_forward_more_chunks_than_the_shared_tables(oracle_mod):
    """131,173 tokens = 2049 complete chunks, past the score kernel's shared-memory pair count (1024
    chunks) and the sorted scatter's tables (2048 chunks): the global-atomic count and the plain scatter
    run. Sampled rows, with the chunk boundaries around both limits."""
    B, H, T, D, topk = 1, 1, 64 * 2049 + 37, 64, 8
    rng = np.random.default_rng(11)
    edges = [0, 63, 64, 64 * 1024 - 1, 64 * 1024, 64 * 1025 - 1, 64 * 2048 - 1, 64 * 2048, 64 * 2049 - 1, T - 1]
    rows = np.unique(np.concatenate([rng.integers(0, T, 384), edges]))
    stats, _ = run_forward_case(oracle_mod, B, H, T, D, topk, seed=77, landmarks="chunk_mean", rows=rows)
    assert stats["rows"] == len(rows)


def test_forward_is_deterministic_in_selection_and_close_in_output():
    Q, K, V, L = inputs.forward_inputs(1, 2, 4096, 128, 3, device=DEV)
    o1, i1, w1 = hsa.hsa_forward(Q, K, V, L, 16)
    o2, i2, w2 = hsa.hsa_forward(Q, K, V, L, 16)
    assert torch.equal(i1, i2) and torch.equal(w1, w2)
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2


# ---------------------------------------------------------------------------------------------
# decode


def oracle_decode(oracle_mod, q, Kc, Vc, Lc, lens, topk, chunk=64, qs=None, qk_norm=False, scale=None):
    """Oracle decode: selection from (q or qs, Lc) on the host, then the selected chunks gathered."""
    B, H, D = q.shape
    scale = scale or 1 / math.sqrt(D)
    sel = oracle_mod.decode_select(host(q if qs is None else qs), host(Lc), lens.cpu().numpy(), chunk=chunk, topk=topk,
                                   scale=scale, all_scores=True)
    if Kc.shape[1] != H:  # grouped key heads: each query head gathers from its key head's cache
        Kc, Vc, Lc = (x.repeat_interleave(H // Kc.shape[1], dim=1) for x in (Kc, Vc, Lc))
    idx = torch.as_tensor(sel["sel_idx"], device=Kc.device, dtype=torch.int64).clamp(min=0)   # [B,H,k]
    tok = (idx[..., None] * chunk + torch.arange(chunk, device=Kc.device)).reshape(B, H, -1)
    Kg = torch.gather(Kc, 2, tok[..., None].expand(-1, -1, -1, D)).reshape(B * H, topk, chunk, D)
    Vg = torch.gather(Vc, 2, tok[..., None].expand(-1, -1, -1, D)).reshape(B * H, topk, chunk, D)
    Lg = torch.gather(Lc, 2, idx[..., None].expand(-1, -1, -1, D)).reshape(B * H, topk, D)
    nsel = (sel["sel_idx"] >= 0).sum(-1).reshape(-1)
    out, w = oracle_mod.attend_gathered(host(q).reshape(B * H, D), host(Lg), host(Kg), host(Vg), nsel,
                                        scale=scale, qk_norm=qk_norm,
                                        qs=None if qs is None else host(qs).reshape(B * H, D))
    return dict(out=out, sel_idx=sel["sel_idx"].reshape(B * H, topk), sel_w=w, sel_s=sel["sel_s"].reshape(B * H, topk),
                next_s=sel["next_s"].reshape(-1), all_s=sel["all_s"].reshape(B * H, -1))


def compare_decode_rows(oracle_mod, orc, g_idx, g_w, g_out, q, Kc, Vc, Lc, qs=None, qk_norm=False, scale=None,
                        chunk=64, label=""):
    """Decode rows (flat (b, h)) against the oracle, by the rule of the forward (tests/parity.py): equal
    selection sets, or a near-tie row (oracle K-th and (K+1)-th scores within 1e-3) whose GPU-kept chunks
    all score within 1e-3 of the oracle's K-th score and whose output matches the oracle evaluated on the
    GPU's set. Returns the number of near-tie rows."""
    BH, D = g_out.shape
    H = q.shape[1]
    G = H // Kc.shape[1]
    scale = scale or 1 / math.sqrt(D)
    topk = g_idx.shape[1]
    tie_rows = []
    for i in range(BH):
        gs, os_ = set(g_idx[i][g_idx[i] >= 0].tolist()), set(orc["sel_idx"][i][orc["sel_idx"][i] >= 0].tolist())
        if gs != os_:
            assert len(gs) == len(os_), f"{label}(b,h)={i}: {len(gs)} chunks kept, oracle keeps {len(os_)}"
            k = len(os_)
            s_k = orc["sel_s"][i, k - 1]
            assert s_k - orc["next_s"][i] < TIE, f"{label}(b,h)={i}: selection differs, gap {s_k - orc['next_s'][i]:.3g}"
            for c in gs:
                assert orc["all_s"][i, c] >= s_k - TIE, f"{label}(b,h)={i}: chunk {c} is not a near-tie choice"
            tie_rows.append(i)
            continue
        d = np.abs(g_out[i] - orc["out"][i])
        assert d.max() <= OUT_MAX_ABS, f"{label}(b,h)={i}: max-abs {d.max():.4g}"
        og = dict(zip(orc["sel_idx"][i].tolist(), orc["sel_w"][i].tolist()))
        for c, ww in zip(g_idx[i].tolist(), g_w[i].tolist()):
            if c >= 0:
                assert abs(ww - og[c]) <= W_MAX_ABS
    if tie_rows:  # the oracle's Steps 3-4 on the GPU's (valid) selection of those rows
        n = len(tie_rows)
        Lg = np.zeros((n, topk, D), np.float32)
        Kg = np.zeros((n, topk, chunk, D), np.float32)
        Vg = np.zeros_like(Kg)
        nsel = np.zeros(n, np.int32)
        for r, i in enumerate(tie_rows):
            b, hk = i // H, (i % H) // G
            kept = [int(c) for c in g_idx[i] if c >= 0]
            for j, c in enumerate(kept):
                Lg[r, j] = host(Lc[b, hk, c])
                Kg[r, j] = host(Kc[b, hk, c * chunk:(c + 1) * chunk])
                Vg[r, j] = host(Vc[b, hk, c * chunk:(c + 1) * chunk])
            nsel[r] = len(kept)
        qr = host(q).reshape(BH, D)[tie_rows]
        qsr = None if qs is None else host(qs).reshape(BH, D)[tie_rows]
        o, _ = oracle_mod.attend_gathered(qr, Lg, Kg, Vg, nsel, scale=scale, qs=qsr, qk_norm=qk_norm)
        dt = np.abs(g_out[tie_rows] - o)
        assert dt.max() <= OUT_MAX_ABS, f"{label}near-tie rows: max-abs {dt.max():.4g}"
    return len(tie_rows)


def check_decode(oracle_mod, q, Kc, Vc, Lc, lens, topk, qs=None, qk_norm=False, scale=None):
    B, H, D = q.shape
    out, idx, w = hsa.hsa_decode(q, Kc, Vc, Lc, lens, topk, qs=qs, qk_norm=qk_norm, scale=scale or 0.0)
    torch.cuda.synchronize()
    orc = oracle_decode(oracle_mod, q, Kc, Vc, Lc, lens, topk, qs=qs, qk_norm=qk_norm, scale=scale)
    g_idx = idx.reshape(B * H, topk).cpu().numpy()
    g_w = w.reshape(B * H, topk).cpu().numpy()
    g_out = host(out).reshape(B * H, D)
    ties = compare_decode_rows(oracle_mod, orc, g_idx, g_w, g_out, q, Kc, Vc, Lc, qs=qs, qk_norm=qk_norm,
                               scale=scale)
    # ordering: by score descending (ties to the lower index) -> sel_w non-increasing
    assert np.all(np.diff(g_w, axis=1) <= 1e-6)
    check_decode.near_tie_rows = ties
    return out, idx, w


@pytest.mark.parametrize("B,H,D,Tmax,lens,topk", [
    (3, 2, 128, 8192, [8192, 5000, 40], 16),
    (2, 2, 64, 64 * 300, [64 * 300, 64 * 300 - 1], 64),
    (1, 4, 128, 64 * 5000 + 17, [64 * 5000 + 17], 32),   # several scan ranges, ragged tail
    (4, 1, 64, 256, [0, 63, 64, 200], 8),
])
def test_decode_matches_oracle(oracle_mod, B, H, D, Tmax, lens, topk):
    q, Kc, Vc, Lc, lens_t, needle = inputs.decode_inputs(B, H, lens, D, seed=300 + Tmax, Tmax=Tmax, device=DEV)
    out, idx, w = check_decode(oracle_mod, q, Kc, Vc, Lc, lens_t, topk)
    for b in range(B):
        n = lens[b] // 64
        if n == 0:
            assert torch.all(out[b] == 0) and torch.all(idx[b] == -1) and torch.all(w[b] == 0)
        elif needle[b] >= 0:
            assert torch.all(idx[b, :, 0] == int(needle[b]))


@pytest.mark.parametrize("T,D,topk", [(4096 + 64, 128, 16), (64 * 150 + 64, 64, 64)])
def test_decode_equals_forward_last_row(T, D, topk):
    B, H = 2, 2
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, 11, device=DEV)
    out, idx, w = hsa.hsa_forward(Q, K, V, L, topk)
    lens = torch.full((B,), T, dtype=torch.int64, device=DEV)
    o2, i2, w2 = hsa.hsa_decode(Q[:, :, T - 1].contiguous(), K, V, L, lens, topk)
    assert torch.equal(i2, idx[:, :, T - 1])
    assert (w2 - w[:, :, T - 1]).abs().max().item() <= 1e-5
    assert (o2.float() - out[:, :, T - 1].float()).abs().max().item() <= 2e-2


@pytest.mark.parametrize("name", ["decode_1m_b16_h8_d128_k16", "decode_16m_b1_h8_d128_k32"])
def test_decode_full_size(oracle_mod, name):
    w = inputs.WORKLOADS[name]
    q, Kc, Vc, Lc, lens, needle = inputs.workload_inputs(w, device=DEV)
    out, idx, ww = check_decode(oracle_mod, q, Kc, Vc, Lc, lens, w.topk)
    print(f"{name}: {check_decode.near_tie_rows} of {w.B * w.H} (b, h) rows took the near-tie branch")
    for b in range(w.B):
        assert torch.all(idx[b, :, 0] == int(needle[b]))
    del q, Kc, Vc, Lc
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------------------------
# backward


@pytest.mark.parametrize("B,H,T,D,topk", [(1, 2, 1100, 64, 8), (1, 1, 2048 + 64, 128, 16), (2, 1, 700, 128, 5),
                                           # chunks with thousands of pairs: several work units each
                                           (1, 2, 8192 + 81, 128, 16),
                                           # 2049 chunks: the dispatch's plain scatter writes the slots
                                           (1, 1, 64 * 2049 + 5, 64, 2),
                                           # topk up to 64
                                           (1, 1, 4096 + 128 + 9, 128, 64), (1, 2, 64 * 60 + 3, 64, 48)])
def test_backward_matches_oracle(oracle_mod, B, H, T, D, topk):
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, 500 + T, device=DEV)
    dO = inputs.upstream_grad(B, H, T, D, 500 + T, device=DEV)
    Qh, Kh, Vh, Lh, dOh = (host(x) for x in (Q, K, V, L, dO))
    scale = 1 / math.sqrt(D)
    orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=scale)
    sel_idx = torch.as_tensor(orc["sel_idx"].reshape(B, H, T, topk), device=DEV)
    sel_w = torch.as_tensor(orc["sel_w"].reshape(B, H, T, topk), dtype=torch.float32, device=DEV)
    out = torch.as_tensor(orc["out"].reshape(B, H, T, D), dtype=torch.float32, device=DEV).to(torch.bfloat16)
    grads = hsa.hsa_backward(Q, K, V, L, out, dO, sel_idx, sel_w)
    ref = oracle_mod.backward(Qh, Kh, Vh, Lh, dOh, orc["sel_idx"].reshape(B, H, T, topk), chunk=64, scale=scale)
    for g, r, n in zip(grads, ref, ("dQ", "dK", "dV", "dL")):
        grad_close(host(g), r, n)


def test_backward_full_size_properties():
    """B1 T65536 H8 D128 topk16, forward then backward on the GPU, checked by properties that hold at
    any size: every gradient is finite; since each row of P sums to one, the sum of dV over a chunk's
    64 keys equals the sum over the chunk's pairs of w * dO; chunks that no token selected get zero
    dK, dV and dL."""
    w = inputs.WORKLOADS["fwdbwd_t64k_h8_d128_k16"]
    Q, K, V, L, dO = inputs.workload_inputs(w, device=DEV)
    out, idx, sw = hsa.hsa_forward(Q, K, V, L, w.topk)
    dQ, dK, dV, dL = hsa.hsa_backward(Q, K, V, L, out, dO, idx, sw)
    torch.cuda.synchronize()
    for g in (dQ, dK, dV, dL):
        assert torch.isfinite(g).all()
    B, H, T, D, N = w.B, w.H, w.T, w.D, w.T // 64
    for b in range(B):
        for h in range(H):
            lhs = dV[b, h].reshape(N, 64, D).sum(1).double()
            valid = idx[b, h] >= 0
            rows = torch.arange(T, device=DEV)[:, None].expand(T, w.topk)[valid]
            chunks = idx[b, h][valid].long()
            contrib = sw[b, h][valid].double()[:, None] * dO[b, h][rows].double()
            rhs = torch.zeros(N, D, dtype=torch.float64, device=DEV).index_add_(0, chunks, contrib)
            err = (lhs - rhs).abs().max().item()
            assert err <= 2e-2 * max(1.0, rhs.abs().max().item()), err
            hit = torch.zeros(N, dtype=torch.bool, device=DEV)
            hit[chunks] = True
            assert torch.all(dL[b, h][~hit] == 0)
            assert torch.all(dK[b, h].reshape(N, 64 * D)[~hit] == 0)
            assert torch.all(dV[b, h].reshape(N, 64 * D)[~hit] == 0)


def test_backward_full_size_two_heads_match_oracle(oracle_mod):
    """B1 T65536 H8 D128 topk16, in the launch configuration the benchmark times: the forward runs on
    the GPU for the whole batch, then heads 0 and 7 (each an independent B1 H1 problem) are given the
    oracle's own forward (selection, weights, bf16 output) and the backward of the whole batch runs on
    the GPU. Their dQ, dK, dV and dL are compared element by element with the oracle's backward; the
    GPU forward of those two heads is compared with the oracle too."""
    w = inputs.WORKLOADS["fwdbwd_t64k_h8_d128_k16"]
    Q, K, V, L, dO = inputs.workload_inputs(w, device=DEV)
    out, idx, sw = hsa.hsa_forward(Q, K, V, L, w.topk)
    torch.cuda.synchronize()
    T, D, topk = w.T, w.D, w.topk
    scale = 1 / math.sqrt(D)
    refs = {}
    for h in (0, w.H - 1):
        Qh, Kh, Vh, Lh, dOh = (host(x[:, h:h + 1]) for x in (Q, K, V, L, dO))
        orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=scale)
        compare_forward_rows(oracle_mod, host(out[:, h]).reshape(-1, D), idx[:, h].reshape(-1, topk).cpu().numpy(),
                             sw[:, h].reshape(-1, topk).cpu().numpy(), orc, Qh, Kh, Vh, Lh, np.arange(T), 64, scale)
        idx[:, h] = torch.as_tensor(orc["sel_idx"].reshape(1, T, topk), device=DEV)
        sw[:, h] = torch.as_tensor(orc["sel_w"].reshape(1, T, topk), dtype=torch.float32, device=DEV)
        out[:, h] = torch.as_tensor(orc["out"].reshape(1, T, D), dtype=torch.float32, device=DEV).to(torch.bfloat16)
        refs[h] = oracle_mod.backward(Qh, Kh, Vh, Lh, dOh, orc["sel_idx"].reshape(1, 1, T, topk), chunk=64,
                                      scale=scale)
    grads = hsa.hsa_backward(Q, K, V, L, out, dO, idx, sw)
    torch.cuda.synchronize()
    for h, ref in refs.items():
        for g, r, n in zip(grads, ref, ("dQ", "dK", "dV", "dL")):
            grad_close(host(g[:, h:h + 1]), r, f"{n} head {h}")


def test_workspace_status_clear_after_calls():
    """A completed forward, backward and decode leave the device status flag of their workspace clear
    (every bounded wait was satisfied)."""
    B, H, T, D, topk = 1, 2, 1100, 128, 8
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, 21, device=DEV)
    ws = torch.empty(hsa.hsa_forward_workspace_size(B, H, T, D, 64, topk), dtype=torch.uint8, device=DEV)
    out, idx, sw = hsa.hsa_forward(Q, K, V, L, topk, workspace=ws)
    hsa.hsa_workspace_status(ws)
    dO = inputs.upstream_grad(B, H, T, D, 21, device=DEV)
    wsb = torch.empty(hsa.hsa_backward_workspace_size(B, H, T, D, 64, topk), dtype=torch.uint8, device=DEV)
    hsa.hsa_backward(Q, K, V, L, out, dO, idx, sw, workspace=wsb)
    hsa.hsa_workspace_status(wsb)
    q, Kc, Vc, Lc, lens_t, _ = inputs.decode_inputs(2, 2, [5000, 777], D, seed=22, Tmax=5056, device=DEV)
    wsd = torch.empty(hsa.hsa_decode_workspace_size(2, 2, 5056, D, 64, topk), dtype=torch.uint8, device=DEV)
    hsa.hsa_decode(q, Kc, Vc, Lc, lens_t, topk, workspace=wsd)
    hsa.hsa_workspace_status(wsd)


def test_bounded_wait_that_runs_out_reports_timeout():
    """A bounded device wait that runs out (the self-test's mbarrier never gets its arrival) is reported
    as HSA_ERR_TIMEOUT by hsa_workspace_status, nothing faults, and the next operator call -- on the same
    workspace, which it clears, and on a fresh one -- runs clean with the same results."""
    B, H, T, D, topk = 1, 2, 1100, 128, 8
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, 23, device=DEV)
    ws = torch.empty(hsa.hsa_forward_workspace_size(B, H, T, D, 64, topk), dtype=torch.uint8, device=DEV)
    stream = torch.cuda.current_stream()
    st = hsa.lib().hsa_selftest_bounded_wait(hsa._ptr(ws), ws.numel(), 2000, ctypes.c_void_p(stream.cuda_stream))
    assert st == 0, hsa.hsa_last_error()
    with pytest.raises(hsa.HSAError, match="HSA_ERR_TIMEOUT"):
        hsa.hsa_workspace_status(ws)
    out, idx, w = hsa.hsa_forward(Q, K, V, L, topk, workspace=ws)
    hsa.hsa_workspace_status(ws)
    ws2 = torch.empty_like(ws)
    out2, idx2, w2 = hsa.hsa_forward(Q, K, V, L, topk, workspace=ws2)
    hsa.hsa_workspace_status(ws2)
    assert torch.equal(idx, idx2) and torch.equal(w, w2)
    assert (out.float() - out2.float()).abs().max().item() <= 2e-2


# ---------------------------------------------------------------------------------------------
# separate retrieval query (q_slc scores the landmarks, q_attn attends)


@pytest.mark.parametrize("B,H,T,D,topk", [(1, 2, 2048 + 37, 128, 16), (1, 2, 1100, 64, 8)])
def test_forward_separate_retrieval_query_matches_oracle(oracle_mod, B, H, T, D, topk):
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, 600 + T, device=DEV)
    Qs = inputs.forward_inputs(B, H, T, D, 700 + T, device=DEV)[0]
    out, idx, w = hsa.hsa_forward(Q, K, V, L, topk, Qs=Qs)
    Qh, Kh, Vh, Lh, Qsh = (host(x) for x in (Q, K, V, L, Qs))
    scale = 1 / math.sqrt(D)
    orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=scale, Qs=Qsh)
    rows = np.arange(B * H * T)
    compare_forward_rows(oracle_mod, host(out).reshape(-1, D), host(idx).reshape(-1, topk),
                         host(w).reshape(-1, topk), orc, Qh, Kh, Vh, Lh, rows, 64, scale, Qs=Qsh)
    # the retrieval query decides: the single-query call selects differently
    _, idx_q, _ = hsa.hsa_forward(Q, K, V, L, topk)
    assert not torch.equal(idx, idx_q)


@pytest.mark.parametrize("D,lens,topk", [(128, [9000, 4100], 8), (64, [64 * 300 - 1, 640], 32)])
def test_decode_separate_retrieval_query_matches_oracle(oracle_mod, D, lens, topk):
    B, H = len(lens), 2
    q, Kc, Vc, Lc, lens_t, _ = inputs.decode_inputs(B, H, lens, D, seed=31 + D, Tmax=max(lens) + 64, device=DEV)
    qs = inputs.decode_inputs(B, H, lens, D, seed=32 + D, Tmax=max(lens) + 64, device=DEV)[0]
    _, idx, _ = check_decode(oracle_mod, q, Kc, Vc, Lc, lens_t, topk, qs=qs)
    _, idx_q, _ = hsa.hsa_decode(q, Kc, Vc, Lc, lens_t, topk)
    assert not torch.equal(idx, idx_q)


@pytest.mark.parametrize("B,H,T,D,topk", [(1, 2, 2048 + 64, 128, 16), (1, 2, 1100, 64, 8),
                                           (1, 1, 4096 + 256, 128, 64)])  # two slot groups per token
def test_backward_separate_retrieval_query_matches_oracle(oracle_mod, B, H, T, D, topk):
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, 800 + T, device=DEV)
    Qs = inputs.forward_inputs(B, H, T, D, 900 + T, device=DEV)[0]
    dO = inputs.upstream_grad(B, H, T, D, 800 + T, device=DEV)
    Qh, Kh, Vh, Lh, Qsh, dOh = (host(x) for x in (Q, K, V, L, Qs, dO))
    scale = 1 / math.sqrt(D)
    orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=scale, Qs=Qsh)
    sel_idx = torch.as_tensor(orc["sel_idx"].reshape(B, H, T, topk), device=DEV)
    sel_w = torch.as_tensor(orc["sel_w"].reshape(B, H, T, topk), dtype=torch.float32, device=DEV)
    out = torch.as_tensor(orc["out"].reshape(B, H, T, D), dtype=torch.float32, device=DEV).to(torch.bfloat16)
    grads = hsa.hsa_backward(Q, K, V, L, out, dO, sel_idx, sel_w, Qs=Qs)
    ref = oracle_mod.backward(Qh, Kh, Vh, Lh, dOh, orc["sel_idx"].reshape(B, H, T, topk), chunk=64, scale=scale,
                              Qs=Qsh)
    for g, r, n in zip(grads, ref, ("dQ", "dK", "dV", "dL", "dQs")):
        grad_close(host(g), r, n)


# ---------------------------------------------------------------------------------------------
# query-key normalisation (Step 3 attends with norm(q) . norm(K_c)); scale 4 as well as 1/sqrt(D), since
# unit vectors at 1/sqrt(D) give nearly uniform in-chunk weights


@pytest.mark.parametrize("B,H,T,D,topk,scale,separate", [
    (1, 2, 2048 + 37, 128, 16, 4.0, False), (1, 2, 2048 + 37, 128, 16, None, True),
    (1, 2, 1100, 64, 8, 4.0, True), (2, 1, 700, 64, 5, None, False),
])
def test_forward_qk_norm_matches_oracle(oracle_mod, B, H, T, D, topk, scale, separate):
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, 1000 + T, device=DEV)
    Qs = inputs.forward_inputs(B, H, T, D, 1100 + T, device=DEV)[0] if separate else None
    sc = scale if scale else 1 / math.sqrt(D)
    out, idx, w = hsa.hsa_forward(Q, K, V, L, topk, scale=sc, Qs=Qs, qk_norm=True)
    Qh, Kh, Vh, Lh = (host(x) for x in (Q, K, V, L))
    Qsh = host(Qs) if separate else None
    orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=sc, Qs=Qsh, qk_norm=True)
    rows = np.arange(B * H * T)
    compare_forward_rows(oracle_mod, host(out).reshape(-1, D), host(idx).reshape(-1, topk),
                         host(w).reshape(-1, topk), orc, Qh, Kh, Vh, Lh, rows, 64, sc, Qs=Qsh, qk_norm=True)
    plain = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=sc, Qs=Qsh)
    if scale:  # the normalisation changes the result well beyond the tolerance
        assert np.abs(plain["out"] - orc["out"]).max() > 0.1


@pytest.mark.parametrize("D,lens,topk,separate", [(128, [9000, 4100], 8, False), (64, [64 * 300 - 1, 640], 32, True)])
def test_decode_qk_norm_matches_oracle(oracle_mod, D, lens, topk, separate):
    B, H = len(lens), 2
    q, Kc, Vc, Lc, lens_t, _ = inputs.decode_inputs(B, H, lens, D, seed=41 + D, Tmax=max(lens) + 64, device=DEV)
    qs = inputs.decode_inputs(B, H, lens, D, seed=42 + D, Tmax=max(lens) + 64, device=DEV)[0] if separate else None
    out, _, _ = check_decode(oracle_mod, q, Kc, Vc, Lc, lens_t, topk, qs=qs, qk_norm=True, scale=4.0)
    plain, _, _ = hsa.hsa_decode(q, Kc, Vc, Lc, lens_t, topk, qs=qs, scale=4.0)
    assert (out.float() - plain.float()).abs().max() > 0.1


@pytest.mark.parametrize("B,H,T,D,topk,separate", [
    (1, 2, 2048 + 64, 128, 16, False), (1, 2, 2048 + 64, 128, 16, True), (1, 2, 1100, 64, 8, False),
    (1, 1, 1100, 64, 8, True),
])
def test_backward_qk_norm_matches_oracle(oracle_mod, B, H, T, D, topk, separate):
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, 1200 + T, device=DEV)
    Qs = inputs.forward_inputs(B, H, T, D, 1300 + T, device=DEV)[0] if separate else None
    dO = inputs.upstream_grad(B, H, T, D, 1200 + T, device=DEV)
    Qh, Kh, Vh, Lh, dOh = (host(x) for x in (Q, K, V, L, dO))
    Qsh = host(Qs) if separate else None
    # the pages' scale: at much larger scales the fusion softmax saturates and ds = w (dO.O_c - dO.out)
    # cancels down to the bf16 rounding of the stored output (the retrieval gradients lose relative
    # accuracy with or without the normalisation)
    sc = 1 / math.sqrt(D)
    orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=sc, Qs=Qsh, qk_norm=True)
    sel_idx = torch.as_tensor(orc["sel_idx"].reshape(B, H, T, topk), device=DEV)
    sel_w = torch.as_tensor(orc["sel_w"].reshape(B, H, T, topk), dtype=torch.float32, device=DEV)
    out = torch.as_tensor(orc["out"].reshape(B, H, T, D), dtype=torch.float32, device=DEV).to(torch.bfloat16)
    grads = hsa.hsa_backward(Q, K, V, L, out, dO, sel_idx, sel_w, scale=sc, Qs=Qs, qk_norm=True)
    ref = oracle_mod.backward(Qh, Kh, Vh, Lh, dOh, orc["sel_idx"].reshape(B, H, T, topk), chunk=64, scale=sc,
                              Qs=Qsh, qk_norm=True)
    for g, r, n in zip(grads, ref, ("dQ", "dK", "dV", "dL", "dQs")):
        grad_close(host(g), r, n)
    plain = oracle_mod.backward(Qh, Kh, Vh, Lh, dOh, orc["sel_idx"].reshape(B, H, T, topk), chunk=64, scale=sc,
                                Qs=Qsh)
    for x, y in zip(ref[:2], plain[:2]):  # dQ and dK: the normalisation's Jacobian matters
        assert np.abs(x - y).sum() > 0.5 * np.abs(x).sum()


# ---------------------------------------------------------------------------------------------
# grouped key/value heads: query head h reads key head h // (H // Hkv); each query head selects its own


def gqa_inputs(B, H, Hkv, T, D, seed):
    Q = inputs.forward_inputs(B, H, T, D, seed, device=DEV)[0]
    _, K, V, L = inputs.forward_inputs(B, Hkv, T, D, seed + 1, device=DEV)
    return Q, K, V, L


@pytest.mark.parametrize("B,H,Hkv,T,D,topk,opts", [
    (1, 4, 2, 2048 + 37, 128, 16, {}), (2, 4, 1, 1100, 64, 8, {}), (1, 8, 2, 1500, 128, 8, {"qk_norm": True}),
    (1, 4, 2, 777, 64, 5, {"separate": True}),
])
def test_forward_grouped_heads_match_oracle(oracle_mod, B, H, Hkv, T, D, topk, opts):
    Q, K, V, L = gqa_inputs(B, H, Hkv, T, D, 1400 + T)
    Qs = inputs.forward_inputs(B, H, T, D, 1500 + T, device=DEV)[0] if opts.get("separate") else None
    qk = opts.get("qk_norm", False)
    sc = 1 / math.sqrt(D)
    out, idx, w = hsa.hsa_forward(Q, K, V, L, topk, Qs=Qs, qk_norm=qk)
    Qh, Kh, Vh, Lh = (host(x) for x in (Q, K, V, L))
    Qsh = None if Qs is None else host(Qs)
    orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=sc, Qs=Qsh, qk_norm=qk)
    compare_forward_rows(oracle_mod, host(out).reshape(-1, D), host(idx).reshape(-1, topk), host(w).reshape(-1, topk),
                         orc, Qh, Kh, Vh, Lh, np.arange(B * H * T), 64, sc, Qs=Qsh, qk_norm=qk)


@pytest.mark.parametrize("B,H,Hkv,D,lens,topk", [
    (2, 4, 2, 128, [9000, 4100], 16), (1, 8, 1, 64, [64 * 700 + 5], 32),
    (1, 16, 1, 128, [64 * 5000 + 17], 32),          # 16 heads per key head, several ranges, ragged tail
    (4, 6, 2, 64, [0, 63, 64 * 20 + 3, 64 * 40], 8),  # empty caches and ranges shorter than 32 landmarks
    (1, 4, 1, 128, [64 * 3000], 40),                # topk above 32: the per-head scan serves it
])
def test_decode_grouped_heads_match_oracle(oracle_mod, B, H, Hkv, D, lens, topk):
    Tmax = max(lens) + 64
    q = inputs.decode_inputs(B, H, lens, D, seed=51 + D, Tmax=Tmax, device=DEV)[0]
    _, Kc, Vc, Lc, lens_t, _ = inputs.decode_inputs(B, Hkv, lens, D, seed=52 + D, Tmax=Tmax, device=DEV)
    out, idx, w = check_decode(oracle_mod, q, Kc, Vc, Lc, lens_t, topk)
    for b in range(B):
        if lens[b] < 64:
            assert torch.all(out[b] == 0) and torch.all(idx[b] == -1) and torch.all(w[b] == 0)


def test_decode_grouped_heads_equal_landmarks_keep_lowest_chunks():
    B, H, Hkv, D, topk = 1, 8, 2, 128, 16
    lens = [64 * 3000]
    q = inputs.decode_inputs(B, H, lens, D, seed=61, device=DEV)[0]
    _, Kc, Vc, Lc, lens_t, _ = inputs.decode_inputs(B, Hkv, lens, D, seed=62, device=DEV)
    Lc[:] = Lc[:, :, :1]
    _, idx, w = hsa.hsa_decode(q, Kc, Vc, Lc, lens_t, topk)
    assert torch.equal(idx.cpu(), torch.arange(topk, dtype=torch.int32).expand(B, H, topk))
    assert torch.allclose(w, torch.full_like(w, 1.0 / topk))


@pytest.mark.parametrize("B,H,Hkv,T,D,topk,opts", [
    (1, 4, 2, 2048 + 64, 128, 16, {}), (1, 4, 1, 1100, 64, 8, {}), (1, 4, 2, 1500, 128, 8, {"qk_norm": True}),
    (1, 4, 2, 1100, 64, 8, {"separate": True, "qk_norm": True}),
])
def test_backward_grouped_heads_match_oracle(oracle_mod, B, H, Hkv, T, D, topk, opts):
    Q, K, V, L = gqa_inputs(B, H, Hkv, T, D, 1600 + T)
    Qs = inputs.forward_inputs(B, H, T, D, 1700 + T, device=DEV)[0] if opts.get("separate") else None
    qk = opts.get("qk_norm", False)
    dO = inputs.upstream_grad(B, H, T, D, 1600 + T, device=DEV)
    Qh, Kh, Vh, Lh, dOh = (host(x) for x in (Q, K, V, L, dO))
    Qsh = None if Qs is None else host(Qs)
    sc = 1 / math.sqrt(D)
    orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=sc, Qs=Qsh, qk_norm=qk)
    sel_idx = torch.as_tensor(orc["sel_idx"].reshape(B, H, T, topk), device=DEV)
    sel_w = torch.as_tensor(orc["sel_w"].reshape(B, H, T, topk), dtype=torch.float32, device=DEV)
    out = torch.as_tensor(orc["out"].reshape(B, H, T, D), dtype=torch.float32, device=DEV).to(torch.bfloat16)
    grads = hsa.hsa_backward(Q, K, V, L, out, dO, sel_idx, sel_w, Qs=Qs, qk_norm=qk)
    ref = oracle_mod.backward(Qh, Kh, Vh, Lh, dOh, orc["sel_idx"].reshape(B, H, T, topk), chunk=64, scale=sc, Qs=Qsh,
                              qk_norm=qk)
    assert grads[1].shape == (B, Hkv, T, D) and grads[3].shape == (B, Hkv, T // 64, D)
    for g, r, n in zip(grads, ref, ("dQ", "dK", "dV", "dL", "dQs")):
        grad_close(host(g), r, n)


# ---------------------------------------------------------------------------------------------
# several query tokens per decode step: token i of Tq sits at cache_len - Tq + i (the prefill's causal
# rule), so each token is a one-token decode against the cache cut at its own position


def check_decode_multi(oracle_mod, q, Kc, Vc, Lc, lens, topk, qs=None, qk_norm=False):
    B, H, Tq, D = q.shape
    out, idx, w = hsa.hsa_decode(q, Kc, Vc, Lc, lens, topk, qs=qs, qk_norm=qk_norm)
    torch.cuda.synchronize()
    assert out.shape == (B, H, Tq, D) and idx.shape == (B, H, Tq, topk)
    for i in range(Tq):
        lens_i = (lens - Tq + i + 1).clamp(min=0)
        orc = oracle_decode(oracle_mod, q[:, :, i].contiguous(), Kc, Vc, Lc, lens_i, topk,
                            qs=None if qs is None else qs[:, :, i].contiguous(), qk_norm=qk_norm)
        g_idx = idx[:, :, i].reshape(B * H, topk).cpu().numpy()
        g_w = w[:, :, i].reshape(B * H, topk).cpu().numpy()
        g_out = host(out[:, :, i]).reshape(B * H, D)
        compare_decode_rows(oracle_mod, orc, g_idx, g_w, g_out, q[:, :, i].contiguous(), Kc, Vc, Lc,
                            qs=None if qs is None else qs[:, :, i].contiguous(), qk_norm=qk_norm,
                            label=f"token {i} ")
    return out, idx, w


@pytest.mark.parametrize("B,H,Hkv,D,lens,Tq,topk", [
    (2, 4, 4, 128, [9000, 4100], 5, 16),           # one query head per key head, 5 tokens: 5 rows per pass
    (1, 8, 2, 64, [64 * 300 + 7], 4, 32),           # 4 heads x 4 tokens = 16 rows per key head
    (2, 2, 1, 128, [64 * 200, 64 * 200 - 3], 16, 8),  # 2 heads x 16 tokens: two row groups of 16
    (3, 2, 2, 64, [130, 64 * 50 + 63, 64], 7, 8),    # tokens with no complete chunk, crossing chunk ends
])
def test_decode_multi_token_matches_oracle(oracle_mod, B, H, Hkv, D, lens, Tq, topk):
    Tmax = max(lens) + 64
    q = inputs.forward_inputs(B, H, Tq, D, 2000 + Tq + D, device=DEV)[0]
    _, Kc, Vc, Lc, lens_t, _ = inputs.decode_inputs(B, Hkv, lens, D, seed=71 + Tq, Tmax=Tmax, device=DEV)
    out, idx, w = check_decode_multi(oracle_mod, q, Kc, Vc, Lc, lens_t, topk)
    for b in range(B):
        for i in range(Tq):
            if (lens[b] - Tq + i + 1) // 64 == 0:
                assert torch.all(out[b, :, i] == 0) and torch.all(idx[b, :, i] == -1)


def test_decode_multi_token_equals_forward_last_rows(oracle_mod):
    """The last Tq rows of a prefill, decoded in one step against the same tensors as the cache."""
    B, H, Hkv, T, D, topk, Tq = 1, 4, 2, 64 * 40 + 9, 128, 16, 12
    Q, K, V, L = gqa_inputs(B, H, Hkv, T, D, 2100)
    q = Q[:, :, T - Tq:].contiguous()
    lens = torch.tensor([T], dtype=torch.int64, device=DEV)
    out_d, idx_d, w_d = hsa.hsa_decode(q, K, V, L, lens, topk)
    Qh, Kh, Vh, Lh = (host(x) for x in (Q, K, V, L))
    rows = np.asarray([(bh * T + t) for bh in range(B * H) for t in range(T - Tq, T)])
    orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=1 / math.sqrt(D), rows=rows)
    compare_forward_rows(oracle_mod, host(out_d).reshape(-1, D), host(idx_d).reshape(-1, topk),
                         host(w_d).reshape(-1, topk), orc, Qh, Kh, Vh, Lh, rows, 64, 1 / math.sqrt(D))


def test_decode_multi_token_with_options(oracle_mod):
    B, H, Hkv, D, lens, Tq, topk = 2, 4, 2, 128, [64 * 90 + 1, 64 * 33], 3, 8
    Tmax = max(lens) + 64
    q = inputs.forward_inputs(B, H, Tq, D, 2200, device=DEV)[0]
    qs = inputs.forward_inputs(B, H, Tq, D, 2201, device=DEV)[0]
    _, Kc, Vc, Lc, lens_t, _ = inputs.decode_inputs(B, Hkv, lens, D, seed=81, Tmax=Tmax, device=DEV)
    check_decode_multi(oracle_mod, q, Kc, Vc, Lc, lens_t, topk, qs=qs, qk_norm=True)


# ---------------------------------------------------------------------------------------------
# variable-length batches, packed token-major: each sequence is its own HSA problem


def varlen_batch(lens, H, Hkv, D, seed, separate=False):
    """Per-sequence [1, H, T, D] inputs and their packed token-major concatenation."""
    seqs = []
    for b, T in enumerate(lens):
        Q = inputs.forward_inputs(1, H, T, D, seed + 2 * b, device=DEV)[0]
        _, K, V, L = inputs.forward_inputs(1, Hkv, T, D, seed + 2 * b + 1, device=DEV)
        Qs = inputs.forward_inputs(1, H, T, D, seed + 100 + b, device=DEV)[0] if separate else None
        seqs.append((Q, K, V, L, Qs))
    pack = lambda xs: torch.cat([x[0].transpose(0, 1) for x in xs]).contiguous()  # [1,h,t,d] -> [t,h,d]
    packed = [pack([s_[i] for s_ in seqs]) for i in range(4)]
    packed.append(pack([s_[4] for s_ in seqs]) if separate else None)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device=DEV)
    return seqs, packed, cu


@pytest.mark.parametrize("lens,H,Hkv,D,topk,opts", [
    ([1000, 64, 30, 2500, 700], 4, 2, 128, 8, {}),
    ([600, 129, 1700], 2, 2, 64, 16, {"qk_norm": True, "separate": True}),
    ([40, 20], 2, 1, 128, 4, {}),                    # no sequence has a complete chunk
    # one long sequence among short ones, padded to its length: most of the scoring kernel's work items
    # (256 rows of one head) lie past their sequence's end, in long runs per CTA
    ([16384] + [100] * 7, 2, 2, 128, 16, {}),
])
def test_forward_varlen_matches_per_sequence_oracle(oracle_mod, lens, H, Hkv, D, topk, opts):
    sep, qk = opts.get("separate", False), opts.get("qk_norm", False)
    seqs, (Q, K, V, L, Qs), cu = varlen_batch(lens, H, Hkv, D, 3000 + D, separate=sep)
    out, idx, w = hsa.hsa_forward_varlen(Q, K, V, L, cu, max(lens), topk, Qs=Qs, qk_norm=qk)
    sc = 1 / math.sqrt(D)
    for b, (Qb, Kb, Vb, Lb, Qsb) in enumerate(seqs):
        T = lens[b]
        rows = slice(int(cu[b]), int(cu[b + 1]))
        g = lambda x, n: host(x[rows].transpose(0, 1)).reshape(-1, n)  # [t,h,n] -> (h, t) rows
        Qh, Kh, Vh, Lh = (host(x) for x in (Qb, Kb, Vb, Lb))
        Qsh = None if Qsb is None else host(Qsb)
        orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=sc, Qs=Qsh, qk_norm=qk)
        compare_forward_rows(oracle_mod, g(out, D), g(idx, topk), g(w, topk), orc, Qh, Kh, Vh, Lh,
                             np.arange(H * T), 64, sc, Qs=Qsh, qk_norm=qk)


def test_forward_varlen_equal_lengths_equals_batched_call():
    """[B, T, H, D] is the equal-length case: the same kernels, so the same selection as the batched call
    and the same output up to the order of the fp32 reductions (which is not fixed between runs)."""
    B, H, T, D, topk = 2, 4, 1100, 128, 16
    Q, K, V, L = inputs.forward_inputs(B, H, T, D, 3100, device=DEV)
    out_b, idx_b, w_b = hsa.hsa_forward(Q, K, V, L, topk)
    tm = lambda x: x.transpose(1, 2).reshape(-1, x.shape[1], x.shape[3]).contiguous()  # [B,H,T,D] -> [B*T,H,D]
    cu = torch.arange(0, (B + 1) * T, T, dtype=torch.int32, device=DEV)
    out_v, idx_v, w_v = hsa.hsa_forward_varlen(tm(Q), tm(K), tm(V), tm(L), cu, T, topk)
    assert torch.equal(idx_v, tm(idx_b))
    assert torch.equal(w_v, tm(w_b))
    assert (out_v.float() - tm(out_b).float()).abs().max() <= 2e-2


@pytest.mark.parametrize("lens,H,Hkv,D,topk,opts", [
    ([700, 1300, 65], 4, 2, 128, 8, {}),
    ([900, 300], 2, 2, 64, 8, {"separate": True, "qk_norm": True}),
])
def test_backward_varlen_matches_per_sequence_oracle(oracle_mod, lens, H, Hkv, D, topk, opts):
    sep, qk = opts.get("separate", False), opts.get("qk_norm", False)
    seqs, (Q, K, V, L, Qs), cu = varlen_batch(lens, H, Hkv, D, 3200 + D, separate=sep)
    dO = torch.cat([inputs.upstream_grad(1, H, T, D, 3300 + T, device=DEV)[0].transpose(0, 1) for T in lens])
    dO = dO.contiguous()
    sc = 1 / math.sqrt(D)
    outs, sels, ws_, refs = [], [], [], []
    for b, (Qb, Kb, Vb, Lb, Qsb) in enumerate(seqs):
        T = lens[b]
        Qh, Kh, Vh, Lh = (host(x) for x in (Qb, Kb, Vb, Lb))
        Qsh = None if Qsb is None else host(Qsb)
        orc = oracle_mod.forward(Qh, Kh, Vh, Lh, chunk=64, topk=topk, scale=sc, Qs=Qsh, qk_norm=qk)
        dOb = host(dO[int(cu[b]):int(cu[b + 1])].transpose(0, 1))[None]
        refs.append(oracle_mod.backward(Qh, Kh, Vh, Lh, dOb, orc["sel_idx"].reshape(1, H, T, topk), chunk=64,
                                        scale=sc, Qs=Qsh, qk_norm=qk))
        outs.append(torch.as_tensor(orc["out"].reshape(H, T, D)).transpose(0, 1))
        sels.append(torch.as_tensor(orc["sel_idx"].reshape(H, T, topk)).transpose(0, 1))
        ws_.append(torch.as_tensor(orc["sel_w"].reshape(H, T, topk)).transpose(0, 1))
    out = torch.cat(outs).to(DEV, torch.float32).to(torch.bfloat16).contiguous()
    sel_idx = torch.cat(sels).to(DEV, torch.int32).contiguous()
    sel_w = torch.cat(ws_).to(DEV, torch.float32).contiguous()
    grads = hsa.hsa_backward_varlen(Q, K, V, L, out, dO, sel_idx, sel_w, cu, max(lens), Qs=Qs, qk_norm=qk)
    cuN = np.concatenate([[0], np.cumsum([T // 64 for T in lens])])
    for b, T in enumerate(lens):
        r, rl = slice(int(cu[b]), int(cu[b + 1])), slice(int(cuN[b]), int(cuN[b + 1]))
        names = ("dQ", "dK", "dV", "dL", "dQs")
        for g, ref, n in zip(grads, refs[b], names):
            gb = g[rl] if n == "dL" else g[r]
            grad_close(host(gb.transpose(0, 1))[None], ref, f"{n} (sequence {b})")
