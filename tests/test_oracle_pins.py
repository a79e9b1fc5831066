"""Pins of the oracle's method arithmetic against closed forms, exact rationals,
library routines (torch SDPA, numpy/scipy statistics) and brute force."""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.stats
import torch

from oracle import arkv as A
from oracle import e4m3

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ quantization
def test_quantize_hand_cases():
    codes, s = A.quantize_token_head(np.array([448.0, -224.0, 0.5, 0.0]))
    assert s == np.float32(1.0)
    assert list(codes) == [0x7E, 0xF6, 0x30, 0x00]
    codes, s = A.quantize_token_head(np.array([0.0, -0.0, 0.0]))
    assert s == np.float32(1.0) and list(codes) == [0x00, 0x80, 0x00]
    # amax = 3: s = fl32(3/448); 1/s = 149.33 -> 144 (0x71); 2/s = 298.67 -> 288 (0x79); 3/s -> 448
    codes, s = A.quantize_token_head(np.array([1.0, 2.0, 3.0]))
    assert s == np.float32(3.0) / np.float32(448.0)
    assert list(codes) == [0x71, 0x79, 0x7E]


def test_quantize_e5m2_hand_cases():
    """The second FP8 format: s = fl32(amax / 57344)."""
    codes, s = A.quantize_token_head(np.array([57344.0, -28672.0, 0.5, 0.0]), "e5m2")
    assert s == np.float32(1.0)
    assert list(codes) == [0x7B, 0xF7, 0x38, 0x00]
    # amax = 3: 1/s = 19114.7 -> 20480 (0x75); 2/s = 38229.3 -> 40960 (0x79); 3/s -> 57344
    codes, s = A.quantize_token_head(np.array([1.0, 2.0, 3.0]), "e5m2")
    assert s == np.float32(3.0) / np.float32(57344.0)
    assert list(codes) == [0x75, 0x79, 0x7B]


def test_quantize_error_bound():
    """|x - deq(q(x))| <= half an E4M3 spacing at the scaled magnitude (plus fp32 rounding)."""
    rng = np.random.default_rng(1)
    x = A.np.asarray(rng.standard_normal((64, 128)), np.float32).astype(np.float64)
    codes, s = A.quantize_token_head(x)
    xr = A.dequantize(codes, s)
    y = np.abs(x) / s[:, None]
    spacing = np.exp2(np.maximum(np.floor(np.log2(np.maximum(y, 2.0 ** -9))), -6) - 3)
    assert (np.abs(x - xr) <= (0.5 * spacing * (1 + 2e-6) + 1e-7 * y) * s[:, None]).all()
    assert (np.abs(codes & 0x7F) <= 0x7E).all()
    assert (np.max(codes & 0x7F, axis=1) == 0x7E).all()   # the absmax element maps to 448


# ------------------------------------------------------------------ attention
def _sdpa(q, K, V):
    qt = torch.from_numpy(q)[None, :, None, :]            # [1, G, 1, D]
    kt = torch.from_numpy(K)[None, None].expand(1, q.shape[0], *K.shape)
    vt = torch.from_numpy(V)[None, None].expand(1, q.shape[0], *V.shape)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, :, 0].numpy()


def test_full_budget_attention_equals_exact_softmax_attention():
    """beta=1, r=1: nothing is evicted or quantized, and the decode attention is plain
    softmax attention (torch SDPA in float64)."""
    rng = np.random.default_rng(2)
    D, G, N, W = 32, 4, 300, 16
    K = rng.standard_normal((N, D)); V = rng.standard_normal((N, D))
    row = A.Row.from_prefill(K, V, rng.random(N), rng.random(N), np.full(N, 3))
    rec = A.reassign_row(row, N, W, beta=1.0, r=1.0, gamma=1.0)
    assert rec["n_sel"] == N - W and rec["n_o"] == N - W and row.orig.all()
    q = rng.standard_normal((G, D))
    o, x = A.decode_row(row, q)
    np.testing.assert_allclose(o, _sdpa(q, K, V), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(x.sum(), G, rtol=1e-12)


@pytest.mark.parametrize("fmt,tdtype", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_mixed_cache_attention_equals_attention_over_dequantized_tensors(fmt, tdtype):
    """Brute force from the cache tensors: dequantize with torch's float8 decoder and
    run SDPA; must equal the oracle's attention over the tri-state row."""
    rng = np.random.default_rng(3)
    D, G, N = 16, 2, 50
    K = rng.standard_normal((N, D)); V = rng.standard_normal((N, D))
    row = A.Row.from_prefill(K, V, np.zeros(N), np.zeros(N), np.ones(N), fmt)
    qmask = rng.random(N) < 0.5
    row.kc[qmask], row.sk[qmask] = A.quantize_token_head(K[qmask], fmt)
    row.vc[qmask], row.sv[qmask] = A.quantize_token_head(V[qmask], fmt)
    row.orig[qmask] = False
    f8 = lambda c: torch.from_numpy(c.copy()).view(tdtype).double().numpy()
    Kd = np.where(qmask[:, None], f8(row.kc) * row.sk[:, None].astype(np.float64), K)
    Vd = np.where(qmask[:, None], f8(row.vc) * row.sv[:, None].astype(np.float64), V)
    q = rng.standard_normal((G, D))
    o, _ = A.decode_row(row, q)
    np.testing.assert_allclose(o, _sdpa(q, Kd, Vd), rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------ scores
def test_score_hand_fixture():
    g = json.load(open(os.path.join(GOLD, "score_hand.json")))
    obs = np.array(g["observations"])
    mu, m2, cnt = np.zeros(3), np.zeros(3), np.zeros(3, np.int64)
    for x in obs:
        mu, m2, cnt = A.welford_update(mu, m2, cnt, x)
    fr = lambda pairs: np.array([a / b for a, b in pairs])
    np.testing.assert_allclose(mu, fr(g["mu"]), rtol=1e-15)
    np.testing.assert_allclose(m2 / cnt, fr(g["sigma2"]), rtol=1e-14)
    np.testing.assert_allclose(A.heavy_hitter_score(mu, m2, cnt, 1.0), fr(g["S_gamma1"]), rtol=1e-15)
    np.testing.assert_allclose(A.heavy_hitter_score(mu, m2, cnt, 0.5), fr(g["S_gamma_half"]),
                               rtol=1e-15)


def test_welford_equals_exact_rational_mean_and_variance():
    rng = np.random.default_rng(4)
    xs = rng.random((40, 7))
    mu, m2, cnt = np.zeros(7), np.zeros(7), np.zeros(7, np.int64)
    for x in xs:
        mu, m2, cnt = A.welford_update(mu, m2, cnt, x)
    for j in range(7):
        fx = [Fraction(float(v)) for v in xs[:, j]]
        m = sum(fx) / len(fx)
        var = sum((v - m) ** 2 for v in fx) / len(fx)
        assert abs(mu[j] - float(m)) <= 1e-15 * float(m)
        assert abs(m2[j] / cnt[j] - float(var)) <= 1e-12 * float(var)
    np.testing.assert_allclose(m2 / cnt, np.var(xs, axis=0), rtol=1e-12)
    np.testing.assert_array_equal(A.heavy_hitter_score(mu, m2, cnt, 0.0), mu)


# ------------------------------------------------------------------ prefill statistics
def test_row_stats_closed_forms():
    n = 37
    H, v, k = A.attention_row_stats(np.full(n, 1.0 / n))
    assert abs(H - 1.0) < 1e-14 and abs(v) < 1e-13 and k == 0.0
    p = np.zeros(n); p[5] = 1.0
    H, v, k = A.attention_row_stats(p)
    assert H == 0.0 and abs(v - (n - 1)) < 1e-12
    assert abs(k - (((n - 1) ** 3 + 1) / (n * (n - 1)) - 3)) < 1e-12


def test_row_stats_match_scipy():
    rng = np.random.default_rng(5)
    for n in (2, 10, 1000):
        p = rng.random(n) ** 3; p /= p.sum()
        H, v, k = A.attention_row_stats(p)
        assert abs(H - scipy.stats.entropy(p) / math.log(n)) < 1e-12
        assert abs(v - n * n * np.var(p)) < 1e-9 * max(1, v)
        assert abs(k - scipy.stats.kurtosis(p, fisher=True, bias=True)) < 1e-9 * max(1, abs(k))


def test_prefill_row_uniform_and_welford_init():
    """q = 0 gives uniform causal attention: H = 1, v = 0, kappa = 0; the initial
    observations of key k are G/(P_i+1) for every query i with P_i >= k."""
    rng = np.random.default_rng(6)
    G, n_obs, N, D = 2, 5, 12, 8
    K = rng.standard_normal((N, D))
    st, mu, m2, cnt = A.prefill_row(np.zeros((G, n_obs, D)), K)
    np.testing.assert_allclose(st[..., 0], 1.0, atol=1e-14)
    np.testing.assert_allclose(st[..., 1], 0.0, atol=1e-13)
    assert (st[..., 2] == 0.0).all()
    for k in range(N):
        xs = [G / (P + 1) for P in range(N - n_obs, N) if P >= k]
        assert cnt[k] == min(n_obs, N - k) == len(xs)
        assert abs(mu[k] - np.mean(xs)) < 1e-15
        assert abs(m2[k] / cnt[k] - np.var(xs)) < 1e-15


def test_prefill_row_welford_matches_library_moments():
    rng = np.random.default_rng(7)
    G, n_obs, N, D = 3, 6, 40, 16
    K = rng.standard_normal((N, D)); q = rng.standard_normal((G, n_obs, D))
    st, mu, m2, cnt = A.prefill_row(q, K)
    xs = [[] for _ in range(N)]
    for i in range(n_obs):
        P = N - n_obs + i
        lg = torch.from_numpy(q[:, i]) @ torch.from_numpy(K[:P + 1]).T / math.sqrt(D)
        p = torch.softmax(lg, dim=-1).numpy()
        for j, x in enumerate(p.sum(0)):
            xs[j].append(x)
        for h in range(G):
            assert abs(st[h, i, 0] - scipy.stats.entropy(p[h]) / math.log(P + 1)) < 1e-12
    for j in range(N):
        assert abs(mu[j] - np.mean(xs[j])) < 1e-14
        assert abs(m2[j] / cnt[j] - np.var(xs[j])) < 1e-14


def test_oq_ratio_closed_forms():
    same = np.tile([[0.4, 3.0, 5.0]], (6, 1))
    np.testing.assert_allclose(A.oq_ratio(same, 0.55), 0.55, rtol=1e-15)
    st = np.array([[1.0, 0.0, 0.0], [0.0, 1.0, 1.0]])      # s = 0 and s = (1 + .5 + .5)/3 = 2/3
    r = A.oq_ratio(st, 0.5)
    assert r[0] == 0.05 and r[1] == 0.95                   # 0 -> clipped up, 1.0 -> clipped down
    st = np.array([[0.5, 1.0, 1.0], [0.5, 1.0, -2.0]])      # s = (.5+.5+.5)/3 = .5, (.5+.5+0)/3 = 1/3
    r = A.oq_ratio(st, 0.3)
    np.testing.assert_allclose(r, [0.3 * 0.5 / (5 / 12), 0.3 * (1 / 3) / (5 / 12)], rtol=1e-14)


# ------------------------------------------------------------------ budget and tiers
def test_budget_tiny_fixture():
    g = json.load(open(os.path.join(GOLD, "budget_tiny.json")))
    n_sel, n_o = A.budget_counts(g["beta"], g["n_t"], g["r"], g["D"], g["W"], 10 ** 9)
    assert (n_sel, n_o, n_sel - n_o) == (g["n_sel"], g["n_o"], g["n_q"])
    D, W = g["D"], g["W"]
    used = (n_o + W) * A.bytes_original(D) + (n_sel - n_o) * A.bytes_quantized(D)
    assert used == g["bytes"] <= g["budget_bytes"]


def test_budget_special_cases_and_bound():
    D, W = 128, 128
    # r = 1: eviction only (the page's "Base Origin"): n_sel = floor(Rb / b_o), all Original
    n_sel, n_o = A.budget_counts(0.25, 32768, 1.0, D, W, 10 ** 9)
    assert n_sel == n_o == (32768 // 4 - W)
    # r = 0: Quantized only: n_sel = floor(Rb / b_q)
    n_sel, n_o = A.budget_counts(0.25, 32768, 0.0, D, W, 10 ** 9)
    assert n_o == 0 and n_sel == (8192 - 128) * 512 // 264
    # budget at or below the window: nothing kept
    assert A.budget_counts(0.25, 512, 0.5, D, W, 10 ** 9) == (0, 0)
    rng = np.random.default_rng(8)
    for _ in range(2000):
        beta = float(np.float32(rng.uniform(0.05, 1.0)))
        r = float(np.float32(rng.uniform(0, 1)))
        n_t, Dd, Ww = int(rng.integers(300, 200000)), int(rng.choice([64, 128])), int(rng.integers(1, 300))
        n_sel, n_o = A.budget_counts(beta, n_t, r, Dd, Ww, 10 ** 9)
        used = (n_o + Ww) * A.bytes_original(Dd) + (n_sel - n_o) * A.bytes_quantized(Dd)
        if n_sel > 0:
            assert used <= beta * n_t * A.bytes_original(Dd) * (1 + 1e-12)
        assert 0 <= n_o <= n_sel


def _check_tiers_by_pairwise_rule(S, pos, orig, n_sel, n_o, tiers):
    """Independent characterisation of R-7: every kept candidate outranks every
    evicted one; every Original outranks every kept-but-Quantized token that is still
    bf16; counts as the budget says; Quantized tokens never become Original."""
    better = lambda i, j: (S[i] > S[j]) or (S[i] == S[j] and pos[i] < pos[j])
    kept = np.flatnonzero(tiers != A.EVICTED)
    ev = np.flatnonzero(tiers == A.EVICTED)
    assert len(kept) == min(n_sel, len(S))
    assert all(better(i, j) for i in kept for j in ev)
    og = np.flatnonzero(tiers == A.ORIGINAL)
    qo = np.flatnonzero((tiers == A.QUANTIZED) & orig)
    assert len(og) == min(n_o, int(orig[kept].sum()))
    assert all(better(i, j) for i in og for j in qo)
    assert not (tiers[~orig] == A.ORIGINAL).any()


def test_assign_tiers_brute_force_with_ties():
    rng = np.random.default_rng(9)
    for _ in range(300):
        n = int(rng.integers(1, 14))
        S = rng.integers(0, 4, n).astype(np.float64) / 4     # many ties
        pos = rng.permutation(100)[:n]
        orig = rng.random(n) < 0.6
        n_sel = int(rng.integers(0, n + 1)); n_o = int(rng.integers(0, n_sel + 1))
        tiers, _, _ = A.assign_tiers(S, pos, orig, n_sel, n_o)
        _check_tiers_by_pairwise_rule(S, pos, orig, n_sel, n_o, tiers)


def test_equal_scores_keep_lower_positions():
    S = np.full(6, 0.5); pos = np.array([9, 3, 7, 1, 5, 2])
    tiers, _, _ = A.assign_tiers(S, pos, np.ones(6, bool), 3, 1)
    assert set(pos[tiers != A.EVICTED]) == {1, 2, 3}
    assert pos[tiers == A.ORIGINAL].tolist() == [1]


def test_base_quant_and_base_origin_special_cases():
    rng = np.random.default_rng(10)
    N, D, W = 400, 16, 8
    K = rng.standard_normal((N, D)); V = rng.standard_normal((N, D))
    mk = lambda: A.Row.from_prefill(K, V, rng.random(N), rng.random(N), np.full(N, 2))
    row = mk()   # r = 0 with a budget above the all-quantized size: uniform FP8, nothing evicted
    rec = A.reassign_row(row, N, W, beta=1.0, r=0.0, gamma=1.0)
    assert len(row.pos) == N and (~row.orig).sum() == N - W and row.orig[-W:].all()
    row = mk()   # r = 1: eviction only, no FP8 at all
    rec = A.reassign_row(row, N, W, beta=0.25, r=1.0, gamma=1.0)
    assert row.orig.all() and len(row.pos) == W + (N // 4 - W) == W + rec["n_sel"]


# ------------------------------------------------------------------ whole-layer invariants
def test_tiny_oracle_run_invariants():
    from mixed_precision_kv_arkv_b200 import inputs, workloads
    wl = workloads.TINY
    pre = inputs.layer_prefill(wl, 0)
    f = inputs.bf16_to_f64
    lay = A.OracleLayer(wl.batch, wl.hq, wl.hkv, wl.head_dim, wl.window, wl.n_obs,
                        wl.budget_frac, wl.gamma, pre["ctx_len"])
    lay.prefill(f(pre["k"]), f(pre["v"]), f(pre["q_obs"]))
    recs = lay.initial_reassign(wl.oq_ratio)
    N0, D, W = wl.n_ctx, wl.head_dim, wl.window
    for rid, rec in recs.items():
        assert (rec["n_sel"], rec["n_o"]) == (585, 292)
    was_q = {rid: set(row.pos[~row.orig]) for rid, row in lay.rows.items()}
    alive = {rid: set(row.pos) for rid, row in lay.rows.items()}
    for t in range(wl.steps):
        d = inputs.decode_inputs(wl, 0, t)
        o, xs = lay.decode_step(t, f(d["q"]), f(d["k_new"]), f(d["v_new"]))
        for rid, x in xs.items():
            assert abs(x.sum() - wl.group) < 1e-12                      # P6
        recs = lay.reassign(t, wl.oq_ratio)
        n_t = N0 + t + 1
        for rid, row in lay.rows.items():
            win = np.arange(n_t - W, n_t)
            assert set(win) <= set(row.pos) and row.orig[np.isin(row.pos, win)].all()   # P4
            used = row.orig.sum() * A.bytes_original(D) + (~row.orig).sum() * A.bytes_quantized(D)
            assert used <= wl.budget_frac * n_t * A.bytes_original(D)                   # P7
            now = set(row.pos)
            assert now <= alive[rid] | {n_t - 1}                     # no resurrection
            assert was_q[rid] & set(row.pos[row.orig]) == set()     # no Q -> O
            alive[rid], was_q[rid] = now, set(row.pos[~row.orig])
            assert (np.diff(row.pos) > 0).all()
