"""ARKV tri-state KV cache: the method written out plainly in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Page cited throughout:
"ARKV: Adaptive and Resource-Efficient KV Cache Management under Limited Memory
Budget for Long-Context Inference in LLMs" (gist.science/ko/paper/2603.08727),
section 기술요약 §2 (methodology), sub-sections:
  §2.가  per-layer Original:Quantization (OQ) ratio from prefill attention
         entropy, variance and kurtosis;
  §2.나  heavy-hitter score S_k = mu_k + gamma * sigma_k^2 from the cumulative
         attention distribution, updated during decoding;
  §2.다  tri-state assignment (Original bf16 / Quantization FP8 / Eviction) under
         a memory budget, a protected window of the W newest tokens, and
         dequantization of quantized tokens right before attention.

Where the page leaves a step open, the reading taken is named R-<n>:
  R-1  tiers are chosen per row = (layer, sequence, kv-head)
  R-2  prefill statistics come from the last n_obs = W prefill queries (causal)
  R-3  the observation of token k at a step is x_k = sum over the G query heads
       of the group of the attention probability p_hk
  R-4  sigma^2 is the population variance M2/n
  R-5  the Welford count n is the number of observations so far
  R-6  per decode step: append -> attend -> score -> reassign when
       (t + 1) % T_r == 0; one reassignment right after prefill
  R-7  transitions are monotone (Original -> Quantized -> Evicted); ranking by
       (S descending, position ascending); the kept set is the top n_sel; the
       Originals are the first n_o kept tokens that are still bf16
  R-8  the byte budget counts bf16 K+V, FP8 codes and the two fp32 scales,
       window included, relative to the current context length
  R-9  OQ-ratio map: s_l = ((1 - H_l) + v_l/(1+v_l) + k+_l/(1+k+_l)) / 3,
       r_l = clip(r_bar * s_l / mean(s), 0.05, 0.95)          (parity unpinned)
  R-10 slots are kept in position order here
  R-11 r = n_O / (n_O + n_Q) over the non-window kept tokens
The FP8 path (scale and code) is float32, as the format fixes it; the budget
arithmetic is float64 with the operations in the order written, so that any
implementation doing the same operations obtains the same integers.  The
Quantization tier's format is E4M3 unless a caller names E5M2 (the page says
"FP8", which covers both).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import e4m3, e5m2

ORIGINAL, QUANTIZED, EVICTED = 0, 1, 2
E4M3_MAX = np.float32(448.0)
# the Quantization tier's FP8 formats: codec and largest finite value
FORMATS = {"e4m3": (e4m3, E4M3_MAX), "e5m2": (e5m2, np.float32(57344.0))}


# ------------------------------------------------------------------ sizes (R-8)
def bytes_original(D: int) -> int:
    """Bytes one Original token-head occupies: bf16 K and V."""
    return 4 * D


def bytes_quantized(D: int) -> int:
    """Bytes one Quantized token-head occupies: E4M3 K and V codes + two fp32 scales."""
    return 2 * D + 8


# ------------------------------------------------------------------ FP8 (§2.다)
def quantize_token_head(x: np.ndarray, fmt: str = "e4m3"):
    """Quantize the last axis (one token-head vector) to FP8 with an absmax scale.

    s = fl32(amax / FMAX) (s = 1 when amax = 0); code = RNE_FP8(fl32(x / s)), with
    FMAX = 448 for E4M3 and 57344 for E5M2.
    Returns (codes uint8 [..., D], scales float32 [...]).
    """
    codec, fmax = FORMATS[fmt]
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    s = np.where(amax == 0, np.float32(1.0), amax / fmax).astype(np.float32)
    codes = codec.encode((x32 / s[..., None]).astype(np.float32))
    return codes, s


def dequantize(codes: np.ndarray, scales: np.ndarray, fmt: str = "e4m3") -> np.ndarray:
    """The dequantized value, code value times its scale, exact in float64."""
    return FORMATS[fmt][0].decode(codes) * np.asarray(scales, np.float64)[..., None]


# ------------------------------------------------------------------ attention
def softmax(logits: np.ndarray) -> np.ndarray:
    m = np.max(logits, axis=-1, keepdims=True)
    e = np.exp(logits - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention_probs(q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """p[h, k] = softmax_k(q_h . K_k / sqrt(D)) for queries q [G, D] and keys K [n, D]."""
    return softmax((q @ K.T) / math.sqrt(q.shape[-1]))


# ------------------------------------------------------------------ prefill statistics (§2.가)
def attention_row_stats(p: np.ndarray):
    """Entropy, variance and kurtosis of one attention distribution p over n keys.

    H = -sum p ln p / ln n (normalised entropy; 0 when n = 1),
    v = n * sum p^2 - 1 (n^2 times the variance of the probabilities),
    kappa = m4 / m2^2 - 3 with m_j = mean_k (p_k - 1/n)^j (0 when m2 = 0).
    """
    n = p.shape[-1]
    nz = p[p > 0]
    H = float(-np.sum(nz * np.log(nz)) / math.log(n)) if n > 1 else 0.0
    v = float(n * np.sum(p * p) - 1.0)
    d = p - 1.0 / n
    m2 = float(np.mean(d * d))
    m4 = float(np.mean(d ** 4))
    kappa = m4 / (m2 * m2) - 3.0 if m2 > 0 else 0.0
    return H, v, kappa


def welford_update(mu, m2, cnt, x):
    """One Welford step per element (R-4, R-5): n += 1; d = x - mu; mu += d/n; M2 += d (x - mu)."""
    cnt = cnt + 1
    d = x - mu
    mu = mu + d / cnt
    m2 = m2 + d * (x - mu)
    return mu, m2, cnt


def prefill_row(q_obs: np.ndarray, K: np.ndarray):
    """Statistics and initial scores of one row from its prefill (R-2, R-3).

    q_obs [G, n_obs, D]: the group's observation queries at the last n_obs prefill
    positions; K [N, D]: the row's prefill keys.  Query i sits at position
    P_i = N - n_obs + i and sees keys 0..P_i.  Returns per-query (H, v, kappa)
    [G, n_obs, 3] and the Welford state (mu, M2, count) of every key after the
    observations x_k(i) = sum_h p_{h,i,k}, taken in query order.
    """
    G, n_obs, _ = q_obs.shape
    N = K.shape[0]
    stats = np.zeros((G, n_obs, 3))
    mu, m2, cnt = np.zeros(N), np.zeros(N), np.zeros(N, np.int64)
    for i in range(n_obs):
        P = N - n_obs + i
        p = attention_probs(q_obs[:, i, :], K[:P + 1])           # [G, P+1]
        for h in range(G):
            stats[h, i] = attention_row_stats(p[h])
        x = p.sum(axis=0)
        mu[:P + 1], m2[:P + 1], cnt[:P + 1] = welford_update(mu[:P + 1], m2[:P + 1],
                                                             cnt[:P + 1], x)
    return stats, mu, m2, cnt


def oq_ratio(layer_stats: np.ndarray, r_bar: float) -> np.ndarray:
    """Per-layer Original share from (H, v, kappa) layer means [L, 3] (reading R-9).

    More concentrated attention (low entropy, high variance, high kurtosis) marks a
    more sensitive layer, which keeps a larger Original share (§2.가).
    """
    H, v, k = layer_stats[:, 0], layer_stats[:, 1], layer_stats[:, 2]
    kp = np.maximum(k, 0.0)
    s = ((1.0 - H) + v / (1.0 + v) + kp / (1.0 + kp)) / 3.0
    ms = float(np.mean(s))
    if ms <= 0:
        return np.full(len(s), float(r_bar))
    return np.clip(r_bar * s / ms, 0.05, 0.95)


# ------------------------------------------------------------------ budget and tiers (§2.다)
def budget_counts(beta: float, n_t: int, r: float, D: int, W: int, n_cand: int):
    """Kept and Original counts of one row (R-8, R-11).

    beta and r enter as the float32 values the caller holds.  With b_o, b_q the
    bytes of an Original and a Quantized token-head:
      Rb = beta*N_t*b_o - W*b_o            (budget left after the window)
      n_sel = min(floor(Rb / (r*b_o + (1-r)*b_q)), n_cand),  n_o = floor(r*n_sel).
    """
    b_o = float(bytes_original(D))
    b_q = float(bytes_quantized(D))
    beta = float(np.float32(beta))
    r = float(np.float32(r))
    rb = beta * float(n_t) * b_o - float(W) * b_o
    denom = r * b_o + (1.0 - r) * b_q
    n_sel = int(math.floor(rb / denom)) if rb > 0 else 0
    n_sel = max(0, min(n_sel, int(n_cand)))
    n_o = int(math.floor(r * float(n_sel)))
    return n_sel, n_o


def heavy_hitter_score(mu, m2, cnt, gamma: float):
    """S_k = mu_k + gamma * sigma_k^2 with sigma^2 = M2/n (§2.나, R-4)."""
    return mu + float(gamma) * (m2 / cnt)


def assign_tiers(S, pos, is_original, n_sel: int, n_o: int):
    """New tier of each candidate (R-7).

    Candidates are ranked by (S descending, position ascending).  The first n_sel
    are kept; walking the kept ones in rank order, the first n_o that are still
    Original stay Original; every other kept one is Quantized; the rest are
    Evicted.  Returns (tiers, S_cut_keep, S_cut_orig): the scores of the last
    kept and of the last Original candidate (None when there is none).
    """
    order = np.lexsort((pos, -S))
    tiers = np.full(len(S), EVICTED, np.int8)
    count_o, s_cut_o = 0, None
    for idx in order[:n_sel]:
        if is_original[idx] and count_o < n_o:
            tiers[idx] = ORIGINAL
            count_o += 1
            s_cut_o = float(S[idx])
        else:
            tiers[idx] = QUANTIZED
    s_cut_keep = float(S[order[n_sel - 1]]) if n_sel > 0 else None
    return tiers, s_cut_keep, s_cut_o


# ------------------------------------------------------------------ per-row cache state
@dataclass
class Row:
    """Live tokens of one row, in position order (R-10)."""
    D: int
    pos: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))
    orig: np.ndarray = field(default_factory=lambda: np.zeros(0, bool))
    kf: np.ndarray = None        # float64 [n, D]: bf16 values (Original tokens)
    vf: np.ndarray = None
    kc: np.ndarray = None        # uint8 [n, D]: E4M3 codes (Quantized tokens)
    vc: np.ndarray = None
    sk: np.ndarray = None        # float32 [n]: scales (Quantized tokens)
    sv: np.ndarray = None
    cnt: np.ndarray = None       # Welford count
    mu: np.ndarray = None
    m2: np.ndarray = None
    fmt: str = "e4m3"            # FP8 format of the Quantized tokens

    @staticmethod
    def from_prefill(K, V, mu, m2, cnt, fmt: str = "e4m3"):
        n, D = K.shape
        return Row(D=D, pos=np.arange(n, dtype=np.int64), orig=np.ones(n, bool),
                   kf=K.copy(), vf=V.copy(), kc=np.zeros((n, D), np.uint8),
                   vc=np.zeros((n, D), np.uint8), sk=np.ones(n, np.float32),
                   sv=np.ones(n, np.float32), cnt=cnt.astype(np.int64).copy(),
                   mu=mu.copy(), m2=m2.copy(), fmt=fmt)

    def subset(self, keep):
        for name in ("pos", "orig", "kf", "vf", "kc", "vc", "sk", "sv", "cnt", "mu", "m2"):
            setattr(self, name, getattr(self, name)[keep])

    def keys_values(self):
        """K and V as attention sees them: bf16 values, or dequantized codes (§2.다)."""
        Kq = dequantize(self.kc, self.sk, self.fmt)
        Vq = dequantize(self.vc, self.sv, self.fmt)
        o = self.orig[:, None]
        return np.where(o, self.kf, Kq), np.where(o, self.vf, Vq)

    def append(self, pos, k, v):
        D = self.D
        self.pos = np.append(self.pos, np.int64(pos))
        self.orig = np.append(self.orig, True)
        self.kf = np.vstack([self.kf, k[None]])
        self.vf = np.vstack([self.vf, v[None]])
        self.kc = np.vstack([self.kc, np.zeros((1, D), np.uint8)])
        self.vc = np.vstack([self.vc, np.zeros((1, D), np.uint8)])
        self.sk = np.append(self.sk, np.float32(1))
        self.sv = np.append(self.sv, np.float32(1))
        self.cnt = np.append(self.cnt, np.int64(0))
        self.mu = np.append(self.mu, 0.0)
        self.m2 = np.append(self.m2, 0.0)


def decode_row(row: Row, q: np.ndarray):
    """Attention of the group's queries q [G, D] over the row's live tokens (§2.다
    reconstruction), then the score observation and Welford update (§2.나).

    Returns (o [G, D], x [n]) with x_k = sum_h p_hk (R-3)."""
    K, V = row.keys_values()
    p = attention_probs(q, K)
    o = p @ V
    x = p.sum(axis=0)
    row.mu, row.m2, row.cnt = welford_update(row.mu, row.m2, row.cnt, x)
    return o, x


def reassign_row(row: Row, n_t: int, W: int, beta: float, r: float, gamma: float):
    """Tri-state reassignment of one row (§2.다, R-7, R-8).

    The W newest positions stay Original; the other live tokens are ranked by S and
    cut by the budget.  Newly Quantized tokens are quantized from their bf16
    values; already Quantized tokens keep their codes; Evicted tokens are removed.
    Returns a record with the counts, the per-candidate tiers and the cut scores.
    """
    D = row.D
    window = row.pos >= n_t - W
    cand = ~window
    S = heavy_hitter_score(row.mu, row.m2, row.cnt, gamma)
    n_sel, n_o = budget_counts(beta, n_t, r, D, W, int(cand.sum()))
    tiers_c, cut_keep, cut_o = assign_tiers(S[cand], row.pos[cand], row.orig[cand], n_sel, n_o)
    tiers = np.full(len(row.pos), ORIGINAL, np.int8)
    tiers[cand] = tiers_c
    demote = row.orig & (tiers == QUANTIZED)
    if demote.any():
        row.kc[demote], row.sk[demote] = quantize_token_head(row.kf[demote], row.fmt)
        row.vc[demote], row.sv[demote] = quantize_token_head(row.vf[demote], row.fmt)
        row.orig[demote] = False
    rec = {"pos": row.pos.copy(), "tier": tiers, "S": S, "cand": cand, "n_sel": n_sel,
           "n_o": n_o, "cut_keep": cut_keep, "cut_orig": cut_o}
    row.subset(tiers != EVICTED)
    return rec


# ------------------------------------------------------------------ one layer
class OracleLayer:
    """One attention layer's rows, stepped through prefill, decode and reassignment.

    ctx_len [B] holds each sequence's prefill length N0; the context length after the
    append of decode step t is N_t = N0 + t + 1.  `rows` restricts the work to a
    subset of row indices (b * Hkv + g).
    """

    def __init__(self, batch, hq, hkv, D, W, n_obs, beta, gamma, ctx_len, rows=None, fmt="e4m3"):
        self.B, self.Hq, self.Hkv, self.D = batch, hq, hkv, D
        self.fmt = fmt
        self.G = hq // hkv
        self.W, self.n_obs, self.beta, self.gamma = W, n_obs, beta, gamma
        self.ctx_len = np.asarray(ctx_len, np.int64)
        self.row_ids = list(range(batch * hkv)) if rows is None else list(rows)
        self.rows: dict[int, Row] = {}
        self.query_stats: dict[int, np.ndarray] = {}

    def prefill(self, k, v, q_obs):
        """k, v [B, Hkv, Nmax, D] and q_obs [B, Hq, n_obs, D] as float64 values."""
        for rid in self.row_ids:
            b, g = divmod(rid, self.Hkv)
            n = int(self.ctx_len[b])
            qg = q_obs[b, g * self.G:(g + 1) * self.G]
            st, mu, m2, cnt = prefill_row(qg, k[b, g, :n])
            self.query_stats[rid] = st
            self.rows[rid] = Row.from_prefill(k[b, g, :n], v[b, g, :n], mu, m2, cnt, self.fmt)

    def layer_stats(self) -> np.ndarray:
        """Mean (H, v, kappa) over every (sequence, query head, observation query)."""
        allst = np.concatenate([s.reshape(-1, 3) for s in self.query_stats.values()])
        return allst.mean(axis=0)

    def initial_reassign(self, r):
        """The reassignment right after prefill, at N_t = N0 (R-6)."""
        return {rid: reassign_row(row, int(self.ctx_len[rid // self.Hkv]), self.W, self.beta,
                                  r, self.gamma)
                for rid, row in self.rows.items()}

    def decode_step(self, t, q, k_new, v_new):
        """q [B, Hq, D], k_new / v_new [B, Hkv, D] float64.  Returns o [B, Hq, D] (only
        the rows held are filled) and the observations x per row."""
        o = np.zeros((self.B, self.Hq, self.D))
        xs = {}
        for rid, row in self.rows.items():
            b, g = divmod(rid, self.Hkv)
            row.append(int(self.ctx_len[b]) + t, k_new[b, g], v_new[b, g])
            o[b, g * self.G:(g + 1) * self.G], xs[rid] = decode_row(
                row, q[b, g * self.G:(g + 1) * self.G])
        return o, xs

    def reassign(self, t, r):
        return {rid: reassign_row(row, int(self.ctx_len[rid // self.Hkv]) + t + 1, self.W,
                                  self.beta, r, self.gamma)
                for rid, row in self.rows.items()}
