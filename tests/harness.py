"""Test harness: moves state between the oracle's per-row token lists and the CUDA
library's packed device layout, and compares the two.  Layout conversion only;
it holds none of the method's arithmetic."""
from __future__ import annotations

import numpy as np
import torch

from mixed_precision_kv_arkv_b200 import abi, inputs
from mixed_precision_kv_arkv_b200.cache import LayerCache, Workspace, make_cfg, stream_ptr
from oracle import arkv as A

F = inputs.bf16_to_f64


def bits_to_bf16_tensor(bits: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def capacities(wl, r: float, n_max: int):
    c = make_cfg(wl.batch, wl.hq, wl.hkv, wl.head_dim, wl.window, wl.n_obs, wl.gamma, wl.budget_frac, 1, 1,
                 wl.quant_format)
    return abi.arkv_row_capacity(c, n_max, r, wl.reassign_interval)


def layer_cfg(wl, cap_o: int, cap_q: int):
    return make_cfg(wl.batch, wl.hq, wl.hkv, wl.head_dim, wl.window, wl.n_obs, wl.gamma,
                    wl.budget_frac, cap_o, cap_q, wl.quant_format)


def new_oracle_layer(wl, ctx_len, rows=None) -> A.OracleLayer:
    return A.OracleLayer(wl.batch, wl.hq, wl.hkv, wl.head_dim, wl.window, wl.n_obs, wl.budget_frac,
                         wl.gamma, ctx_len, rows, wl.quant_format)


# ------------------------------------------------------------------ oracle -> device
def upload_rows(lay: A.OracleLayer, cache: LayerCache, rows=None):
    """Write the oracle's rows into the packed device cache (bf16 segment = Original
    tokens, fp8 segment = Quantized tokens, both in position order)."""
    rows = lay.rows.keys() if rows is None else rows
    dev = cache.k16.device
    for rid in rows:
        row = lay.rows[rid]
        o, q = row.orig, ~row.orig
        no, nq = int(o.sum()), int(q.sum())
        assert no <= cache.cfg.cap_bf16 and nq <= cache.cfg.cap_fp8
        cache.k16[rid, :no] = bits_to_bf16_tensor(inputs.round_bf16(row.kf[o]), dev)
        cache.v16[rid, :no] = bits_to_bf16_tensor(inputs.round_bf16(row.vf[o]), dev)
        cache.pos16[rid, :no] = torch.from_numpy(row.pos[o].astype(np.int32)).to(dev)
        cache.mu16[rid, :no] = torch.from_numpy(row.mu[o].astype(np.float64)).to(dev)
        cache.m2_16[rid, :no] = torch.from_numpy(row.m2[o].astype(np.float64)).to(dev)
        cache.k8[rid, :nq] = torch.from_numpy(row.kc[q]).to(dev)
        cache.v8[rid, :nq] = torch.from_numpy(row.vc[q]).to(dev)
        cache.sk[rid, :nq] = torch.from_numpy(row.sk[q]).to(dev)
        cache.sv[rid, :nq] = torch.from_numpy(row.sv[q]).to(dev)
        cache.pos8[rid, :nq] = torch.from_numpy(row.pos[q].astype(np.int32)).to(dev)
        cache.mu8[rid, :nq] = torch.from_numpy(row.mu[q].astype(np.float64)).to(dev)
        cache.m2_8[rid, :nq] = torch.from_numpy(row.m2[q].astype(np.float64)).to(dev)
        cache.n_bf16[rid] = no
        cache.n_fp8[rid] = nq


# ------------------------------------------------------------------ device -> host
def download_row(cache: LayerCache, rid: int) -> dict:
    """One row of the device cache, tokens sorted by position."""
    n16, n8 = int(cache.n_bf16[rid]), int(cache.n_fp8[rid])
    g = lambda t, n: t[rid, :n].cpu().numpy()
    pos = np.concatenate([g(cache.pos16, n16), g(cache.pos8, n8)]).astype(np.int64)
    order = np.argsort(pos, kind="stable")
    D = cache.cfg.head_dim
    k16 = cache.k16[rid, :n16].view(torch.int16).cpu().numpy().view(np.uint16)
    v16 = cache.v16[rid, :n16].view(torch.int16).cpu().numpy().view(np.uint16)
    kb = np.concatenate([k16, np.zeros((n8, D), np.uint16)])[order]
    vb = np.concatenate([v16, np.zeros((n8, D), np.uint16)])[order]
    kc = np.concatenate([np.zeros((n16, D), np.uint8), g(cache.k8, n8)])[order]
    vc = np.concatenate([np.zeros((n16, D), np.uint8), g(cache.v8, n8)])[order]
    return {
        "pos": pos[order],
        "orig": np.concatenate([np.ones(n16, bool), np.zeros(n8, bool)])[order],
        "k16": kb, "v16": vb, "kc": kc, "vc": vc,
        "sk": np.concatenate([np.ones(n16, np.float32), g(cache.sk, n8)])[order],
        "sv": np.concatenate([np.ones(n16, np.float32), g(cache.sv, n8)])[order],
        "mu": np.concatenate([g(cache.mu16, n16), g(cache.mu8, n8)])[order],
        "m2": np.concatenate([g(cache.m2_16, n16), g(cache.m2_8, n8)])[order],
        "slots": np.concatenate([np.arange(n16), cache.cfg.cap_bf16 + np.arange(n8)])[order],
    }


# ------------------------------------------------------------------ comparisons
def max_rel_per_row(o_gpu: np.ndarray, o_ref: np.ndarray) -> float:
    """max over output rows of max_i |o_i - o*_i| / max_i |o*_i| (reading R-15)."""
    err = np.abs(o_gpu - o_ref).max(axis=-1)
    den = np.abs(o_ref).max(axis=-1)
    return float((err / den).max())


def score_rel_err(gpu: dict, row: A.Row, gamma: float) -> float:
    """Largest |S - S*| / |S*| over tokens matched by position (R-16 floor)."""
    assert np.array_equal(gpu["pos"], row.pos)
    S_ref = A.heavy_hitter_score(row.mu, row.m2, row.cnt, gamma)
    S_gpu = gpu["mu"] + gamma * (gpu["m2"] / row.cnt)
    return float(np.max(np.abs(S_gpu - S_ref) / (np.abs(S_ref) + 1e-300)))


def tier_mismatches(rec: dict, tier_by_pos: dict, rel: float = 1e-6):
    """Positions whose tier differs between the oracle record and the device, split
    into (non-exempt, exempt): a token is exempt when its oracle score lies within
    `rel` of either cut (reading R-17)."""
    bad, exempt = [], []
    cuts = [c for c in (rec["cut_keep"], rec["cut_orig"]) if c is not None]
    for p, t, s in zip(rec["pos"], rec["tier"], rec["S"]):
        tg = tier_by_pos.get(int(p), A.EVICTED)
        if tg == t:
            continue
        if any(abs(s - c) <= rel * abs(c) for c in cuts):
            exempt.append(int(p))
        else:
            bad.append((int(p), int(t), int(tg), float(s)))
    return bad, exempt


def device_tiers(pre: dict, tier_dbg_row: np.ndarray) -> dict:
    """Position -> tier, from the pre-call row state and the per-slot tier output."""
    return {int(p): int(tier_dbg_row[s]) for p, s in zip(pre["pos"], pre["slots"])}


def assert_same_fp8(gpu: dict, row: A.Row):
    """Codes and scales of tokens Quantized on both sides are bit-exact."""
    q = (~gpu["orig"]) & (~row.orig)
    assert np.array_equal(gpu["kc"][q], row.kc[q])
    assert np.array_equal(gpu["vc"][q], row.vc[q])
    assert np.array_equal(gpu["sk"][q].view(np.uint32), row.sk[q].view(np.uint32))
    assert np.array_equal(gpu["sv"][q].view(np.uint32), row.sv[q].view(np.uint32))


def assert_same_bf16(gpu: dict, row: A.Row):
    o = gpu["orig"] & row.orig
    assert np.array_equal(gpu["k16"][o], inputs.round_bf16(row.kf[o]))
    assert np.array_equal(gpu["v16"][o], inputs.round_bf16(row.vf[o]))


class DeviceLayer:
    """Device buffers and workspaces of one layer for the tests."""

    def __init__(self, wl, cap_o, cap_q, device, n_ctx_max=None):
        self.wl = wl
        self.cfg = layer_cfg(wl, cap_o, cap_q)
        self.cache = LayerCache(self.cfg, device)
        self.ws_dec = Workspace(abi.arkv_workspace_bytes(self.cfg, abi.ARKV_WS_DECODE), device)
        self.ws_re = Workspace(abi.arkv_workspace_bytes(self.cfg, abi.ARKV_WS_REASSIGN), device)
        n_ctx_max = n_ctx_max or wl.n_ctx
        self.n_stride = n_ctx_max
        self.ws_pre = Workspace(abi.arkv_workspace_bytes(self.cfg, abi.ARKV_WS_PREFILL, n_ctx_max), device)
        self.tier_dbg = torch.zeros((wl.rows, cap_o + cap_q), dtype=torch.uint8, device=device)
        self.device = device

    def s(self):
        return stream_ptr()

    def prefill(self, k, v, q_obs, ctx_len, r, with_tiers=True):
        """arkv_prefill_stats + arkv_quantize_pack on torch device tensors."""
        wl, dev = self.wl, self.device
        R, N = wl.rows, self.n_stride
        self.mu0 = torch.zeros((R, N), dtype=torch.float64, device=dev)
        self.m2_0 = torch.zeros((R, N), dtype=torch.float64, device=dev)
        self.stats = torch.zeros(3, dtype=torch.float64, device=dev)
        self.qstats = torch.zeros((wl.batch, wl.hq, wl.n_obs, 3), dtype=torch.float64, device=dev)
        abi.arkv_prefill_stats(self.cfg, q_obs.data_ptr(), k.data_ptr(), N, ctx_len.data_ptr(),
                               self.stats.data_ptr(), self.qstats.data_ptr(), self.mu0.data_ptr(),
                               self.m2_0.data_ptr(), self.ws_pre.ptr, self.ws_pre.nbytes, self.s())
        self.tier_out = torch.full((R, N), 255, dtype=torch.uint8, device=dev)
        if r is not None:
            self.pack(k, v, ctx_len, r, self.mu0, self.m2_0)

    def pack(self, k, v, ctx_len, r, mu0, m2_0):
        abi.arkv_quantize_pack(self.cfg, r, k.data_ptr(), v.data_ptr(), self.n_stride, ctx_len.data_ptr(),
                               mu0.data_ptr(), m2_0.data_ptr(), self.cache.c, self.tier_out.data_ptr(),
                               self.ws_pre.ptr, self.ws_pre.nbytes, self.s())

    def decode(self, step, q, kn, vn, ctx_len, o):
        abi.arkv_decode_attn(self.cfg, step, q.data_ptr(), kn.data_ptr(), vn.data_ptr(), ctx_len.data_ptr(),
                             self.cache.c, o.data_ptr(), self.ws_dec.ptr, self.ws_dec.nbytes, self.s())

    def score(self, step, ctx_len):
        abi.arkv_score_update(self.cfg, step, ctx_len.data_ptr(), self.cache.c, self.ws_dec.ptr,
                              self.ws_dec.nbytes, self.s())

    def reassign(self, step, r, ctx_len):
        self.tier_dbg.fill_(255)
        abi.arkv_reassign(self.cfg, step, r, ctx_len.data_ptr(), self.cache.c, self.tier_dbg.data_ptr(),
                          self.ws_re.ptr, self.ws_re.nbytes, self.s())
