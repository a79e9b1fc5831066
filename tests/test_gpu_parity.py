"""GPU parity: every C-ABI call against the CPU oracle on the same seeded inputs.

Tolerances: FP8 codes and scales bit-exact; tiers bit-exact except tokens whose
oracle score lies within 1e-6 relative of a cut; scores S within 1e-5 relative;
attention outputs within 2e-3 of the row's largest magnitude (max over each
output row); prefill statistics (float64 on both sides) within 1e-8 relative."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from mixed_precision_kv_arkv_b200 import abi, inputs, workloads
from mixed_precision_kv_arkv_b200.build import build
from oracle import arkv as A
from oracle import e4m3, e5m2
from tests import harness as H

pytestmark = pytest.mark.gpu

O_TOL, S_TOL, STAT_TOL = 2e-3, 1e-5, 1e-8


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    abi.lib()


def to_dev(bits, dev):
    return H.bits_to_bf16_tensor(bits, dev)


# ------------------------------------------------------------------ FP8 conversion
@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_fp8_encode_exhaustive(cuda, fmt):
    """All 2^32 float32 bit patterns: device conversion == oracle encoder (NaN
    inputs: a NaN code of the format, sign not compared)."""
    codec = {"e4m3": e4m3, "e5m2": e5m2}[fmt]
    chunk = 1 << 28
    out = torch.empty(chunk, dtype=torch.uint8, device=cuda)
    idx = torch.arange(chunk, dtype=torch.int64, device=cuda)
    for c in range((1 << 32) // chunk):
        start = c * chunk
        b = idx + start
        b = torch.where(b >= (1 << 31), b - (1 << 32), b).to(torch.int32).view(torch.float32)
        abi.arkv_fp8_encode(abi.FORMATS[fmt], b.data_ptr(), out.data_ptr(), chunk, H.stream_ptr())
        got = out.cpu().numpy()
        ref = codec.encode_bits_range(start, chunk)
        bits = (np.arange(chunk, dtype=np.uint64) + start).astype(np.uint32)
        isnan = ((bits & 0x7F800000) == 0x7F800000) & ((bits & 0x007FFFFF) != 0)
        assert np.array_equal(got[~isnan], ref[~isnan]), f"chunk {c}"
        g = got[isnan]
        if fmt == "e4m3":
            assert ((g & 0x7F) == 0x7F).all()
        else:   # exponent all ones and a nonzero mantissa
            assert ((g & 0x7C) == 0x7C).all() and ((g & 0x03) != 0).all()


# ------------------------------------------------------------------ scenario runner
def _r_for(wl):
    return wl.oq_ratio if wl.oq_ratio is not None else wl.r_bar


def run_scenario(wl, steps, dev, rows=None, r=None, kernel_parity=False, seed=0, layer=0,
                 exempt_budget=0.002):
    """Prefill, initial pack and `steps` decode steps on both sides, compared at
    every call.  Free-running unless kernel_parity (then every step starts from the
    oracle's state).  Returns a summary of the largest errors seen."""
    r = _r_for(wl) if r is None else r
    pre = inputs.layer_prefill(wl, layer, seed, seqs=None)
    ctx = pre["ctx_len"]
    lay = H.new_oracle_layer(wl, ctx, rows)
    lay.prefill(H.F(pre["k"]), H.F(pre["v"]), H.F(pre["q_obs"]))
    rows = lay.row_ids
    cap_o, cap_q = H.capacities(wl, r, wl.n_ctx + steps)
    dl = H.DeviceLayer(wl, cap_o, cap_q, dev)
    k_t, v_t, q_t = to_dev(pre["k"], dev), to_dev(pre["v"], dev), to_dev(pre["q_obs"], dev)
    ctx_t = torch.from_numpy(ctx).to(dev)
    dl.prefill(k_t, v_t, q_t, ctx_t, r=None)
    torch.cuda.synchronize()
    summary = {"stat_rel": 0.0, "s0_rel": 0.0, "o_rel": 0.0, "s_rel": 0.0, "exempt": 0, "tokens": 0}

    # prefill statistics and initial scores
    qs = dl.qstats.cpu().numpy()
    for rid in rows:
        b, g = divmod(rid, wl.hkv)
        ref = lay.query_stats[rid]                               # [G, n_obs, 3]
        got = qs[b, g * wl.group:(g + 1) * wl.group]
        rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-12)
        summary["stat_rel"] = max(summary["stat_rel"], float(rel.max()))
        row = lay.rows[rid]
        n = int(ctx[b])
        S_ref = A.heavy_hitter_score(row.mu, row.m2, row.cnt, wl.gamma)
        mu_g = dl.mu0[rid, :n].double().cpu().numpy()
        m2_g = dl.m2_0[rid, :n].double().cpu().numpy()
        S_g = mu_g + wl.gamma * m2_g / row.cnt
        summary["s0_rel"] = max(summary["s0_rel"], float(np.max(np.abs(S_g - S_ref) / S_ref)))
    assert summary["stat_rel"] <= STAT_TOL, summary
    assert summary["s0_rel"] <= S_TOL, summary

    # initial pack, from the oracle's prefill scores (kernel parity of the pack)
    mu0 = torch.zeros_like(dl.mu0)
    m20 = torch.zeros_like(dl.m2_0)
    for rid in rows:
        row = lay.rows[rid]
        mu0[rid, :len(row.mu)] = torch.from_numpy(row.mu.astype(np.float64)).to(dev)
        m20[rid, :len(row.m2)] = torch.from_numpy(row.m2.astype(np.float64)).to(dev)
    dl.pack(k_t, v_t, ctx_t, r, mu0, m20)
    recs = lay.initial_reassign(r)
    tier_out = dl.tier_out.cpu().numpy()
    for rid in rows:
        n = int(ctx[rid // wl.hkv])
        tiers = {p: int(tier_out[rid, p]) for p in range(n)}
        bad, ex = H.tier_mismatches(recs[rid], tiers)
        assert not bad, (rid, bad[:5])
        summary["exempt"] += len(ex)
        if ex:
            H.upload_rows(lay, dl.cache, [rid])
        gpu = H.download_row(dl.cache, rid)
        assert np.array_equal(gpu["pos"], lay.rows[rid].pos)
        assert np.array_equal(gpu["orig"], lay.rows[rid].orig)
        H.assert_same_fp8(gpu, lay.rows[rid])
        H.assert_same_bf16(gpu, lay.rows[rid])
    assert int(dl.cache.status.item()) == 0

    o = torch.zeros((wl.batch, wl.hq, wl.head_dim), dtype=torch.float32, device=dev)
    summary["log"] = []                     # one record per reassignment interval
    iv = {"o_rel": 0.0, "s_rel": 0.0}
    for t in range(steps):
        if kernel_parity:
            H.upload_rows(lay, dl.cache, rows)
        d = inputs.decode_inputs(wl, layer, t, seed)
        o_ref, _ = lay.decode_step(t, H.F(d["q"]), H.F(d["k_new"]), H.F(d["v_new"]))
        dl.decode(t, to_dev(d["q"], dev), to_dev(d["k_new"], dev), to_dev(d["v_new"], dev), ctx_t, o)
        dl.score(t, ctx_t)
        og = o.cpu().numpy()
        assert np.isfinite(og).all(), (t, np.argwhere(~np.isfinite(og).all(-1)).tolist()[:8])  # every row, not only the compared ones
        for rid in rows:
            b, g = divmod(rid, wl.hkv)
            sl = slice(g * wl.group, (g + 1) * wl.group)
            iv["o_rel"] = max(iv["o_rel"], H.max_rel_per_row(og[b, sl], o_ref[b, sl]))
            gpu = H.download_row(dl.cache, rid)
            iv["s_rel"] = max(iv["s_rel"], H.score_rel_err(gpu, lay.rows[rid], wl.gamma))
        summary["o_rel"] = max(summary["o_rel"], iv["o_rel"])
        summary["s_rel"] = max(summary["s_rel"], iv["s_rel"])
        assert summary["o_rel"] <= O_TOL, (t, summary)
        assert summary["s_rel"] <= S_TOL, (t, summary)
        if (t + 1) % wl.reassign_interval == 0:
            exempt_before = summary["exempt"]
            pre_rows = {rid: H.download_row(dl.cache, rid) for rid in rows}
            recs = lay.reassign(t, r)
            dl.reassign(t, r, ctx_t)
            td = dl.tier_dbg.cpu().numpy()
            for rid in rows:
                tiers = H.device_tiers(pre_rows[rid], td[rid])
                bad, ex = H.tier_mismatches(recs[rid], tiers)
                assert not bad, (t, rid, bad[:5])
                summary["exempt"] += len(ex)
                summary["tokens"] += len(recs[rid]["pos"])
                if ex:
                    H.upload_rows(lay, dl.cache, [rid])
                gpu = H.download_row(dl.cache, rid)
                assert np.array_equal(gpu["pos"], lay.rows[rid].pos), (t, rid)
                assert np.array_equal(gpu["orig"], lay.rows[rid].orig), (t, rid)
                H.assert_same_fp8(gpu, lay.rows[rid])
                H.assert_same_bf16(gpu, lay.rows[rid])
                n_t = int(ctx[rid // wl.hkv]) + t + 1
                win = gpu["pos"] >= n_t - wl.window
                assert win.sum() == wl.window and gpu["orig"][win].all()
            assert int(dl.cache.status.item()) == 0
            rec = {"step": t, "o_rel": iv["o_rel"], "s_rel": iv["s_rel"],
                   "exempt": summary["exempt"] - exempt_before,
                   "tokens": sum(len(recs[rid]["pos"]) for rid in rows)}
            summary["log"].append(rec)
            print(f"PARITY {wl.name} rows={list(rows)} " + " ".join(f"{k}={v:.3g}" if isinstance(v, float)
                                                                 else f"{k}={v}" for k, v in rec.items()))
            iv = {"o_rel": 0.0, "s_rel": 0.0}
    if summary["tokens"]:
        assert summary["exempt"] <= exempt_budget * summary["tokens"] + 2, summary
    return summary


# ------------------------------------------------------------------ scenarios
def test_tiny_free_running_lockstep(cuda):
    s = run_scenario(workloads.TINY, workloads.TINY.steps, cuda)
    print("tiny free-running", s)


def test_tiny_kernel_parity(cuda):
    s = run_scenario(workloads.TINY, 8, cuda, kernel_parity=True)
    print("tiny kernel parity", s)


SMALL_D128_G3 = workloads.LLAMA3_3B.with_(name="small_d128_g3", cfg_id=11, layers=1, batch=2,
                                          n_ctx=3000, n_ctx_min=3000, steps=20, reassign_interval=4)
SMALL_RAGGED = workloads.RAGGED.with_(name="small_ragged", cfg_id=12, layers=1, batch=3, hq=8, hkv=2,
                                      n_ctx=2600, n_ctx_min=700, steps=12, reassign_interval=3)
SMALL_CLUSTER = workloads.QWEN3_8B.with_(name="small_clustered", cfg_id=13, layers=1, hq=8, hkv=2,
                                         n_ctx=6000, n_ctx_min=6000, steps=8, reassign_interval=4,
                                         hh_span_len=128)


# query groups of one and two heads (the unused columns of the query operand stay zero)
SMALL_D128_G1 = workloads.LLAMA3_3B.with_(name="small_d128_g1", cfg_id=14, layers=1, batch=2, hq=4, hkv=4,
                                          n_ctx=2500, n_ctx_min=2500, steps=8, reassign_interval=4)
SMALL_D64_G2 = workloads.TINY.with_(name="small_d64_g2", cfg_id=15, hq=4, hkv=2, steps=8)


# the Quantization tier in the second FP8 format (E5M2), at both head dims
SMALL_E5M2_D128 = SMALL_D128_G3.with_(name="small_e5m2_d128", cfg_id=16, quant_format="e5m2")
TINY_E5M2 = workloads.TINY.with_(name="tiny_e5m2", cfg_id=17, quant_format="e5m2")


@pytest.mark.parametrize("wl", [SMALL_D128_G3, SMALL_RAGGED, SMALL_CLUSTER, SMALL_D128_G1, SMALL_D64_G2,
                                SMALL_E5M2_D128, TINY_E5M2],
                         ids=lambda w: w.name)
def test_small_workloads(cuda, wl):
    s = run_scenario(wl, wl.steps, cuda)
    print(wl.name, s)


def test_base_origin_and_base_quant_modes(cuda):
    """r = 1: eviction only, no FP8 (the page's Base Origin); r = 0 with a budget
    above the all-quantized size: every non-window token FP8, nothing evicted
    (Base Quant)."""
    wl = workloads.TINY.with_(steps=4)
    run_scenario(wl, 4, cuda, r=1.0)
    wlq = workloads.TINY.with_(name="tiny_all_quant", budget_frac=1.0, steps=4)
    run_scenario(wlq, 4, cuda, r=0.0)


def test_uniform_attention_ties_break_by_position(cuda):
    """q = 0 gives every prefill key the same observations, so many scores tie
    exactly; the kept set must be the lowest positions among the tied ones, and
    the device must choose exactly the oracle's tokens (no exemption)."""
    wl = workloads.TINY
    pre = inputs.layer_prefill(wl, 0)
    pre["q_obs"][:] = 0
    ctx = pre["ctx_len"]
    lay = H.new_oracle_layer(wl, ctx)
    lay.prefill(H.F(pre["k"]), H.F(pre["v"]), H.F(pre["q_obs"]))
    cap_o, cap_q = H.capacities(wl, 0.5, wl.n_ctx + 4)
    dl = H.DeviceLayer(wl, cap_o, cap_q, cuda)
    k_t, v_t, q_t = to_dev(pre["k"], cuda), to_dev(pre["v"], cuda), to_dev(pre["q_obs"], cuda)
    ctx_t = torch.from_numpy(ctx).to(cuda)
    dl.prefill(k_t, v_t, q_t, ctx_t, r=None)
    mu0, m20 = torch.zeros_like(dl.mu0), torch.zeros_like(dl.m2_0)
    for rid, row in lay.rows.items():
        mu0[rid, :len(row.mu)] = torch.from_numpy(row.mu.astype(np.float64)).to(cuda)
        m20[rid, :len(row.m2)] = torch.from_numpy(row.m2.astype(np.float64)).to(cuda)
    dl.pack(k_t, v_t, ctx_t, 0.5, mu0, m20)
    recs = lay.initial_reassign(0.5)
    tier_out = dl.tier_out.cpu().numpy()
    for rid, rec in recs.items():
        got = np.array([tier_out[rid, p] for p in rec["pos"]])
        assert np.array_equal(got, rec["tier"])
        c = rec["cand"]
        kept = rec["pos"][c & (rec["tier"] != A.EVICTED)]
        ev = rec["pos"][c & (rec["tier"] == A.EVICTED)]
        assert len(np.unique(rec["S"][c])) < len(rec["S"][c]) // 2   # the scores do tie
        assert kept.max() < ev.min()
        orig = rec["pos"][c & (rec["tier"] == A.ORIGINAL)]
        assert orig.max() < rec["pos"][c & (rec["tier"] == A.QUANTIZED)].min()


def test_append_into_full_bf16_segment_is_flagged_not_written(cuda):
    wl = workloads.TINY
    pre = inputs.layer_prefill(wl, 0)
    ctx = pre["ctx_len"]
    lay = H.new_oracle_layer(wl, ctx)
    lay.prefill(H.F(pre["k"]), H.F(pre["v"]), H.F(pre["q_obs"]))
    lay.initial_reassign(0.5)
    n_o = max(int(row.orig.sum()) for row in lay.rows.values())
    n_q = max(int((~row.orig).sum()) for row in lay.rows.values())
    dl = H.DeviceLayer(wl, n_o, n_q, cuda)
    H.upload_rows(lay, dl.cache)
    d = inputs.decode_inputs(wl, 0, 0)
    o = torch.zeros((wl.batch, wl.hq, wl.head_dim), dtype=torch.float32, device=cuda)
    dl.decode(0, to_dev(d["q"], cuda), to_dev(d["k_new"], cuda), to_dev(d["v_new"], cuda),
              torch.from_numpy(ctx).to(cuda), o)
    torch.cuda.synchronize()
    assert int(dl.cache.status.item()) & abi.ARKV_STATUS_BF16_FULL
    assert dl.cache.n_bf16.cpu().tolist() == [int(r.orig.sum()) for r in lay.rows.values()]
    assert torch.isfinite(o).all()
