"""GPU parity of arkv_decode_attn with early_start = 1: three layers' calls issued
back to back on one stream (each may read its own cache while the previous layer's
kernel is still running), then their score updates and, every interval, their
reassignments; every output and score is compared with the oracle at every step."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from mixed_precision_kv_arkv_b200 import abi, inputs, workloads
from mixed_precision_kv_arkv_b200.build import build
from tests import harness as H

pytestmark = pytest.mark.gpu

O_TOL, S_TOL = 2e-3, 1e-5

WL = workloads.LLAMA3_3B.with_(name="three_layers_early_start", cfg_id=18, layers=3, batch=2,
                               n_ctx=3000, n_ctx_min=2200, steps=12, reassign_interval=4)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build()
    abi.lib()


def test_early_start_across_layers(cuda):
    wl, L, r = WL, WL.layers, WL.r_bar
    lays, dls, ctxs = [], [], []
    for l in range(L):
        pre = inputs.layer_prefill(wl, l, 0, seqs=None)
        ctx = pre["ctx_len"]
        lay = H.new_oracle_layer(wl, ctx)
        lay.prefill(H.F(pre["k"]), H.F(pre["v"]), H.F(pre["q_obs"]))
        lay.initial_reassign(r)
        cap_o, cap_q = H.capacities(wl, r, wl.n_ctx + wl.steps)
        dl = H.DeviceLayer(wl, cap_o, cap_q, cuda)
        dl.cfg.early_start = 1
        H.upload_rows(lay, dl.cache)                      # both sides start from the oracle's pack
        lays.append(lay), dls.append(dl), ctxs.append(torch.from_numpy(ctx).to(cuda))
    torch.cuda.synchronize()
    o = torch.zeros((L, wl.batch, wl.hq, wl.head_dim), dtype=torch.float32, device=cuda)
    worst = {"o_rel": 0.0, "s_rel": 0.0, "exempt": 0}
    for t in range(wl.steps):
        dev_in, o_ref = [], []
        for l in range(L):
            d = inputs.decode_inputs(wl, l, t, 0)
            o_ref.append(lays[l].decode_step(t, H.F(d["q"]), H.F(d["k_new"]), H.F(d["v_new"]))[0])
            dev_in.append([H.bits_to_bf16_tensor(d[k], cuda) for k in ("q", "k_new", "v_new")])
        torch.cuda.synchronize()                          # no copy into a cache right before its call
        for l in range(L):
            dls[l].decode(t, *dev_in[l], ctxs[l], o[l])
        for l in range(L):
            dls[l].score(t, ctxs[l])
        reassign = (t + 1) % wl.reassign_interval == 0
        if reassign:
            pre_rows = [{rid: H.download_row(dls[l].cache, rid) for rid in lays[l].row_ids} for l in range(L)]
        og = o.cpu().numpy()
        assert np.isfinite(og).all(), t
        for l in range(L):
            for rid in lays[l].row_ids:
                b, g = divmod(rid, wl.hkv)
                sl = slice(g * wl.group, (g + 1) * wl.group)
                worst["o_rel"] = max(worst["o_rel"], H.max_rel_per_row(og[l, b, sl], o_ref[l][b, sl]))
                gpu = H.download_row(dls[l].cache, rid)
                worst["s_rel"] = max(worst["s_rel"], H.score_rel_err(gpu, lays[l].rows[rid], wl.gamma))
        assert worst["o_rel"] <= O_TOL and worst["s_rel"] <= S_TOL, (t, worst)
        if reassign:
            recs = []
            for l in range(L):
                recs.append(lays[l].reassign(t, r))
                dls[l].reassign(t, r, ctxs[l])
            for l in range(L):
                td = dls[l].tier_dbg.cpu().numpy()
                for rid in lays[l].row_ids:
                    bad, ex = H.tier_mismatches(recs[l][rid], H.device_tiers(pre_rows[l][rid], td[rid]))
                    assert not bad, (t, l, rid, bad[:5])
                    worst["exempt"] += len(ex)
                    if ex:
                        H.upload_rows(lays[l], dls[l].cache, [rid])
                    gpu = H.download_row(dls[l].cache, rid)
                    assert np.array_equal(gpu["pos"], lays[l].rows[rid].pos), (t, l, rid)
                    assert np.array_equal(gpu["orig"], lays[l].rows[rid].orig), (t, l, rid)
                    H.assert_same_fp8(gpu, lays[l].rows[rid])
                assert int(dls[l].cache.status.item()) == 0
            torch.cuda.synchronize()
    print("early start, three layers", worst)
