"""The benchmark's CPU-baseline leg reads one row of the benchmarked cache back into
the oracle and checks one decode step against the device.  Here the "device" is a
CPU-resident cache driven by the oracle itself, so the row read back (positions,
tiers, values, Welford counts derived from the positions) must reproduce the oracle
exactly and the check must report no error."""
import numpy as np
import torch

import bench
from mixed_precision_kv_arkv_b200 import inputs, workloads
from mixed_precision_kv_arkv_b200.cache import LayerCache, make_cfg
from tests import harness as H


def test_check_on_benchmarked_state_is_exact_when_the_device_is_the_oracle():
    wl = workloads.TINY.with_(reassign_interval=4)
    r = wl.oq_ratio
    pre = inputs.layer_prefill(wl, 0)
    lay = H.new_oracle_layer(wl, pre["ctx_len"])
    lay.prefill(H.F(pre["k"]), H.F(pre["v"]), H.F(pre["q_obs"]))
    lay.initial_reassign(r)
    steps = 6                                     # decode steps already taken on the "device"
    dec = {k: [] for k in ("q", "k_new", "v_new")}
    for t in range(steps + 1):
        d = inputs.decode_inputs(wl, 0, t)
        for k in dec:
            dec[k].append(d[k])
        if t < steps:
            lay.decode_step(t, H.F(d["q"]), H.F(d["k_new"]), H.F(d["v_new"]))
            if (t + 1) % wl.reassign_interval == 0:
                lay.reassign(t, r)
    cap_o, cap_q = H.capacities(wl, r, wl.n_ctx + steps + 8)
    cfg = make_cfg(wl.batch, wl.hq, wl.hkv, wl.head_dim, wl.window, wl.n_obs, wl.gamma, wl.budget_frac,
                   cap_o, cap_q)
    cache = LayerCache(cfg, "cpu")
    H.upload_rows(lay, cache)
    to_t = lambda a: torch.from_numpy(np.stack(a).view(np.int16)).view(torch.bfloat16)
    lay0 = {"cache": cache, "dec": {k: to_t(v) for k, v in dec.items()}, "r": r}
    o = torch.zeros((1, wl.batch, wl.hq, wl.head_dim), dtype=torch.float32)

    def device_step(t):                           # the oracle plays the device
        d = inputs.decode_inputs(wl, 0, t)
        og, _ = lay.decode_step(t, H.F(d["q"]), H.F(d["k_new"]), H.F(d["v_new"]))
        o[0] = torch.from_numpy(og.astype(np.float32))
        H.upload_rows(lay, cache)

    out = bench.cpu_baseline_from_state(wl, lay0, pre["ctx_len"], steps, o, 0.2, device_step)
    chk = out["check_on_benchmarked_state"]
    assert chk["positions_equal"] and chk["ok"], chk
    assert chk["o_rel"] < 1e-6 and chk["s_rel"] < 1e-12, chk
    assert out["value"] > 0 and out["single_thread"]["value"] > 0 and out["nproc"] >= 1
