"""arkv_reassign_noalloc -- the reassignment for callers that cannot allocate
device memory when they reassign (inside a CUDA graph capture, under an engine
that reserved all memory up front, inside a host framework that owns the
allocator) -- must leave exactly the cache that arkv_reassign leaves, on two
reassignments in a row.  It takes no workspace: its scratch is a static device
array inside the library.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from mixed_precision_kv_arkv_b200 import abi, inputs
from mixed_precision_kv_arkv_b200.build import build
from mixed_precision_kv_arkv_b200.cache import LayerCache, Workspace, stream_ptr
from tests import harness as H
from tests.test_gpu_parity import SMALL_D128_G3

pytestmark = pytest.mark.gpu


def _clone_cache(src: LayerCache, cfg, dev) -> LayerCache:
    dst = LayerCache(cfg, dev)
    for name, _ in abi.arkv_layer_cache._fields_:
        getattr(dst, name).copy_(getattr(src, name))
    return dst


def _same_cache(a: LayerCache, b: LayerCache):
    assert torch.equal(a.n_bf16, b.n_bf16) and torch.equal(a.n_fp8, b.n_fp8)
    for rid in range(a.n_bf16.numel()):
        n16, n8 = int(a.n_bf16[rid]), int(a.n_fp8[rid])
        for name in ("k16", "v16", "pos16", "mu16", "m2_16"):
            x, y = getattr(a, name)[rid, :n16], getattr(b, name)[rid, :n16]
            assert torch.equal(x.view(torch.int16) if x.dtype == torch.bfloat16 else x,
                               y.view(torch.int16) if y.dtype == torch.bfloat16 else y), name
        for name in ("k8", "v8", "sk", "sv", "pos8", "mu8", "m2_8"):
            assert torch.equal(getattr(a, name)[rid, :n8], getattr(b, name)[rid, :n8]), name
    assert int(a.status.item()) == 0 and int(b.status.item()) == 0


def test_noalloc_reassign_matches_workspace_reassign(cuda):
    build()
    wl = SMALL_D128_G3
    r = wl.r_bar
    steps = 2 * wl.reassign_interval
    cap_o, cap_q = H.capacities(wl, r, wl.n_ctx + steps)
    a = H.DeviceLayer(wl, cap_o, cap_q, cuda)
    pre = inputs.layer_prefill(wl, 0)
    to = lambda bits: H.bits_to_bf16_tensor(bits, cuda)
    ctx = torch.from_numpy(pre["ctx_len"]).to(cuda)
    a.prefill(to(pre["k"]), to(pre["v"]), to(pre["q_obs"]), ctx, r=r)
    b_cache = _clone_cache(a.cache, a.cfg, cuda)
    b_ws = Workspace(abi.arkv_workspace_bytes(a.cfg, abi.ARKV_WS_DECODE), cuda)
    need = abi.arkv_workspace_bytes(a.cfg, abi.ARKV_WS_REASSIGN)
    assert 0 < need <= abi.ARKV_NOALLOC_SCRATCH_BYTES
    td_b = torch.full_like(a.tier_dbg, 255)
    o_a = torch.zeros((wl.batch, wl.hq, wl.head_dim), dtype=torch.float32, device=cuda)
    o_b = torch.zeros_like(o_a)
    calls = 0
    for t in range(steps):
        d = inputs.decode_inputs(wl, 0, t)
        q, kn, vn = to(d["q"]), to(d["k_new"]), to(d["v_new"])
        a.decode(t, q, kn, vn, ctx, o_a)
        a.score(t, ctx)
        abi.arkv_decode_attn(a.cfg, t, q.data_ptr(), kn.data_ptr(), vn.data_ptr(), ctx.data_ptr(),
                             b_cache.c, o_b.data_ptr(), b_ws.ptr, b_ws.nbytes, stream_ptr())
        abi.arkv_score_update(a.cfg, t, ctx.data_ptr(), b_cache.c, b_ws.ptr, b_ws.nbytes, stream_ptr())
        if (t + 1) % wl.reassign_interval == 0:
            a.reassign(t, r, ctx)
            td_b.fill_(255)
            abi.arkv_reassign_noalloc(a.cfg, t, r, ctx.data_ptr(), b_cache.c, td_b.data_ptr(),
                                      stream_ptr())
            torch.cuda.synchronize()
            assert torch.equal(a.tier_dbg, td_b)
            assert int((td_b != 255).sum()) > 0
            _same_cache(a.cache, b_cache)
            calls += 1
        assert torch.equal(o_a, o_b)
    assert calls == 2


def test_noalloc_rejects_layers_beyond_its_scratch(cuda):
    build()
    big = H.make_cfg(64, 32, 8, 128, 128, 128, 1.0, 0.25, 200_000, 200_000)
    assert abi.arkv_workspace_bytes(big, abi.ARKV_WS_REASSIGN) > abi.ARKV_NOALLOC_SCRATCH_BYTES
    dummy = torch.zeros(16, dtype=torch.int32, device=cuda)
    cache = abi.arkv_layer_cache(*[dummy.data_ptr()] * 15)
    rc = abi.arkv_reassign_noalloc(big, 0, 0.5, dummy.data_ptr(), cache, None, stream_ptr(),
                                   check=False)
    assert rc == abi.ARKV_EINVAL
    assert "scratch" in abi.arkv_last_error_string()


def test_noalloc_reassign_in_a_cuda_graph(cuda):
    """The entry point's stated use: captured into a CUDA graph (no allocation is
    possible there) and replayed, it leaves the cache that arkv_reassign leaves."""
    build()
    wl = SMALL_D128_G3
    r = wl.r_bar
    t_re = wl.reassign_interval - 1
    cap_o, cap_q = H.capacities(wl, r, wl.n_ctx + wl.reassign_interval)
    a = H.DeviceLayer(wl, cap_o, cap_q, cuda)
    pre = inputs.layer_prefill(wl, 0)
    to = lambda bits: H.bits_to_bf16_tensor(bits, cuda)
    ctx = torch.from_numpy(pre["ctx_len"]).to(cuda)
    a.prefill(to(pre["k"]), to(pre["v"]), to(pre["q_obs"]), ctx, r=r)
    o = torch.zeros((wl.batch, wl.hq, wl.head_dim), dtype=torch.float32, device=cuda)
    for t in range(t_re + 1):
        d = inputs.decode_inputs(wl, 0, t)
        a.decode(t, to(d["q"]), to(d["k_new"]), to(d["v_new"]), ctx, o)
        a.score(t, ctx)
    b_cache = _clone_cache(a.cache, a.cfg, cuda)
    warm = _clone_cache(a.cache, a.cfg, cuda)
    # the first call looks the scratch address up, which a capture does not allow
    abi.arkv_reassign_noalloc(a.cfg, t_re, r, ctx.data_ptr(), warm.c, None, stream_ptr())
    torch.cuda.synchronize()
    td_b = torch.full_like(a.tier_dbg, 255)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        abi.arkv_reassign_noalloc(a.cfg, t_re, r, ctx.data_ptr(), b_cache.c, td_b.data_ptr(), stream_ptr())
    g.replay()
    a.reassign(t_re, r, ctx)
    torch.cuda.synchronize()
    assert torch.equal(a.tier_dbg, td_b)
    assert int((td_b != 255).sum()) > 0
    _same_cache(a.cache, b_cache)
    del g
