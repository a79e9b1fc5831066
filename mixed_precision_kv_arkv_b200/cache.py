"""Device-memory plumbing around libarkv: torch tensors for one layer's packed
cache and workspaces, and a per-layer driver that issues the C-ABI calls of the
decode path in order.  Nothing here computes any part of the method.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import abi


def make_cfg(batch, hq, hkv, head_dim, window, n_obs, gamma, budget_frac, cap_bf16, cap_fp8,
             quant_format="e4m3", early_start=False):
    return abi.arkv_cfg(batch, hq, hkv, head_dim, window, n_obs, float(gamma), float(budget_frac),
                        cap_bf16, cap_fp8, abi.FORMATS[quant_format], int(bool(early_start)))


class LayerCache:
    """The tri-state cache of one layer (see include/arkv.h, Layout)."""

    def __init__(self, cfg: abi.arkv_cfg, device):
        R, D = cfg.batch * cfg.hkv, cfg.head_dim
        co, cq = cfg.cap_bf16, cfg.cap_fp8
        i32, f32, f64, u8 = torch.int32, torch.float32, torch.float64, torch.uint8
        self.cfg = cfg
        self.k16 = torch.zeros((R, co, D), dtype=torch.bfloat16, device=device)
        self.v16 = torch.zeros((R, co, D), dtype=torch.bfloat16, device=device)
        self.pos16 = torch.zeros((R, co), dtype=i32, device=device)
        self.mu16 = torch.zeros((R, co), dtype=f64, device=device)
        self.m2_16 = torch.zeros((R, co), dtype=f64, device=device)
        self.k8 = torch.zeros((R, cq, D), dtype=u8, device=device)
        self.v8 = torch.zeros((R, cq, D), dtype=u8, device=device)
        self.sk = torch.zeros((R, cq), dtype=f32, device=device)
        self.sv = torch.zeros((R, cq), dtype=f32, device=device)
        self.pos8 = torch.zeros((R, cq), dtype=i32, device=device)
        self.mu8 = torch.zeros((R, cq), dtype=f64, device=device)
        self.m2_8 = torch.zeros((R, cq), dtype=f64, device=device)
        self.n_bf16 = torch.zeros((R,), dtype=i32, device=device)
        self.n_fp8 = torch.zeros((R,), dtype=i32, device=device)
        self.status = torch.zeros((1,), dtype=i32, device=device)
        self.c = abi.arkv_layer_cache(*[getattr(self, n).data_ptr() for n, _ in
                                        abi.arkv_layer_cache._fields_])

    def nbytes(self) -> int:
        return sum(getattr(self, n).numel() * getattr(self, n).element_size()
                   for n, _ in abi.arkv_layer_cache._fields_)


class Workspace:
    """A zero-filled, 256-byte aligned device workspace of a given size."""

    def __init__(self, nbytes: int, device):
        self.buf = torch.zeros(max(int(nbytes), 1) + 256, dtype=torch.uint8, device=device)
        base = self.buf.data_ptr()
        self.off = (-base) % 256
        self.ptr = base + self.off
        self.nbytes = int(nbytes)


def stream_ptr(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


@dataclass
class LayerState:
    """What the decode loop of one layer holds on the device."""
    cfg: abi.arkv_cfg
    cache: LayerCache
    ws_decode: Workspace
    ws_reassign: Workspace
    r: float


def new_layer_state(cfg: abi.arkv_cfg, r: float, device) -> LayerState:
    return LayerState(cfg, LayerCache(cfg, device),
                      Workspace(abi.arkv_workspace_bytes(cfg, abi.ARKV_WS_DECODE), device),
                      Workspace(abi.arkv_workspace_bytes(cfg, abi.ARKV_WS_REASSIGN), device), float(r))


def decode_step(st: LayerState, step: int, q, k_new, v_new, ctx_len, o, reassign_interval: int,
                stream=None, tier_dbg=None):
    """One decode step of one layer: append + attend, score update, and a
    reassignment when (step + 1) % reassign_interval == 0."""
    s = stream_ptr(stream)
    abi.arkv_decode_attn(st.cfg, step, q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(),
                         ctx_len.data_ptr(), st.cache.c, o.data_ptr(), st.ws_decode.ptr,
                         st.ws_decode.nbytes, s)
    abi.arkv_score_update(st.cfg, step, ctx_len.data_ptr(), st.cache.c, st.ws_decode.ptr,
                          st.ws_decode.nbytes, s)
    if (step + 1) % reassign_interval == 0:
        abi.arkv_reassign(st.cfg, step, st.r, ctx_len.data_ptr(), st.cache.c,
                          tier_dbg.data_ptr() if tier_dbg is not None else None,
                          st.ws_reassign.ptr, st.ws_reassign.nbytes, s)
