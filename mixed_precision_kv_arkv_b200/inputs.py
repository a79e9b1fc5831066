"""Seeded synthetic inputs for the ARKV decode path.

This module draws random numbers and lays out the workload structure (sink
token, heavy hitters, shared query direction, ragged lengths).  It holds none
of the method's arithmetic, so both the CPU oracle's tests and the CUDA path
may take their inputs from it.

Recipe (one row = one (layer, sequence, kv-head)):
  * u = sqrt(D) * u_hat, u_hat uniform on the unit sphere, one per (layer, kv-head).
  * prefill keys and values ~ N(0, 1); position 0 is a sink whose key is 4u;
    a share of the other positions are heavy hitters whose key is z + 2u
    (uniform positions, or clustered in non-overlapping spans).
  * queries (prefill observation queries and decode queries) = z + a_l u, with u
    the direction of the query head's kv group and a_l = query_weight(layer), a
    per-layer weight around 0.5 (0.375 .. 0.625): layers differ in how sharply
    their attention concentrates on the sink and heavy hitters, so the layers'
    prefill statistics (and the Original shares drawn from them) differ.
  * decode keys and values appended each step ~ N(0, 1).
  * every value is drawn in float64 and rounded to bfloat16 (via float32, RNE).

Two back ends draw from the same recipe: numpy Philox streams keyed by
(seed, workload, layer, sequence, head, tensor) so that any subset of rows can
be regenerated on the host, and torch generators on a CUDA device for the
full-size benchmark (same distributions, different streams).
"""
from __future__ import annotations

import numpy as np

from .workloads import Workload

_TENSOR = {"dir": 1, "k": 2, "v": 3, "q_obs": 4, "hh": 5, "q": 6, "k_new": 7,
           "v_new": 8, "ctx": 9}


def query_weight(layer: int) -> float:
    """Weight a_l of the shared direction in layer l's queries: 0.5 + 0.25 (f_l - 0.5)
    with f_l = frac(0.6180339887 l), an even spread over [0.375, 0.625)."""
    f = (0.6180339887 * layer) % 1.0
    return 0.5 + 0.25 * (f - 0.5)


def _rng(seed: int, wl: Workload, layer: int, seq: int, head: int, tensor: str,
         extra: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence([seed, wl.cfg_id, layer, seq, head, _TENSOR[tensor], extra])
    return np.random.Generator(np.random.Philox(ss))


# --------------------------------------------------------------------------- bf16
def round_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> float32 (round to nearest) -> bfloat16 bits (round to nearest even)."""
    f = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((f >> 16) & 1) + 0x7FFF
    return ((f + bias) >> 16).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- structure
def ctx_lengths(wl: Workload, seed: int = 0) -> np.ndarray:
    """Prefill length of every sequence: fixed, or uniform in [n_ctx_min, n_ctx]."""
    if not wl.ragged:
        return np.full(wl.batch, wl.n_ctx, dtype=np.int32)
    rng = _rng(seed, wl, 0, 0, 0, "ctx")
    return rng.integers(wl.n_ctx_min, wl.n_ctx + 1, size=wl.batch).astype(np.int32)


def direction(wl: Workload, layer: int, g: int, seed: int = 0) -> np.ndarray:
    """u = sqrt(D) * (uniform unit vector) for kv-head g of a layer, float64 [D]."""
    z = _rng(seed, wl, layer, 0, g, "dir").standard_normal(wl.head_dim)
    return np.sqrt(wl.head_dim) * z / np.linalg.norm(z)


def heavy_hitters(wl: Workload, layer: int, b: int, g: int, n: int, seed: int = 0) -> np.ndarray:
    """Sorted heavy-hitter positions of one row (never the sink, never in the last W)."""
    rng = _rng(seed, wl, layer, b, g, "hh")
    count = int(wl.hh_frac * n)
    if wl.hh_spans == 0:
        return np.sort(rng.choice(np.arange(1, n), size=count, replace=False))
    span, hi = wl.hh_span_len, n - wl.hh_span_len - wl.window
    starts: list[int] = []
    while len(starts) < wl.hh_spans:
        s = int(rng.integers(1, hi + 1))
        if all(abs(s - t) >= span for t in starts):
            starts.append(s)
    pool = np.concatenate([np.arange(s, s + span) for s in sorted(starts)])
    return np.sort(rng.choice(pool, size=min(count, pool.size), replace=False))


# --------------------------------------------------------------------------- numpy back end
def layer_prefill(wl: Workload, layer: int, seed: int = 0, seqs=None, kv_heads=None) -> dict:
    """Prefill K, V (bf16 bits, [B, Hkv, n_ctx, D], zero past each ctx_len) and the
    observation queries (bf16 bits, [B, Hq, n_obs, D]) of one layer.

    `seqs` / `kv_heads` restrict generation to a subset of rows; the other rows
    stay zero.  Each row has its own streams, so a subset matches the full draw.
    """
    B, Hkv, D, G, N = wl.batch, wl.hkv, wl.head_dim, wl.group, wl.n_ctx
    seqs = range(B) if seqs is None else seqs
    kv_heads = range(Hkv) if kv_heads is None else kv_heads
    ctx = ctx_lengths(wl, seed)
    k = np.zeros((B, Hkv, N, D), np.uint16)
    v = np.zeros((B, Hkv, N, D), np.uint16)
    q_obs = np.zeros((B, wl.hq, wl.n_obs, D), np.uint16)
    for g in kv_heads:
        u = direction(wl, layer, g, seed)
        for b in seqs:
            n = int(ctx[b])
            kk = _rng(seed, wl, layer, b, g, "k").standard_normal((n, D))
            hh = heavy_hitters(wl, layer, b, g, n, seed)
            kk[hh] += 2.0 * u
            kk[0] = 4.0 * u
            k[b, g, :n] = round_bf16(kk)
            v[b, g, :n] = round_bf16(_rng(seed, wl, layer, b, g, "v").standard_normal((n, D)))
            for j in range(G):
                h = g * G + j
                z = _rng(seed, wl, layer, b, h, "q_obs").standard_normal((wl.n_obs, D))
                q_obs[b, h] = round_bf16(z + query_weight(layer) * u)
    return {"k": k, "v": v, "q_obs": q_obs, "ctx_len": ctx}


def decode_inputs(wl: Workload, layer: int, step: int, seed: int = 0) -> dict:
    """Decode-step query [B, Hq, D] and the appended key/value [B, Hkv, D] (bf16 bits)."""
    B, Hkv, D, G = wl.batch, wl.hkv, wl.head_dim, wl.group
    q = np.zeros((B, wl.hq, D), np.uint16)
    kn = np.zeros((B, Hkv, D), np.uint16)
    vn = np.zeros((B, Hkv, D), np.uint16)
    for g in range(Hkv):
        u = direction(wl, layer, g, seed)
        for b in range(B):
            for j in range(G):
                h = g * G + j
                z = _rng(seed, wl, layer, b, h, "q", step).standard_normal(D)
                q[b, h] = round_bf16(z + query_weight(layer) * u)
            kn[b, g] = round_bf16(_rng(seed, wl, layer, b, g, "k_new", step).standard_normal(D))
            vn[b, g] = round_bf16(_rng(seed, wl, layer, b, g, "v_new", step).standard_normal(D))
    return {"q": q, "k_new": kn, "v_new": vn}


# --------------------------------------------------------------------------- torch back end
def layer_prefill_torch(wl: Workload, layer: int, device, seed: int = 0, ctx=None) -> dict:
    """Same recipe as `layer_prefill`, drawn by torch on `device` (benchmark sizes)."""
    import torch

    B, Hkv, D, G, N = wl.batch, wl.hkv, wl.head_dim, wl.group, wl.n_ctx
    gen = torch.Generator(device=device)
    gen.manual_seed((seed * 1000003 + wl.cfg_id * 7919 + layer) & 0x7FFFFFFFFFFF)
    if ctx is None:
        ctx = ctx_lengths(wl, seed)
    f32 = torch.float32
    z = torch.randn((Hkv, D), generator=gen, device=device, dtype=f32)
    u = (D ** 0.5) * z / z.norm(dim=1, keepdim=True)                     # [Hkv, D]
    k = torch.randn((B, Hkv, N, D), generator=gen, device=device, dtype=f32)
    v = torch.randn((B, Hkv, N, D), generator=gen, device=device, dtype=f32)
    for b in range(B):
        n = int(ctx[b])
        for g in range(Hkv):
            cnt = int(wl.hh_frac * n)
            if wl.hh_spans == 0:
                hh = torch.randperm(n - 1, generator=gen, device=device)[:cnt] + 1
            else:
                span, hi = wl.hh_span_len, n - wl.hh_span_len - wl.window
                starts: list[int] = []
                while len(starts) < wl.hh_spans:
                    s = int(torch.randint(1, hi + 1, (1,), generator=gen, device=device))
                    if all(abs(s - t) >= span for t in starts):
                        starts.append(s)
                pool = torch.cat([torch.arange(s, s + span, device=device) for s in starts])
                hh = pool[torch.randperm(pool.numel(), generator=gen, device=device)[:cnt]]
            k[b, g, hh] += 2.0 * u[g]
            k[b, g, 0] = 4.0 * u[g]
            if n < N:
                k[b, g, n:] = 0
                v[b, g, n:] = 0
    q_obs = torch.randn((B, wl.hq, wl.n_obs, D), generator=gen, device=device, dtype=f32)
    q_obs += query_weight(layer) * u.repeat_interleave(G, dim=0)[None, :, None, :]
    bf = torch.bfloat16
    return {"k": k.to(bf), "v": v.to(bf), "q_obs": q_obs.to(bf), "u": u,
            "ctx_len": torch.as_tensor(np.asarray(ctx, np.int32), device=device)}


def decode_inputs_torch(wl: Workload, u: "torch.Tensor", steps: int, device, seed: int = 0,
                        layer: int = 0) -> dict:
    """Decode queries and appended K/V for `steps` steps of one layer, drawn on `device`.

    Shapes: q [steps, B, Hq, D], k_new / v_new [steps, B, Hkv, D], all bfloat16.
    """
    import torch

    B, Hkv, D, G = wl.batch, wl.hkv, wl.head_dim, wl.group
    gen = torch.Generator(device=device)
    gen.manual_seed((seed * 1000033 + wl.cfg_id * 104729 + layer + 17) & 0x7FFFFFFFFFFF)
    q = torch.randn((steps, B, wl.hq, D), generator=gen, device=device)
    q += query_weight(layer) * u.repeat_interleave(G, dim=0)[None, None]
    kn = torch.randn((steps, B, Hkv, D), generator=gen, device=device)
    vn = torch.randn((steps, B, Hkv, D), generator=gen, device=device)
    bf = torch.bfloat16
    return {"q": q.to(bf), "k_new": kn.to(bf), "v_new": vn.to(bf)}
