"""The five synthetic workloads the ARKV decode path is measured and checked on.

Each workload is an attention stack shaped like one of the models the ARKV page
evaluates (LLaMA3 3B/8B, Qwen3 8B; "ARKV: Adaptive and Resource-Efficient KV
Cache Management ...", 기술요약 §4 실험 결과) with a long prefill context, a
tri-state KV budget and a number of decode steps.  These records hold shapes and
policy knobs only; no arithmetic of the method lives here.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    cfg_id: int               # stream id for the seeded generator
    layers: int
    batch: int
    hq: int                   # query heads
    hkv: int                  # key/value heads
    head_dim: int
    n_ctx: int                # prefill length (maximum length for a ragged batch)
    n_ctx_min: int            # minimum prefill length (== n_ctx unless ragged)
    steps: int                # decode steps
    budget_frac: float        # beta: fraction of the full bf16 KV bytes a row may keep
    oq_ratio: float | None    # fixed Original share r, or None: per layer from prefill stats
    window: int               # W: protected most-recent tokens, always bf16
    gamma: float              # weight of the variance in S_k = mu_k + gamma * sigma_k^2
    reassign_interval: int    # T_r: decode steps between tier reassignments
    hh_frac: float            # share of prefill positions that are heavy hitters
    hh_spans: int = 0         # 0: heavy hitters uniform; else clustered in this many spans
    hh_span_len: int = 512
    r_bar: float = 0.55       # mean Original share when r comes from prefill stats
    quant_format: str = "e4m3"  # FP8 format of the Quantized tier ("e4m3" or "e5m2")

    @property
    def group(self) -> int:
        return self.hq // self.hkv

    @property
    def rows(self) -> int:
        """Rows per layer: one row is one (sequence, kv-head) pair."""
        return self.batch * self.hkv

    @property
    def n_obs(self) -> int:
        """Prefill observation queries per sequence (the last W prefill positions)."""
        return self.window

    @property
    def ragged(self) -> bool:
        return self.n_ctx_min != self.n_ctx

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY = Workload("tiny_l1_b1_h8x2_d64_n2048", 1, layers=1, batch=1, hq=8, hkv=2,
                head_dim=64, n_ctx=2048, n_ctx_min=2048, steps=16, budget_frac=0.25,
                oq_ratio=0.5, window=64, gamma=1.0, reassign_interval=1, hh_frac=0.05)

LLAMA3_3B = Workload("llama3_3b_l28_b1_h24x8_d128_n8192", 2, layers=28, batch=1, hq=24,
                     hkv=8, head_dim=128, n_ctx=8192, n_ctx_min=8192, steps=64,
                     budget_frac=0.25, oq_ratio=None, window=128, gamma=1.0,
                     reassign_interval=16, hh_frac=0.05)

LLAMA3_8B = Workload("llama3_8b_l32_b4_h32x8_d128_n32768", 3, layers=32, batch=4, hq=32,
                     hkv=8, head_dim=128, n_ctx=32768, n_ctx_min=32768, steps=128,
                     budget_frac=0.25, oq_ratio=None, window=128, gamma=1.0,
                     reassign_interval=16, hh_frac=0.05)

QWEN3_8B = Workload("qwen3_8b_l36_b1_h32x8_d128_n131072", 4, layers=36, batch=1, hq=32,
                    hkv=8, head_dim=128, n_ctx=131072, n_ctx_min=131072, steps=64,
                    budget_frac=0.25, oq_ratio=None, window=256, gamma=0.5,
                    reassign_interval=16, hh_frac=0.02, hh_spans=8, hh_span_len=512)

RAGGED = Workload("ragged_l32_b32_h32x8_d128_n4096to16384", 5, layers=32, batch=32, hq=32,
                  hkv=8, head_dim=128, n_ctx=16384, n_ctx_min=4096, steps=256,
                  budget_frac=0.30, oq_ratio=0.3, window=64, gamma=1.0,
                  reassign_interval=16, hh_frac=0.05)

ALL = (TINY, LLAMA3_3B, LLAMA3_8B, QWEN3_8B, RAGGED)

# The page's comparison axes on the LLaMA3-8B data (the same generator stream): the
# uncompressed cache (every token bf16), eviction only (Base Origin, the ARKV budget
# with no quantized tier) and quantization only (Base Quant: every non-window token
# FP8, none evicted -- the budget covers them all).
LLAMA3_8B_FULL = LLAMA3_8B.with_(name="llama3_8b_full_bf16", budget_frac=1.0, oq_ratio=1.0)
LLAMA3_8B_BASE_ORIGIN = LLAMA3_8B.with_(name="llama3_8b_base_origin", oq_ratio=1.0)
LLAMA3_8B_BASE_QUANT = LLAMA3_8B.with_(name="llama3_8b_base_quant", budget_frac=0.52, oq_ratio=0.0)
# The same ARKV workload with the Quantized tier in the other FP8 format (E5M2).
LLAMA3_8B_E5M2 = LLAMA3_8B.with_(name="llama3_8b_e5m2", quant_format="e5m2")
MODES = (LLAMA3_8B_FULL, LLAMA3_8B_BASE_ORIGIN, LLAMA3_8B_BASE_QUANT, LLAMA3_8B_E5M2)

BY_NAME = {w.name: w for w in ALL + MODES}
BY_ID = {w.cfg_id: w for w in ALL}
