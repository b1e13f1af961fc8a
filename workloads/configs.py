"""The seeded synthetic workloads of the gated-prefill path.

Every workload is one batch of sequences in the varlen layout: sequence b has
N_b tokens, one contiguous prunable span [p0_b, p1_b) (the `{state}` document
of the TokenGate README, "Quick start"), and a keep budget K_b (the
`max_kept_prefill_tokens` argument; -1 means "keep every state token").

Shapes follow Qwen3-1.7B at the gate layer (hidden 2048, 16 query heads,
8 KV heads, head_dim 128; TokenGate paper page, "Main Findings" and the
README's model list) except for the tiny oracle-sized case.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    seqlens: tuple            # N_b per sequence
    spans: tuple              # (p0_b, p1_b) per sequence, 0-indexed, half-open
    budgets: tuple            # K_b per sequence; -1 = keep all prunable tokens
    D: int                    # hidden size at the gate layer
    I: int                    # gate MLP hidden size
    Hq: int                   # query heads
    Hkv: int                  # key/value heads
    d: int                    # head_dim
    eps: float = 1e-6         # RMSNorm epsilon
    n_layers: int = 1         # gated-attention layers above the gate
    seed: int = 0
    n_outlier_channels: int = 2
    outlier_scale: float = 8.0
    qkv_std: float = 1.0 / 8.0  # "N(0,1)/sqrt(64)"
    g_std: float = 0.5
    c_high: float = 0.5
    note: str = ""
    extra: dict = field(default_factory=dict, compare=False, hash=False)

    @property
    def B(self) -> int:
        return len(self.seqlens)

    @property
    def T(self) -> int:
        return int(sum(self.seqlens))

    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int32)

    def span_array(self) -> np.ndarray:
        return np.asarray(self.spans, dtype=np.int32).reshape(self.B, 2)

    def budget_array(self) -> np.ndarray:
        return np.asarray(self.budgets, dtype=np.int32).reshape(self.B)

    def kept_counts(self) -> np.ndarray:
        """M_b = (N_b - |P_b|) + min(K_b, |P_b|), with K_b < 0 meaning all.

        This is only a shape calculation (how many rows the caller must
        allocate); it involves no score.
        """
        out = []
        for n, (p0, p1), k in zip(self.seqlens, self.spans, self.budgets):
            p = p1 - p0
            kk = p if (k < 0 or k > p) else k
            out.append(n - p + kk)
        return np.asarray(out, dtype=np.int64)

    def cu_kept(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.kept_counts())]).astype(np.int32)

    def with_budget(self, k) -> "Workload":
        return replace(self, budgets=tuple([k] * self.B),
                       name=f"{self.name.split('_k')[0]}_k{'all' if k < 0 else k}")


def _qwen3_17b(name, seqlens, spans, budgets, **kw) -> Workload:
    return Workload(name=name, seqlens=tuple(seqlens), spans=tuple(spans),
                    budgets=tuple(budgets), D=2048, I=256, Hq=16, Hkv=8, d=128, **kw)


def _varlen_budgets(seed: int, n: int, lo: float, hi: float) -> list:
    """Budgets drawn log-uniform in [lo, hi], seeded (a shape choice, not method arithmetic)."""
    rng = np.random.Generator(np.random.Philox(key=np.array([seed, 0xB0D6E7], dtype=np.uint64)))
    u = rng.random(n)
    return [int(round(math.exp(math.log(lo) + x * (math.log(hi) - math.log(lo))))) for x in u]


def masked_budgets(w: "Workload", seed: int = 0) -> list:
    """The smaller budget of a training step, one per sequence: log-uniform in
    [1, |P_b| / 2] (the pages sample it that way), seeded."""
    out = []
    for b, (p0, p1) in enumerate(w.spans):
        hi = max(1.0, (p1 - p0) / 2.0)
        out.append(_varlen_budgets(1000 + seed * 97 + b, 1, 1.0, hi)[0])
    return out


def _build() -> dict:
    cfg = {}
    cfg["c0_tiny"] = Workload(
        name="c0_tiny", seqlens=(512,), spans=((64, 448),), budgets=(64,),
        D=256, I=64, Hq=4, Hkv=2, d=64, note="tiny oracle check")
    cfg["c1_16k"] = _qwen3_17b("c1_16k", [16384], [(256, 16256)], [2000],
                               note="Qwen3-1.7B gate layer at 16k")
    for k in (100, 500, 2000, -1):
        nm = f"c2_32k_k{'all' if k < 0 else k}"
        cfg[nm] = _qwen3_17b(nm, [32768], [(128, 32640)], [k], n_layers=14,
                             note="Qwen3-1.7B at 32k, 14 gated layers above the gate")
    cfg["c3_full_budget_16k"] = _qwen3_17b(
        "c3_full_budget_16k", [16384], [(256, 16256)], [-1],
        note="training-time full-budget gated attention, masked budget")
    cfg["c4_128k"] = _qwen3_17b("c4_128k", [131072], [(128, 130944)], [2000],
                                note="long context 128k")
    # head_dim 256 (the pages' key-bias kernel serves it for the Qwen3.5 models; their
    # head counts are not given: 8 query and 2 KV heads, a small-model GQA layout)
    cfg["c5_hd256_16k"] = Workload(
        name="c5_hd256_16k", seqlens=(16384,), spans=((256, 16256),), budgets=(2000,),
        D=2048, I=256, Hq=8, Hkv=2, d=256, note="head_dim 256 at 16k")
    lens = [8192, 24576, 65536, 131072]
    cfg["c4_varlen"] = _qwen3_17b(
        "c4_varlen", lens, [(128, n - 128) for n in lens], _varlen_budgets(4, 4, 100, 4000),
        seed=4, note="varlen batch of 4, K_b log-uniform in [100, 4000]")
    return cfg


CONFIGS = _build()


def get_config(name: str) -> Workload:
    try:
        return CONFIGS[name]
    except KeyError as e:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(CONFIGS)}") from e
