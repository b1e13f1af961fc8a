"""Shared test helpers: moving seeded inputs onto the GPU and the parity bars."""

from __future__ import annotations

import contextlib
import os

import numpy as np
import torch

# parity bars of the gated-prefill path
SCORE_REL = 1e-4           # |s_gpu - s_ref| <= 1e-4 * max(|s_ref|, rms(s_ref))
ATTN_MAX_ABS = 2e-2        # bf16 in, fp32 accumulate
ATTN_MEAN_ABS = 2e-3
GLS_ABS = 2e-6             # fp32 logsigmoid vs fp64
LSE_ABS = 1e-3
NEAR_TIE_REL = 1e-5        # end-to-end selections may differ only among such near-ties


def bf16_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def bf16_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def f32_dev(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def i32_dev(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def score_error(s_gpu: np.ndarray, s_ref: np.ndarray) -> float:
    """max_t |s_gpu - s_ref| / max(|s_ref|, rms(s_ref)) over the given entries."""
    s_ref = np.asarray(s_ref, np.float64)
    rms = float(np.sqrt(np.mean(s_ref ** 2))) if s_ref.size else 1.0
    den = np.maximum(np.abs(s_ref), rms)
    return float(np.max(np.abs(np.asarray(s_gpu, np.float64) - s_ref) / den)) if s_ref.size else 0.0


def prunable_mask(w) -> np.ndarray:
    m = np.zeros(w.T, dtype=bool)
    cu = w.cu_seqlens()
    for b, (p0, p1) in enumerate(w.spans):
        m[cu[b] + p0: cu[b] + p1] = True
    return m


def assert_attention_close(out_gpu: np.ndarray, out_ref: np.ndarray, what: str = ""):
    err = np.abs(out_gpu.astype(np.float64) - out_ref)
    mx, mean = float(err.max()) if err.size else 0.0, float(err.mean()) if err.size else 0.0
    assert mx <= ATTN_MAX_ABS and mean <= ATTN_MEAN_ABS, f"{what}: max-abs {mx:.3e}, mean-abs {mean:.3e}"
    return mx, mean


def check_selection_swaps(keep_gpu: np.ndarray, keep_ref: np.ndarray, s_ref: np.ndarray):
    """End-to-end selections (each side on its own scores) may differ only by
    swaps of near-tied scores: every token kept by one side and dropped by the
    other must be within NEAR_TIE_REL of a token of the opposite swap set."""
    only_gpu = np.nonzero((keep_gpu == 1) & (keep_ref == 0))[0]
    only_ref = np.nonzero((keep_gpu == 0) & (keep_ref == 1))[0]
    assert len(only_gpu) == len(only_ref)
    for i in only_ref:
        tol = NEAR_TIE_REL * max(1.0, abs(float(s_ref[i])))
        assert np.any(np.abs(s_ref[only_gpu] - s_ref[i]) <= tol), f"token {i} swapped without a near-tie"
    return len(only_ref)


@contextlib.contextmanager
def attention_kernel(name):
    """Run the enclosed calls with TG_ATTENTION_KERNEL = name ("persistent" or "per_unit";
    None leaves the library's own choice); the previous setting is restored after."""
    old = os.environ.get("TG_ATTENTION_KERNEL")
    if name is not None:
        os.environ["TG_ATTENTION_KERNEL"] = name
    try:
        yield
    finally:
        if name is not None:
            if old is None:
                os.environ.pop("TG_ATTENTION_KERNEL", None)
            else:
                os.environ["TG_ATTENTION_KERNEL"] = old
