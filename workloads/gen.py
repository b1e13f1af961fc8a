"""Seeded input generators (shared by the CPU oracle and the CUDA path).

Each tensor comes from its own Philox stream keyed by (seed, tensor id, layer),
so a tensor's values do not depend on which other tensors were drawn or in
which order.  bf16 tensors are returned as their raw uint16 bit patterns
(numpy has no bfloat16); `bf16_bits_to_f32` widens them exactly.

Distributions (the workload definitions of the gated-prefill benchmark):
  hidden  ~ N(0, 1), with `n_outlier_channels` seeded channels scaled by 8
  gamma   ~ 1 + N(0, 0.1)            (RMSNorm weight)
  W1      ~ N(0, 1/D)  [D, I]        (gate MLP first layer, fan_in = D)
  b1, b2  ~ N(0, 0.1)
  w2      ~ N(0, 1/I)  [I]           (gate MLP output layer, fan_in = I)
  Q, K, V ~ N(0, 1) * qkv_std
  g_h     ~ N(0, 0.5),  c_h ~ U(0, 0.5)   per query head and layer
  N(m, s) names the standard deviation s.
"""

from __future__ import annotations

import numpy as np

# tensor ids of the Philox key; fixed so that streams never collide
_ID = {
    "hidden": 1, "outliers": 2, "gamma": 3, "W1": 4, "b1": 5, "w2": 6, "b2": 7,
    "q": 10, "k": 11, "v": 12, "g": 13, "c": 14, "scores": 20,
}


def _rng(seed: int, name: str, layer: int = 0) -> np.random.Generator:
    key = np.array([np.uint64(seed), np.uint64((_ID[name] << 32) | (layer & 0xFFFFFFFF))],
                   dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even) and
    return the 16-bit patterns.  Used only to quantise synthetic inputs."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _normal_bf16(rng: np.random.Generator, shape, std: float, chunk_rows: int = 8192) -> np.ndarray:
    shape = tuple(int(s) for s in shape)
    out = np.empty(shape, dtype=np.uint16)
    if len(shape) >= 2 and shape[0] > chunk_rows:
        for r0 in range(0, shape[0], chunk_rows):
            r1 = min(shape[0], r0 + chunk_rows)
            x = rng.standard_normal((r1 - r0,) + shape[1:], dtype=np.float32)
            if std != 1.0:
                x *= np.float32(std)
            out[r0:r1] = f32_to_bf16_bits(x)
        return out
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    out[...] = f32_to_bf16_bits(x)
    return out


def make_gate_weights(w, seed: int | None = None) -> dict:
    """The gate's parameters and the hidden states' outlier channels (the small part of
    make_gate_inputs, drawn from the same streams)."""
    seed = w.seed if seed is None else seed
    D, I = w.D, w.I
    orng = _rng(seed, "outliers")
    outl = np.sort(orng.choice(D, size=w.n_outlier_channels, replace=False)) \
        if w.n_outlier_channels > 0 else np.zeros(0, dtype=np.int64)
    gamma = f32_to_bf16_bits(1.0 + 0.1 * _rng(seed, "gamma").standard_normal(D).astype(np.float32))
    W1 = _normal_bf16(_rng(seed, "W1"), (D, I), 1.0 / np.sqrt(D))
    b1 = (0.1 * _rng(seed, "b1").standard_normal(I)).astype(np.float32)
    w2 = (_rng(seed, "w2").standard_normal(I) / np.sqrt(I)).astype(np.float32)
    b2 = np.float32(0.1 * _rng(seed, "b2").standard_normal())
    return {"gamma": gamma, "W1": W1, "b1": b1, "w2": w2, "b2": float(b2),
            "outlier_channels": outl.astype(np.int64)}


def make_gate_inputs(w, seed: int | None = None) -> dict:
    """Hidden states at the gate layer plus the gate's parameters."""
    seed = w.seed if seed is None else seed
    T, D = w.T, w.D
    out = make_gate_weights(w, seed)
    hidden = np.empty((T, D), dtype=np.uint16)
    rng = _rng(seed, "hidden")
    scale = np.ones(D, dtype=np.float32)
    scale[out["outlier_channels"]] = np.float32(w.outlier_scale)
    for r0 in range(0, T, 8192):
        r1 = min(T, r0 + 8192)
        x = rng.standard_normal((r1 - r0, D), dtype=np.float32)
        x *= scale[None, :]
        hidden[r0:r1] = f32_to_bf16_bits(x)
    out["hidden"] = hidden
    return out


def make_attention_inputs(w, M: int, layer: int = 0, seed: int | None = None,
                          qkv_std: float | None = None) -> dict:
    """Upper-layer Q/K/V for M kept rows plus the layer's gain and temperature
    parameters.  They stand in for the projections of the kept hidden states."""
    seed = w.seed if seed is None else seed
    std = w.qkv_std if qkv_std is None else qkv_std
    q = _normal_bf16(_rng(seed, "q", layer), (M, w.Hq, w.d), std)
    k = _normal_bf16(_rng(seed, "k", layer), (M, w.Hkv, w.d), std)
    v = _normal_bf16(_rng(seed, "v", layer), (M, w.Hkv, w.d), std)
    g = (w.g_std * _rng(seed, "g", layer).standard_normal(w.Hq)).astype(np.float32)
    c = (w.c_high * _rng(seed, "c", layer).random(w.Hq)).astype(np.float32)
    return {"q": q, "k": k, "v": v, "g": g, "c": c}


def make_scores(n: int, std: float = 2.0, seed: int = 0, layer: int = 0) -> np.ndarray:
    """Gate scores ~ N(0, std) as float32 (inputs for selection/attention-only cases)."""
    return (std * _rng(seed, "scores", layer).standard_normal(n)).astype(np.float32)
