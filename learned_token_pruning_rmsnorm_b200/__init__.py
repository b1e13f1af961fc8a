"""TokenGate gated-prefill hot path on B200 (sm_100a).

Thin Python binding over the C ABI of libtokengate.so (include/tokengate.h).
The functions carry the C names; each marshals torch CUDA tensors into raw
pointers plus the current stream and calls the library.  Nothing here
computes: scoring, selection, compaction and attention all run in the CUDA
kernels, and a missing library is an error, not a fallback.

Tensors: bf16 as torch.bfloat16, fp32 as torch.float32, indices as
torch.int32, keep flags as torch.uint8; all contiguous on one CUDA device.
"""

from __future__ import annotations

import ctypes as C
import math

import numpy as np
import torch

from . import _lib
from ._lib import TokenGateError, load  # noqa: F401

__all__ = [
    "TokenGateError", "load", "tg_abi_version", "tg_kept_count", "tg_gate_prepare", "tg_score",
    "tg_select_topk", "tg_compact", "tg_gather_kept", "tg_gather_rows", "tg_gated_attention",
    "tg_gated_attention_gates", "tg_next_gate_span", "tg_gated_attention_backward", "tg_masked_gated_attention",
    "tg_gated_prefill_layer",
    "tg_device_status", "tg_selftest_bounded_wait",
]


def _dev(t: torch.Tensor, dtype, name: str, shape=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _i32_dev(a, device, name: str) -> torch.Tensor:
    if isinstance(a, torch.Tensor) and a.is_cuda:
        return _dev(a, torch.int32, name)
    return torch.from_numpy(_lib.host_i32(a)).to(device)


def tg_abi_version() -> int:
    return int(load().tg_abi_version())


def tg_kept_count(cu_seqlens, span, k):
    """Host-side kept counts: returns (M_total, cu_kept as a numpy int32 array)."""
    cu = _lib.host_i32(cu_seqlens)
    sp = _lib.host_i32(span).reshape(-1)
    kk = _lib.host_i32(k).reshape(-1)
    B = len(cu) - 1
    out = np.zeros(B + 1, dtype=np.int32)
    tot = load().tg_kept_count(cu.ctypes.data, sp.ctypes.data, kk.ctypes.data, B, out.ctypes.data)
    if tot < 0:
        _lib.check(_lib.TG_ERR_INVALID_ARG)
    return int(tot), out


def tg_gate_prepare(gamma: torch.Tensor, W1: torch.Tensor, Wg: torch.Tensor | None = None) -> torch.Tensor:
    D, I = W1.shape
    _dev(gamma, torch.bfloat16, "gamma", (D,))
    _dev(W1, torch.bfloat16, "W1")
    if Wg is None:
        Wg = torch.empty((I, D), dtype=torch.bfloat16, device=W1.device)
    _dev(Wg, torch.bfloat16, "Wg", (I, D))
    _lib.check(load().tg_gate_prepare(gamma.data_ptr(), W1.data_ptr(), D, I, Wg.data_ptr(),
                                      _lib.stream_handle(W1.device)))
    return Wg


def tg_score(hidden, cu_seqlens, span, Wg, b1, w2, b2: float, eps: float = 1e-6, scores=None):
    T, D = hidden.shape
    I = Wg.shape[0]
    dev = hidden.device
    _dev(hidden, torch.bfloat16, "hidden")
    _dev(Wg, torch.bfloat16, "Wg", (I, D))
    _dev(b1, torch.float32, "b1", (I,))
    _dev(w2, torch.float32, "w2", (I,))
    cu = _i32_dev(cu_seqlens, dev, "cu_seqlens")
    sp = _i32_dev(span, dev, "span")
    if scores is None:
        scores = torch.zeros(T, dtype=torch.float32, device=dev)
    _dev(scores, torch.float32, "scores", (T,))
    _lib.check(load().tg_score(hidden.data_ptr(), cu.data_ptr(), sp.data_ptr(), cu.numel() - 1, T, D,
                               Wg.data_ptr(), b1.data_ptr(), w2.data_ptr(), float(b2), I, float(eps),
                               scores.data_ptr(), _lib.stream_handle(dev)))
    return scores


def tg_select_topk(scores, cu_seqlens, span, k, keep=None, cu_kept=None, M_total=None):
    """Keep flags [T] uint8.  With cu_kept and M_total also returns the fused
    compaction map (kept_idx, pos, rank, gls) written by the same pass."""
    T = scores.shape[0]
    dev = scores.device
    _dev(scores, torch.float32, "scores")
    cu = _i32_dev(cu_seqlens, dev, "cu_seqlens")
    sp = _i32_dev(span, dev, "span")
    kk = _i32_dev(k, dev, "k")
    if keep is None:
        keep = torch.empty(T, dtype=torch.uint8, device=dev)
    _dev(keep, torch.uint8, "keep", (T,))
    emit = cu_kept is not None
    cmap = None
    if emit:
        M = int(M_total)
        ck = _i32_dev(cu_kept, dev, "cu_kept")
        cmap = {"kept_idx": torch.empty(M, dtype=torch.int32, device=dev),
                "pos": torch.empty(M, dtype=torch.int32, device=dev),
                "rank": torch.empty(M, dtype=torch.int32, device=dev),
                "gls": torch.empty(M, dtype=torch.float32, device=dev)}
        if M == 0:
            emit = False
    _lib.check(load().tg_select_topk(scores.data_ptr(), cu.data_ptr(), sp.data_ptr(), kk.data_ptr(),
                                     cu.numel() - 1, T, keep.data_ptr(),
                                     ck.data_ptr() if emit else None,
                                     cmap["kept_idx"].data_ptr() if emit else None,
                                     cmap["pos"].data_ptr() if emit else None,
                                     cmap["rank"].data_ptr() if emit else None,
                                     cmap["gls"].data_ptr() if emit else None, _lib.stream_handle(dev)))
    return keep if cmap is None else (keep, cmap)


def tg_gather_kept(hidden, kept_idx, hidden_kept=None):
    """Row gather of a compaction map written by tg_select_topk (tg_compact
    with keep = NULL)."""
    T, D = hidden.shape
    M = kept_idx.shape[0]
    dev = hidden.device
    _dev(hidden, torch.bfloat16, "hidden")
    _dev(kept_idx, torch.int32, "kept_idx")
    if hidden_kept is None:
        hidden_kept = torch.empty((M, D), dtype=torch.bfloat16, device=dev)
    _dev(hidden_kept, torch.bfloat16, "hidden_kept", (M, D))
    _lib.check(load().tg_compact(hidden.data_ptr(), None, None, None, None, 1, T, D, None, M,
                                 hidden_kept.data_ptr(), None, None, None, kept_idx.data_ptr(),
                                 _lib.stream_handle(dev)))
    return hidden_kept


def tg_gather_rows(src, kept_idx, dst=None):
    """dst[m] = src[kept_idx[m]] for any contiguous device tensor src of shape
    [T, ...] whose rows are 4 or 8 bytes or a multiple of 16 bytes (e.g. a
    layer's [T, Hkv, d] K or V cache, or a [T] int32 position map).  Returns
    dst ([M, ...], same dtype)."""
    if not src.is_cuda or not src.is_contiguous():
        raise ValueError("src must be a contiguous CUDA tensor")
    _dev(kept_idx, torch.int32, "kept_idx")
    T = src.shape[0]
    M = kept_idx.shape[0]
    row_bytes = (src[0].numel() if T > 0 else int(np.prod(src.shape[1:]))) * src.element_size()
    if dst is None:
        dst = torch.empty((M,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    if not dst.is_contiguous() or dst.dtype != src.dtype or tuple(dst.shape) != (M,) + tuple(src.shape[1:]):
        raise ValueError("dst must be a contiguous [M, ...] tensor of src's dtype")
    _lib.check(load().tg_gather_rows(src.data_ptr(), T, row_bytes, kept_idx.data_ptr(), M, _lib.ptr(dst),
                                     _lib.stream_handle(src.device)))
    return dst


def tg_compact(hidden, scores, keep, cu_seqlens, span, cu_kept, M_total: int, with_hidden: bool = True):
    """Returns a dict with hidden_kept (or None), pos, rank, gls, kept_idx."""
    T = scores.shape[0]
    dev = scores.device
    _dev(scores, torch.float32, "scores", (T,))
    _dev(keep, torch.uint8, "keep", (T,))
    D = hidden.shape[1] if hidden is not None else 0
    if hidden is not None:
        _dev(hidden, torch.bfloat16, "hidden", (T, D))
    cu = _i32_dev(cu_seqlens, dev, "cu_seqlens")
    sp = _i32_dev(span, dev, "span")
    ck = _i32_dev(cu_kept, dev, "cu_kept")
    M = int(M_total)
    hk = torch.empty((M, D), dtype=torch.bfloat16, device=dev) if (with_hidden and hidden is not None) else None
    pos = torch.empty(M, dtype=torch.int32, device=dev)
    rank = torch.empty(M, dtype=torch.int32, device=dev)
    gls = torch.empty(M, dtype=torch.float32, device=dev)
    kept_idx = torch.empty(M, dtype=torch.int32, device=dev)
    _lib.check(load().tg_compact(_lib.ptr(hidden), scores.data_ptr(), keep.data_ptr(), cu.data_ptr(),
                                 sp.data_ptr(), cu.numel() - 1, T, D, ck.data_ptr(), M, _lib.ptr(hk),
                                 pos.data_ptr(), rank.data_ptr(), gls.data_ptr(), kept_idx.data_ptr(),
                                 _lib.stream_handle(dev)))
    return {"hidden_kept": hk, "pos": pos, "rank": rank, "gls": gls, "kept_idx": kept_idx}


_WS_CACHE = {}


def prefill_workspace(B: int, max_M: int, Hq: int, Hkv: int, d: int, n_layers: int, device) -> torch.Tensor | None:
    """Zero-filled scratch for tg_gated_prefill_layer: the attention's causal-split scratch
    and the selection's first-pass histogram (one per device and size, reused; calls sharing
    it must not run concurrently)."""
    n = int(load().tg_gated_prefill_workspace_size(B, max_M, Hq, Hkv, d, n_layers))
    if n == 0:
        return None
    key = (torch.device(device), n, "prefill")
    ws = _WS_CACHE.get(key)
    if ws is None:
        ws = torch.zeros(n, dtype=torch.uint8, device=device)
        _WS_CACHE[key] = ws
    return ws


def attention_workspace(B: int, max_M: int, Hq: int, Hkv: int, d: int, device) -> torch.Tensor | None:
    """Zero-filled scratch for tg_gated_attention's causal work split (one per
    device and size, reused; calls sharing it must not run concurrently)."""
    n = int(load().tg_gated_attention_workspace_size(B, max_M, Hq, Hkv, d))
    if n == 0:
        return None
    key = (torch.device(device), n)
    ws = _WS_CACHE.get(key)
    if ws is None:
        ws = torch.zeros(n, dtype=torch.uint8, device=device)
        _WS_CACHE[key] = ws
    return ws


def tg_masked_gated_attention(q, k, v, scores, cu_seqlens, span, kbud, g, c, sm_scale: float | None = None,
                              out=None):
    """Full-length gated attention for the budgets `kbud`: pruned keys masked, rows of
    pruned queries zero.  q [T, Hq, d], k/v [T, Hkv, d] bf16, scores [T] fp32.
    Returns (out [T, Hq, d] bf16, keep [T] uint8)."""
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    dev = q.device
    for t, nm in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, torch.bfloat16, nm)
    _dev(scores, torch.float32, "scores", (T,))
    _dev(g, torch.float32, "g", (Hq,))
    _dev(c, torch.float32, "c", (Hq,))
    to_host = lambda x: x.cpu() if isinstance(x, torch.Tensor) else x  # noqa: E731
    M, cu_kept = tg_kept_count(to_host(cu_seqlens), to_host(span), to_host(kbud))
    max_M = int(np.max(np.diff(cu_kept))) if len(cu_kept) > 1 else 0
    cu = _i32_dev(cu_seqlens, dev, "cu_seqlens")
    sp = _i32_dev(span, dev, "span")
    kb = _i32_dev(kbud, dev, "kbud")
    ck = torch.from_numpy(cu_kept).to(dev)
    B = cu.numel() - 1
    if out is None:
        out = torch.empty((T, Hq, d), dtype=torch.bfloat16, device=dev)
    keep = torch.empty(T, dtype=torch.uint8, device=dev)
    n = int(load().tg_masked_gated_attention_workspace_size(B, T, M, max_M, Hq, Hkv, d))
    key = (torch.device(dev), n, "masked")
    ws = _WS_CACHE.get(key)
    if ws is None:
        ws = torch.zeros(max(n, 256), dtype=torch.uint8, device=dev)
        _WS_CACHE[key] = ws
    scale = float(1.0 / math.sqrt(d) if sm_scale is None else sm_scale)
    _lib.check(load().tg_masked_gated_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), scores.data_ptr(),
                                                cu.data_ptr(), sp.data_ptr(), kb.data_ptr(), ck.data_ptr(), B, T, M,
                                                max_M, Hq, Hkv, d, g.data_ptr(), c.data_ptr(), scale, out.data_ptr(),
                                                keep.data_ptr(), ws.data_ptr(), ws.numel(),
                                                _lib.stream_handle(dev)))
    return out, keep


def tg_gated_attention(q, k, v, cu_kept, max_M: int, pos, rank, gls, g, c, sm_scale: float | None = None,
                       out=None, lse=None, want_lse: bool = False, ws="auto"):
    M, Hq, d = q.shape
    Hkv = k.shape[1]
    dev = q.device
    _dev(q, torch.bfloat16, "q")
    _dev(k, torch.bfloat16, "k", (M, Hkv, d))
    _dev(v, torch.bfloat16, "v", (M, Hkv, d))
    _dev(pos, torch.int32, "pos", (M,))
    _dev(rank, torch.int32, "rank", (M,))
    _dev(gls, torch.float32, "gls", (M,))
    _dev(g, torch.float32, "g", (Hq,))
    _dev(c, torch.float32, "c", (Hq,))
    ck = _i32_dev(cu_kept, dev, "cu_kept")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((M, Hq, d), dtype=torch.bfloat16, device=dev)
    _dev(out, torch.bfloat16, "out", (M, Hq, d))
    if lse is None and want_lse:
        lse = torch.empty((M, Hq), dtype=torch.float32, device=dev)
    if lse is not None:
        _dev(lse, torch.float32, "lse", (M, Hq))
    if isinstance(ws, str):
        ws = attention_workspace(ck.numel() - 1, int(max_M), Hq, Hkv, d, dev)
    _lib.check(load().tg_gated_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), ck.data_ptr(), ck.numel() - 1,
                                         M, int(max_M), Hq, Hkv, d, pos.data_ptr(), rank.data_ptr(),
                                         gls.data_ptr(), g.data_ptr(), c.data_ptr(), float(sm_scale),
                                         out.data_ptr(), _lib.ptr(lse), _lib.ptr(ws),
                                         0 if ws is None else ws.numel(), _lib.stream_handle(dev)))
    return (out, lse) if want_lse or lse is not None else out


def tg_next_gate_span(span, k):
    """Host-side: the next gate's prunable span in this gate's kept order
    ([B, 2] int32 numpy array)."""
    sp = _lib.host_i32(span).reshape(-1)
    kk = _lib.host_i32(k).reshape(-1)
    B = len(kk)
    if len(sp) != 2 * B:
        raise ValueError("span must be [B, 2] for B budgets")
    out = np.zeros(2 * B, dtype=np.int32)
    _lib.check(load().tg_next_gate_span(sp.ctypes.data, kk.ctypes.data, B, out.ctypes.data))
    return out.reshape(B, 2)


def tg_gated_attention_gates(q, k, v, cu_kept, max_M: int, pos, rank, gls, g, c, sm_scale: float | None = None,
                             out=None, lse=None, want_lse: bool = False, ws="auto"):
    """tg_gated_attention with the bias summed over several gates: gls and g are
    sequences of [M] and [Hq] fp32 device tensors, one per gate (1 to 4)."""
    M, Hq, d = q.shape
    Hkv = k.shape[1]
    dev = q.device
    _dev(q, torch.bfloat16, "q")
    _dev(k, torch.bfloat16, "k", (M, Hkv, d))
    _dev(v, torch.bfloat16, "v", (M, Hkv, d))
    _dev(pos, torch.int32, "pos", (M,))
    _dev(rank, torch.int32, "rank", (M,))
    gls, g = list(gls), list(g)
    if len(gls) != len(g):
        raise ValueError("one gls and one g per gate")
    for i, (a, b) in enumerate(zip(gls, g)):
        _dev(a, torch.float32, f"gls[{i}]", (M,))
        _dev(b, torch.float32, f"g[{i}]", (Hq,))
    _dev(c, torch.float32, "c", (Hq,))
    ck = _i32_dev(cu_kept, dev, "cu_kept")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((M, Hq, d), dtype=torch.bfloat16, device=dev)
    _dev(out, torch.bfloat16, "out", (M, Hq, d))
    if lse is None and want_lse:
        lse = torch.empty((M, Hq), dtype=torch.float32, device=dev)
    if lse is not None:
        _dev(lse, torch.float32, "lse", (M, Hq))
    if isinstance(ws, str):
        ws = attention_workspace(ck.numel() - 1, int(max_M), Hq, Hkv, d, dev)
    n = len(gls)
    gls_arr = (C.c_void_p * max(n, 1))(*[t.data_ptr() for t in gls])
    g_arr = (C.c_void_p * max(n, 1))(*[t.data_ptr() for t in g])
    _lib.check(load().tg_gated_attention_gates(q.data_ptr(), k.data_ptr(), v.data_ptr(), ck.data_ptr(),
                                               ck.numel() - 1, M, int(max_M), Hq, Hkv, d, pos.data_ptr(),
                                               rank.data_ptr(), n, gls_arr, g_arr, c.data_ptr(), float(sm_scale),
                                               out.data_ptr(), _lib.ptr(lse), _lib.ptr(ws),
                                               0 if ws is None else ws.numel(), _lib.stream_handle(dev)))
    return (out, lse) if want_lse or lse is not None else out


def tg_gated_attention_backward(q, k, v, out, dout, lse, cu_kept, max_M: int, pos, rank, gls, g, c,
                                sm_scale: float | None = None, want_dscore: bool = True):
    """Gradients of tg_gated_attention for dout: returns a dict with dq, dk, dv
    (bf16, shaped like q, k, v), dgls [M], dscore [M] (d loss / d score of each
    kept row; None unless want_dscore), dg [Hq] and dc [Hq] (fp32).  out and lse
    are the forward's outputs."""
    M, Hq, d = q.shape
    Hkv = k.shape[1]
    dev = q.device
    _dev(q, torch.bfloat16, "q")
    _dev(k, torch.bfloat16, "k", (M, Hkv, d))
    _dev(v, torch.bfloat16, "v", (M, Hkv, d))
    _dev(out, torch.bfloat16, "out", (M, Hq, d))
    _dev(dout, torch.bfloat16, "dout", (M, Hq, d))
    _dev(lse, torch.float32, "lse", (M, Hq))
    _dev(pos, torch.int32, "pos", (M,))
    _dev(rank, torch.int32, "rank", (M,))
    _dev(gls, torch.float32, "gls", (M,))
    _dev(g, torch.float32, "g", (Hq,))
    _dev(c, torch.float32, "c", (Hq,))
    ck = _i32_dev(cu_kept, dev, "cu_kept")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    res = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
           "dgls": torch.empty(M, dtype=torch.float32, device=dev),
           "dscore": torch.empty(M, dtype=torch.float32, device=dev) if want_dscore else None,
           "dg": torch.empty(Hq, dtype=torch.float32, device=dev), "dc": torch.empty(Hq, dtype=torch.float32, device=dev)}
    n = int(load().tg_gated_attention_backward_workspace_size(M, Hq, Hkv, d))
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
    _lib.check(load().tg_gated_attention_backward(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(), ck.data_ptr(),
        ck.numel() - 1, M, int(max_M), Hq, Hkv, d, pos.data_ptr(), rank.data_ptr(), gls.data_ptr(), g.data_ptr(),
        c.data_ptr(), float(sm_scale), res["dq"].data_ptr(), res["dk"].data_ptr(), res["dv"].data_ptr(),
        res["dgls"].data_ptr(), _lib.ptr(res["dscore"]), res["dg"].data_ptr(), res["dc"].data_ptr(), ws.data_ptr(),
        ws.numel(), _lib.stream_handle(dev)))
    return res


def tg_gated_attention_backward_gates(q, k, v, out, dout, lse, cu_kept, max_M: int, pos, rank, gls, g, c,
                                      sm_scale: float | None = None, want_dscore: bool = True):
    """Gradients of tg_gated_attention_gates for dout: gls and g are lists with one
    tensor per gate ([M] and [Hq] fp32).  Returns a dict with dq, dk, dv, dc as for one
    gate, and lists dgls, dscore (or None), dg with one tensor per gate."""
    M, Hq, d = q.shape
    Hkv = k.shape[1]
    dev = q.device
    n = len(gls)
    if n != len(g):
        raise ValueError("one gain tensor per gate")
    _dev(q, torch.bfloat16, "q")
    _dev(k, torch.bfloat16, "k", (M, Hkv, d))
    _dev(v, torch.bfloat16, "v", (M, Hkv, d))
    _dev(out, torch.bfloat16, "out", (M, Hq, d))
    _dev(dout, torch.bfloat16, "dout", (M, Hq, d))
    _dev(lse, torch.float32, "lse", (M, Hq))
    _dev(pos, torch.int32, "pos", (M,))
    _dev(rank, torch.int32, "rank", (M,))
    for i in range(n):
        _dev(gls[i], torch.float32, f"gls[{i}]", (M,))
        _dev(g[i], torch.float32, f"g[{i}]", (Hq,))
    _dev(c, torch.float32, "c", (Hq,))
    ck = _i32_dev(cu_kept, dev, "cu_kept")
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(d)
    res = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
           "dgls": [torch.empty(M, dtype=torch.float32, device=dev) for _ in range(n)],
           "dscore": [torch.empty(M, dtype=torch.float32, device=dev) for _ in range(n)] if want_dscore else None,
           "dg": [torch.empty(Hq, dtype=torch.float32, device=dev) for _ in range(n)],
           "dc": torch.empty(Hq, dtype=torch.float32, device=dev)}
    arr = lambda ts: (C.c_void_p * n)(*[t.data_ptr() for t in ts])  # noqa: E731
    gls_a, g_a, dgls_a, dg_a = arr(gls), arr(g), arr(res["dgls"]), arr(res["dg"])
    dsc_a = arr(res["dscore"]) if want_dscore else None
    nb = int(load().tg_gated_attention_backward_workspace_size(M, Hq, Hkv, d))
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
    _lib.check(load().tg_gated_attention_backward_gates(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(), lse.data_ptr(), ck.data_ptr(),
        ck.numel() - 1, M, int(max_M), Hq, Hkv, d, pos.data_ptr(), rank.data_ptr(), n, gls_a, g_a, c.data_ptr(),
        float(sm_scale), res["dq"].data_ptr(), res["dk"].data_ptr(), res["dv"].data_ptr(), dgls_a, dsc_a, dg_a,
        res["dc"].data_ptr(), ws.data_ptr(), ws.numel(), _lib.stream_handle(dev)))
    return res


def tg_device_status(clear: bool = True, device=None):
    """(status, word): the device status word of the current device; status is
    TG_OK or TG_ERR_TIMEOUT.  Synchronises the current stream."""
    w = C.c_int32(0)
    st = load().tg_device_status(C.byref(w), 1 if clear else 0, _lib.stream_handle(device))
    if st not in (_lib.TG_OK, _lib.TG_ERR_TIMEOUT):
        _lib.check(st)
    return st, int(w.value)


def tg_selftest_bounded_wait(timeout_ns: int, device=None) -> None:
    _lib.check(load().tg_selftest_bounded_wait(int(timeout_ns), _lib.stream_handle(device)))


class PrefillBuffers:
    """Device outputs of one gated prefill, sized on the host from (N, span, K)."""

    def __init__(self, T, D, M, n_layers, Hq, d, device, with_hidden=True, with_lse=False):
        self.scores = torch.zeros(T, dtype=torch.float32, device=device)
        self.keep = torch.empty(T, dtype=torch.uint8, device=device)
        self.hidden_kept = torch.empty((M, D), dtype=torch.bfloat16, device=device) if with_hidden else None
        self.pos = torch.empty(M, dtype=torch.int32, device=device)
        self.rank = torch.empty(M, dtype=torch.int32, device=device)
        self.gls = torch.empty(M, dtype=torch.float32, device=device)
        self.kept_idx = torch.empty(M, dtype=torch.int32, device=device)
        self.out = [torch.empty((M, Hq, d), dtype=torch.bfloat16, device=device) for _ in range(n_layers)]
        self.lse = [torch.empty((M, Hq), dtype=torch.float32, device=device) for _ in range(n_layers)] \
            if with_lse else None


class PrefillCall:
    """A prepared tg_gated_prefill_layer call: the argument struct and the
    host pointer arrays are built once, so that repeated launches (timing
    loops, CUDA-graph capture) only cross the ABI."""

    def __init__(self, hidden, cu_seqlens, span, k, Wg, b1, w2, b2, eps, layers, bufs: PrefillBuffers,
                 Hq, Hkv, d, sm_scale=None, gathers=()):
        """`gathers`: (src [T, ...], dst [M, ...]) pairs of contiguous device tensors that
        the call gathers by the compaction map beside the attention (tg_gather_rows)."""
        dev = hidden.device
        T, D = hidden.shape
        I = Wg.shape[0]
        self.cu = _i32_dev(cu_seqlens, dev, "cu_seqlens")
        self.sp = _i32_dev(span, dev, "span")
        self.kk = _i32_dev(k, dev, "k")
        M, cu_kept = tg_kept_count(cu_seqlens if not isinstance(cu_seqlens, torch.Tensor) else cu_seqlens.cpu(),
                                   span if not isinstance(span, torch.Tensor) else span.cpu(),
                                   k if not isinstance(k, torch.Tensor) else k.cpu())
        self.M = M
        self.max_M = int(np.max(np.diff(cu_kept))) if len(cu_kept) > 1 else 0
        self.ck = torch.from_numpy(cu_kept).to(dev)
        self.keep_alive = [hidden, Wg, b1, w2, bufs, layers]
        nl = len(layers)
        arr = lambda xs: (C.c_void_p * max(nl, 1))(*[x for x in xs])  # noqa: E731
        self._q = arr([L["q"].data_ptr() for L in layers])
        self._k = arr([L["k"].data_ptr() for L in layers])
        self._v = arr([L["v"].data_ptr() for L in layers])
        self._g = arr([L["g"].data_ptr() for L in layers])
        self._c = arr([L["c"].data_ptr() for L in layers])
        self._o = arr([o.data_ptr() for o in bufs.out])
        self._lse = arr([x.data_ptr() for x in bufs.lse]) if bufs.lse is not None else None
        a = _lib.PrefillLayerArgs()
        a.hidden, a.cu_seqlens, a.span, a.k = hidden.data_ptr(), self.cu.data_ptr(), self.sp.data_ptr(), \
            self.kk.data_ptr()
        a.B, a.T, a.D = self.cu.numel() - 1, T, D
        a.Wg, a.b1, a.w2, a.b2, a.I, a.eps = Wg.data_ptr(), b1.data_ptr(), w2.data_ptr(), float(b2), I, float(eps)
        a.cu_kept, a.M_total, a.max_M = self.ck.data_ptr(), M, self.max_M
        a.scores, a.keep = bufs.scores.data_ptr(), bufs.keep.data_ptr()
        a.hidden_kept = _lib.ptr(bufs.hidden_kept)
        a.pos, a.rank, a.gls, a.kept_idx = bufs.pos.data_ptr(), bufs.rank.data_ptr(), bufs.gls.data_ptr(), \
            bufs.kept_idx.data_ptr()
        a.n_layers, a.Hq, a.Hkv, a.d = nl, Hq, Hkv, d
        a.sm_scale = float(1.0 / math.sqrt(d) if sm_scale is None else sm_scale)
        cast = lambda x: C.cast(x, C.c_void_p) if x is not None else None  # noqa: E731
        a.q, a.kk, a.v, a.g, a.c, a.out = (cast(self._q), cast(self._k), cast(self._v), cast(self._g),
                                           cast(self._c), cast(self._o))
        a.lse = cast(self._lse)
        self.ws = prefill_workspace(a.B, self.max_M, Hq, Hkv, d, nl, dev)
        a.attn_ws = _lib.ptr(self.ws)
        a.attn_ws_bytes = 0 if self.ws is None else self.ws.numel()
        gathers = list(gathers)
        ng = len(gathers)
        self._gsrc = (C.c_void_p * max(ng, 1))(*[src.data_ptr() for src, _ in gathers])
        self._gdst = (C.c_void_p * max(ng, 1))(*[dst.data_ptr() for _, dst in gathers])
        self._grow = (C.c_int64 * max(ng, 1))(*[src[0].numel() * src.element_size() for src, _ in gathers])
        self.keep_alive.append(gathers)
        a.n_gather = ng
        a.gather_src = C.cast(self._gsrc, C.POINTER(C.c_void_p))
        a.gather_dst = C.cast(self._gdst, C.POINTER(C.c_void_p))
        a.gather_row_bytes = C.cast(self._grow, C.POINTER(C.c_int64))
        self.args = a
        self.device = dev
        self.bufs = bufs

    def __call__(self, stream: int | None = None):
        st = _lib.stream_handle(self.device) if stream is None else stream
        _lib.check(load().tg_gated_prefill_layer(C.byref(self.args), st))
        return self.bufs


def tg_gated_prefill_layer(hidden, cu_seqlens, span, k, Wg, b1, w2, b2, eps, layers, Hq, Hkv, d,
                           sm_scale=None, with_hidden=True, with_lse=False):
    """One call of the whole gated prefill.  `layers` is a list of dicts with
    q, k, v (bf16 [M, H, d]) and g, c (fp32 [Hq]).  Returns PrefillBuffers."""
    T, D = hidden.shape
    M, _ = tg_kept_count(cu_seqlens if not isinstance(cu_seqlens, torch.Tensor) else cu_seqlens.cpu(),
                         span if not isinstance(span, torch.Tensor) else span.cpu(),
                         k if not isinstance(k, torch.Tensor) else k.cpu())
    bufs = PrefillBuffers(T, D, M, len(layers), Hq, d, hidden.device, with_hidden, with_lse)
    call = PrefillCall(hidden, cu_seqlens, span, k, Wg, b1, w2, b2, eps, layers, bufs, Hq, Hkv, d, sm_scale)
    return call()
