"""fp64 CPU oracle of the TokenGate gated-prefill path (test infrastructure).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this module.  The library itself never calls it and has no CPU
fallback.  The oracle is a separate C++ translation unit (tg_oracle.cpp)
loaded through ctypes; it shares no code with the CUDA library.

bf16 tensors cross this interface as uint16 bit patterns.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tg_oracle.cpp")
_SO = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile tg_oracle.cpp into oracle/liboracle.so (g++, OpenMP, no fast-math)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            P = C.c_void_p
            i32, i64, f32, f64 = C.c_int, C.c_int64, C.c_float, C.c_double
            lib.oracle_abi_version.restype = i32
            lib.oracle_set_threads.argtypes = [i32]
            lib.oracle_get_threads.restype = i32
            lib.oracle_gate_fold.argtypes = [P, P, i32, i32, P]
            lib.oracle_score.argtypes = [P, P, P, i32, i32, P, P, P, f32, i32, f64, P]
            lib.oracle_score_unfolded.argtypes = [P, P, P, i32, i32, P, P, P, P, f32, i32, f64, P]
            lib.oracle_kept_count.argtypes = [P, P, P, i32, P]
            lib.oracle_kept_count.restype = i64
            lib.oracle_select_topk.argtypes = [P, P, P, P, i32, P]
            lib.oracle_compact.argtypes = [P, P, P, P, P, i32, i32, P, P, P, P, P, P]
            lib.oracle_gated_attention.argtypes = [P, P, P, P, i32, i32, i32, i32, P, P, P, P, P, f64,
                                                   P, i64, P, P, i32, i32]
            lib.oracle_masked_gated_attention.argtypes = [P, P, P, P, P, i32, i32, i32, i32, P, P, P, P,
                                                          f64, P, i64, P]
            lib.oracle_gated_attention_backward.argtypes = [P, P, P, P, i32, i32, i32, i32, P, P, P, P, P, f64,
                                                            P, P, P, P, P, P, P, i32]
            if lib.oracle_abi_version() != 4:
                raise ImportError("oracle/liboracle.so is stale: rebuild it")
            _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(C.c_void_p)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def gate_fold(gamma_bits, W1_bits) -> np.ndarray:
    """Wg [I, D] bf16 bits = bf16(gamma_i * W1[i, j]) (W1 is [D, I])."""
    g, gp = _c(gamma_bits, np.uint16)
    w, wp = _c(W1_bits, np.uint16)
    D, I = w.shape
    out = np.empty((I, D), dtype=np.uint16)
    _load().oracle_gate_fold(gp, wp, D, I, out.ctypes.data_as(C.c_void_p))
    return out


def score(hidden_bits, cu_seqlens, span, Wg_bits, b1, w2, b2, eps) -> np.ndarray:
    """Gate scores [T] in fp64; NaN where a token is not prunable."""
    h, hp = _c(hidden_bits, np.uint16)
    cu, cup = _c(cu_seqlens, np.int32)
    sp, spp = _c(span, np.int32)
    wg, wgp = _c(Wg_bits, np.uint16)
    b1a, b1p = _c(b1, np.float32)
    w2a, w2p = _c(w2, np.float32)
    T, D = h.shape
    I = wg.shape[0]
    out = np.full(T, np.nan, dtype=np.float64)
    _load().oracle_score(hp, cup, spp, len(cu) - 1, D, wgp, b1p, w2p, float(b2), I, float(eps),
                         out.ctypes.data_as(C.c_void_p))
    return out


def score_unfolded(hidden_bits, cu_seqlens, span, gamma_bits, W1_bits, b1, w2, b2, eps) -> np.ndarray:
    h, hp = _c(hidden_bits, np.uint16)
    cu, cup = _c(cu_seqlens, np.int32)
    sp, spp = _c(span, np.int32)
    ga, gap = _c(gamma_bits, np.uint16)
    w1, w1p = _c(W1_bits, np.uint16)
    b1a, b1p = _c(b1, np.float32)
    w2a, w2p = _c(w2, np.float32)
    T, D = h.shape
    I = w1.shape[1]
    out = np.full(T, np.nan, dtype=np.float64)
    _load().oracle_score_unfolded(hp, cup, spp, len(cu) - 1, D, gap, w1p, b1p, w2p, float(b2), I,
                                  float(eps), out.ctypes.data_as(C.c_void_p))
    return out


def kept_count(cu_seqlens, span, k):
    cu, cup = _c(cu_seqlens, np.int32)
    sp, spp = _c(span, np.int32)
    kk, kp = _c(k, np.int32)
    B = len(cu) - 1
    cu_kept = np.empty(B + 1, dtype=np.int32)
    tot = _load().oracle_kept_count(cup, spp, kp, B, cu_kept.ctypes.data_as(C.c_void_p))
    return int(tot), cu_kept


def select_topk(scores_f32, cu_seqlens, span, k) -> np.ndarray:
    s, sp_ = _c(scores_f32, np.float32)
    cu, cup = _c(cu_seqlens, np.int32)
    sp, spp = _c(span, np.int32)
    kk, kp = _c(k, np.int32)
    keep = np.zeros(len(s), dtype=np.uint8)
    _load().oracle_select_topk(sp_, cup, spp, kp, len(cu) - 1, keep.ctypes.data_as(C.c_void_p))
    return keep


def compact(hidden_bits, scores_f32, keep, cu_seqlens, span, with_hidden: bool = True) -> dict:
    cu, cup = _c(cu_seqlens, np.int32)
    sp, spp = _c(span, np.int32)
    s, sp_ = _c(scores_f32, np.float32)
    kp_, kpp = _c(keep, np.uint8)
    B = len(cu) - 1
    M = int(kp_.astype(np.int64).sum())
    if hidden_bits is not None:
        h, hp = _c(hidden_bits, np.uint16)
        D = h.shape[1]
    else:
        h, hp, D = None, None, 0
    hk = np.empty((M, D), dtype=np.uint16) if (with_hidden and h is not None) else None
    pos = np.empty(M, dtype=np.int32)
    rank = np.empty(M, dtype=np.int32)
    gls = np.empty(M, dtype=np.float64)
    src = np.empty(M, dtype=np.int32)
    cu_kept = np.empty(B + 1, dtype=np.int32)
    vp = lambda a: None if a is None else a.ctypes.data_as(C.c_void_p)  # noqa: E731
    _load().oracle_compact(hp, sp_, kpp, cup, spp, B, D, vp(cu_kept), vp(hk), vp(pos), vp(rank), vp(gls),
                           vp(src))
    return {"cu_kept": cu_kept, "hidden_kept": hk, "pos": pos, "rank": rank, "gls": gls, "src": src}


def gated_attention(q_bits, k_bits, v_bits, cu_kept, pos, rank, gls_f32, g, c, sm_scale=None,
                    rows=None, tau_on_qk_only: bool = False, want_lse: bool = True):
    """Token-gated attention.  Returns (out [R, Hq, d] f64, lse [R, Hq] f64 or None).

    One gate: gls_f32 [M], g [Hq].  Several gates: gls_f32 [G, M] and g [G, Hq];
    each gate adds its own bias term to the logits."""
    q, qp = _c(q_bits, np.uint16)
    k, kp = _c(k_bits, np.uint16)
    v, vp_ = _c(v_bits, np.uint16)
    M, Hq, d = q.shape
    Hkv = k.shape[1]
    cu, cup = _c(cu_kept, np.int32)
    po, pop = _c(pos, np.int32)
    ra, rap = _c(rank, np.int32)
    gl, glp = _c(np.asarray(gls_f32, dtype=np.float32).reshape(-1, M), np.float32)
    ga, gap = _c(np.asarray(g, dtype=np.float32).reshape(-1, Hq), np.float32)
    n_gates = gl.shape[0]
    if ga.shape[0] != n_gates:
        raise ValueError("one row of g per gate")
    ca, cap = _c(c, np.float32)
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(d)
    if rows is not None:
        rw, rwp = _c(rows, np.int64)
        R = len(rw)
    else:
        rw, rwp, R = None, None, M
    out = np.empty((R, Hq, d), dtype=np.float64)
    lse = np.empty((R, Hq), dtype=np.float64) if want_lse else None
    _load().oracle_gated_attention(qp, kp, vp_, cup, len(cu) - 1, Hq, Hkv, d, pop, rap, glp, gap, cap,
                                   float(sm_scale), rwp, R, out.ctypes.data_as(C.c_void_p),
                                   None if lse is None else lse.ctypes.data_as(C.c_void_p),
                                   1 if tau_on_qk_only else 0, n_gates)
    return out, lse


def gated_attention_backward(q_bits, k_bits, v_bits, cu_kept, pos, rank, gls_f32, g, c, dout, sm_scale=None,
                             scores=None, prunable=None) -> dict:
    """Gradients of the token-gated attention for the upstream gradient dout
    [M, Hq, d]: dq [M, Hq, d], dk/dv [M, Hkv, d], dgls, dg, dc [Hq], all fp64.

    One gate: gls_f32 [M] and g [Hq] give dgls [M] and dg [Hq].  Several gates
    (AI summary, "Future Directions"): gls_f32 [G, M] and g [G, Hq] give dgls
    [G, M] and dg [G, Hq], gate i's bias term being softplus(g[i, h]) gls[i, j].

    With the kept rows' gate scores (scores [M] or [G, M] fp32, the s_j whose
    logsigmoid is gls_j) and the rows the gates could prune (prunable [M]
    bool), it also returns dscore ([M] or [G, M]): the gradient that reaches
    each gate's score through the bias (AI summary, "Key Contributions" 2: the
    bias on the logits carries the task loss back to the scoring network).
    Since gls_j = logsigmoid(s_j), d gls_j / d s_j = sigmoid(-s_j), taken here
    from the score itself; rows the gate cannot prune carry no bias and get 0."""
    q, qp = _c(q_bits, np.uint16)
    k, kp = _c(k_bits, np.uint16)
    v, vp_ = _c(v_bits, np.uint16)
    M, Hq, d = q.shape
    Hkv = k.shape[1]
    cu, cup = _c(cu_kept, np.int32)
    po, pop = _c(pos, np.int32)
    ra, rap = _c(rank, np.int32)
    one_gate = np.ndim(gls_f32) == 1
    gl, glp = _c(np.asarray(gls_f32, dtype=np.float32).reshape(-1, M), np.float32)
    ga, gap = _c(np.asarray(g, dtype=np.float32).reshape(-1, Hq), np.float32)
    G = gl.shape[0]
    if ga.shape[0] != G:
        raise ValueError("one row of g per gate")
    ca, cap = _c(c, np.float32)
    go, gop = _c(np.asarray(dout, dtype=np.float64).reshape(M, Hq, d), np.float64)
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(d)
    out = {"dq": np.empty((M, Hq, d)), "dk": np.empty((M, Hkv, d)), "dv": np.empty((M, Hkv, d)),
           "dgls": np.empty((G, M)), "dg": np.empty((G, Hq)), "dc": np.empty(Hq)}
    vp = lambda a: a.ctypes.data_as(C.c_void_p)  # noqa: E731
    _load().oracle_gated_attention_backward(qp, kp, vp_, cup, len(cu) - 1, Hq, Hkv, d, pop, rap, glp, gap, cap,
                                            float(sm_scale), gop, vp(out["dq"]), vp(out["dk"]), vp(out["dv"]),
                                            vp(out["dgls"]), vp(out["dg"]), vp(out["dc"]), G)
    if scores is not None:
        s64 = np.asarray(scores, dtype=np.float64).reshape(G, M)
        mask = np.ones(M, dtype=bool) if prunable is None else np.asarray(prunable, dtype=bool).reshape(M)
        # sigmoid(-s) = exp(-log(1 + e^s)), finite for every s
        sig_neg = np.exp(-np.logaddexp(0.0, np.where(mask[None, :], s64, 0.0)))
        out["dscore"] = np.where(mask[None, :], out["dgls"] * sig_neg, 0.0)
    if one_gate:
        out["dgls"], out["dg"] = out["dgls"][0], out["dg"][0]
        if "dscore" in out:
            out["dscore"] = out["dscore"][0]
    return out


def next_gate_span(first: dict, cu_seqlens, span) -> np.ndarray:
    """Prunable span of a second gate, in the first gate's kept order: the kept
    rows of sequence b that came from its span, found by counting the kept rows
    whose source lies before the span start and before its end."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    sp = np.asarray(span, dtype=np.int64).reshape(-1, 2)
    cuk = first["cu_kept"].astype(np.int64)
    src = first["src"].astype(np.int64)
    out = np.zeros_like(sp)
    for b in range(len(cu) - 1):
        rows = src[cuk[b]:cuk[b + 1]] - cu[b]  # positions (0-indexed) of b's kept tokens
        out[b, 0] = int(np.sum(rows < sp[b, 0]))
        out[b, 1] = int(np.sum(rows < sp[b, 1]))
    return out.astype(np.int32)


def compose_gates(first: dict, second: dict, first_gls=None) -> dict:
    """The map of two stacked gates.  `second` is the compaction a second gate
    made over the rows `first` kept (its `src` indexes those rows).  Positions
    stay the original ones, ranks are the second gate's, and every gate's
    logsigmoid follows the surviving rows: gls is [G, M2], the first gate's
    rows (or `first_gls` [G1, M1] for deeper stacks) then the second gate's."""
    s2 = second["src"].astype(np.int64)
    prev = np.asarray(first["gls"] if first_gls is None else first_gls, dtype=np.float64).reshape(-1, len(first["pos"]))
    return {
        "cu_kept": second["cu_kept"],
        "pos": first["pos"][s2].astype(np.int32),
        "rank": second["rank"].astype(np.int32),
        "gls": np.concatenate([prev[:, s2], np.asarray(second["gls"], dtype=np.float64)[None, :]], axis=0),
        "src": first["src"][s2].astype(np.int32),
    }


def masked_gated_attention(q_bits, k_bits, v_bits, cu_seqlens, span, keep, scores_f32, g, c,
                           sm_scale=None, rows=None) -> np.ndarray:
    q, qp = _c(q_bits, np.uint16)
    k, kp = _c(k_bits, np.uint16)
    v, vp_ = _c(v_bits, np.uint16)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    cu, cup = _c(cu_seqlens, np.int32)
    sp, spp = _c(span, np.int32)
    kk, kkp = _c(keep, np.uint8)
    s, s_p = _c(scores_f32, np.float32)
    ga, gap = _c(g, np.float32)
    ca, cap = _c(c, np.float32)
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(d)
    if rows is not None:
        rw, rwp = _c(rows, np.int64)
        R = len(rw)
    else:
        rw, rwp, R = None, None, T
    out = np.empty((R, Hq, d), dtype=np.float64)
    _load().oracle_masked_gated_attention(qp, kp, vp_, cup, spp, len(cu) - 1, Hq, Hkv, d, kkp, s_p, gap, cap,
                                          float(sm_scale), rwp, R, out.ctypes.data_as(C.c_void_p))
    return out
