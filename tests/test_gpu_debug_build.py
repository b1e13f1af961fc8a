"""The index-checking variant of the library (TG_DEBUG, libtokengate_debug.so).

Its kernels check every row index they derive from cu_kept / cu_seqlens against the
array sizes given on the host, skip an access that would fall outside, and record the
violation in the device status word, which tg_device_status reports as
TG_ERR_INVALID_ARG.  Valid calls give the same results as the release library.  The
inconsistent inputs below are only ever given to this variant: the release kernels
trust the documented contract and would read and write outside the arrays."""

import ctypes as C
import math

import numpy as np
import pytest
import torch

import oracle
from tests import helpers as H
from workloads import CONFIGS, make_attention_inputs, make_gate_inputs, make_scores

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_token_pruning_rmsnorm_b200 import _lib, build
    path = build.build(debug=True)
    lib = C.CDLL(path)
    for name, (args, res) in _lib.SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes, fn.restype = args, res
    assert lib.tg_device_status(None, 1, None) == 0
    return lib


def _attention_case():
    w = CONFIGS["c0_tiny"]
    cu, span, kb = w.cu_seqlens(), w.span_array(), w.budget_array()
    s = make_scores(w.T, std=2.0, seed=w.seed)
    comp = oracle.compact(None, s, oracle.select_topk(s, cu, span, kb), cu, span)
    M = int(comp["cu_kept"][-1])
    ai = make_attention_inputs(w, M, layer=0)
    return w, comp, ai, M


def _attend(lib, w, comp, ai, M, cu_kept, max_M):
    t = [H.bf16_dev(ai["q"]), H.bf16_dev(ai["k"]), H.bf16_dev(ai["v"]), H.i32_dev(cu_kept),
         H.i32_dev(comp["pos"]), H.i32_dev(comp["rank"]), H.f32_dev(comp["gls"]), H.f32_dev(ai["g"]),
         H.f32_dev(ai["c"])]
    out = torch.zeros((M, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    # the persistent kernel is the one whose debug build checks cu_kept against M_total
    with H.attention_kernel("persistent"):
        n = int(lib.tg_gated_attention_workspace_size(w.B, max_M, w.Hq, w.Hkv, w.d))
        ws = torch.zeros(max(n, 256), dtype=torch.uint8, device="cuda")
        st = lib.tg_gated_attention(*[x.data_ptr() for x in t[:4]], w.B, M, max_M, w.Hq, w.Hkv, w.d,
                                    *[x.data_ptr() for x in t[4:]], 1.0 / math.sqrt(w.d), out.data_ptr(), None,
                                    ws.data_ptr(), ws.numel(), None)
    assert st == 0, lib.tg_last_error_string()
    torch.cuda.synchronize()
    return out


def test_debug_build_matches_on_valid_inputs(dbg):
    w, comp, ai, M = _attention_case()
    out = _attend(dbg, w, comp, ai, M, comp["cu_kept"], M)
    word = C.c_int32(0)
    assert dbg.tg_device_status(C.byref(word), 1, None) == 0 and word.value == 0
    ref, _ = oracle.gated_attention(ai["q"], ai["k"], ai["v"], comp["cu_kept"], comp["pos"], comp["rank"],
                                    comp["gls"].astype(np.float32), ai["g"], ai["c"])
    H.assert_attention_close(out.float().cpu().numpy(), ref, "debug build")


def test_debug_build_reports_cu_kept_beyond_M_total(dbg):
    """cu_kept claims 64 more kept rows than the M_total the host passed: the attention
    skips that sequence, writes nothing, and the status word says why."""
    w, comp, ai, M = _attention_case()
    bad = np.array([0, M + 64], dtype=np.int32)
    out = _attend(dbg, w, comp, ai, M, bad, M + 64)
    assert bool((out == 0).all()), "no row may be written"
    word = C.c_int32(0)
    assert dbg.tg_device_status(C.byref(word), 1, None) == 1  # TG_ERR_INVALID_ARG
    assert word.value & (1 << 17) and word.value & (1 << 4)
    assert dbg.tg_device_status(None, 1, None) == 0  # cleared


def test_debug_build_reports_cu_seqlens_beyond_T(dbg):
    """cu_seqlens claims 512 more tokens than the T the host passed (the span reaching past
    T): the score kernel skips the rows past T and records it."""
    w = CONFIGS["c0_tiny"]
    gi = make_gate_inputs(w)
    T = w.T
    hid = H.bf16_dev(gi["hidden"])
    Wg = H.bf16_dev(oracle.gate_fold(gi["gamma"], gi["W1"]))
    b1, w2 = H.f32_dev(gi["b1"]), H.f32_dev(gi["w2"])
    cu = H.i32_dev(np.array([0, T + 512], np.int32))
    sp = H.i32_dev(np.array([64, T + 300], np.int32))
    scores = torch.full((T + 1024,), -7.0, dtype=torch.float32, device="cuda")
    st = dbg.tg_score(hid.data_ptr(), cu.data_ptr(), sp.data_ptr(), 1, T, w.D, Wg.data_ptr(), b1.data_ptr(),
                      w2.data_ptr(), float(gi["b2"]), w.I, float(w.eps), scores.data_ptr(), None)
    assert st == 0
    torch.cuda.synchronize()
    s = scores.cpu().numpy()
    assert (s[T:] == -7.0).all(), "nothing past T may be written"
    ref = oracle.score(gi["hidden"], w.cu_seqlens(), np.array([[64, T]], np.int32),
                       oracle.gate_fold(gi["gamma"], gi["W1"]), gi["b1"], gi["w2"], gi["b2"], w.eps)
    assert H.score_error(s[64:T], ref[64:T]) <= H.SCORE_REL  # rows inside T are still scored
    word = C.c_int32(0)
    assert dbg.tg_device_status(C.byref(word), 1, None) == 1  # TG_ERR_INVALID_ARG
    assert word.value & (1 << 17) and word.value & (1 << 5)
