"""Two copies of libtokengate.so in one process.

The library's only process-wide state (kernel attribute flags, the device
status word, the causal-split memo, the allocation-free scratch) is private to
each copy: only the tg_* entry points are exported, so a second copy loaded
beside the first (another build, another path) binds nothing to it.  The two
copies, called alternately and each after the other's kernels have used TMEM
and shared memory, must give bit-identical scores and attention outputs,
equal to the oracle's within the parity bars."""

import ctypes as C
import math
import shutil

import numpy as np
import pytest
import torch

import oracle
from tests import helpers as H
from workloads import CONFIGS, make_attention_inputs, make_gate_inputs, make_scores

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs(tmp_path_factory):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_token_pruning_rmsnorm_b200 import _lib
    first = _lib.load()
    path = tmp_path_factory.mktemp("copy") / "libtokengate_copy.so"
    shutil.copyfile(_lib.LIB_PATH, path)
    second = C.CDLL(str(path))
    for name, (args, res) in _lib.SIGNATURES.items():
        fn = getattr(second, name)
        fn.argtypes, fn.restype = args, res
    assert first._handle != second._handle
    return first, second


def _scores(lib, w, gi, Wg):
    hid = H.bf16_dev(gi["hidden"])
    b1, w2 = H.f32_dev(gi["b1"]), H.f32_dev(gi["w2"])
    cu, sp = H.i32_dev(w.cu_seqlens()), H.i32_dev(w.span_array().reshape(-1))
    out = torch.full((w.T,), float("nan"), dtype=torch.float32, device="cuda")
    st = lib.tg_score(hid.data_ptr(), cu.data_ptr(), sp.data_ptr(), w.B, w.T, w.D, Wg.data_ptr(), b1.data_ptr(),
                      w2.data_ptr(), float(gi["b2"]), w.I, float(w.eps), out.data_ptr(), None)
    assert st == 0, lib.tg_last_error_string()
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("name", ["c0_tiny", "c2_32k_k2000"])
def test_scores_agree_across_copies(libs, name):
    w = CONFIGS[name]
    gi = make_gate_inputs(w)
    Wg = H.bf16_dev(oracle.gate_fold(gi["gamma"], gi["W1"]))
    runs = [_scores(libs[i % 2], w, gi, Wg) for i in range(4)]
    pm = H.prunable_mask(w)
    for r in runs[1:]:
        np.testing.assert_array_equal(r[pm], runs[0][pm])
    if name == "c0_tiny":
        ref = oracle.score(gi["hidden"], w.cu_seqlens(), w.span_array(), oracle.gate_fold(gi["gamma"], gi["W1"]),
                           gi["b1"], gi["w2"], gi["b2"], w.eps)
        assert H.score_error(runs[0][pm], ref[pm]) <= H.SCORE_REL


@pytest.mark.parametrize("name", ["c0_tiny", "c2_32k_k2000"])
def test_attention_agrees_across_copies(libs, name):
    """c2 at K=2000 takes the causal split, whose arrival counters live in the caller's
    workspace; the copies share that workspace in turn."""
    w = CONFIGS[name]
    cu, sp, kb = w.cu_seqlens(), w.span_array(), w.budget_array()
    s = make_scores(w.T, std=2.0, seed=w.seed)
    keep = oracle.select_topk(s, cu, sp, kb)
    comp = oracle.compact(None, s, keep, cu, sp)
    ck = comp["cu_kept"]
    M, max_M = int(ck[-1]), int(np.max(np.diff(ck)))
    ai = make_attention_inputs(w, M, layer=0)
    q, k, v = H.bf16_dev(ai["q"]), H.bf16_dev(ai["k"]), H.bf16_dev(ai["v"])
    pos, rank, gls = H.i32_dev(comp["pos"]), H.i32_dev(comp["rank"]), H.f32_dev(comp["gls"])
    g, c, ck_d = H.f32_dev(ai["g"]), H.f32_dev(ai["c"]), H.i32_dev(ck)
    nws = int(libs[0].tg_gated_attention_workspace_size(w.B, max_M, w.Hq, w.Hkv, w.d))
    ws = torch.zeros(max(nws, 256), dtype=torch.uint8, device="cuda")
    outs = []
    for i in range(4):
        lib = libs[i % 2]
        out = torch.empty((M, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
        st = lib.tg_gated_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), ck_d.data_ptr(), w.B, M, max_M, w.Hq,
                                    w.Hkv, w.d, pos.data_ptr(), rank.data_ptr(), gls.data_ptr(), g.data_ptr(),
                                    c.data_ptr(), 1.0 / math.sqrt(w.d), out.data_ptr(), None, ws.data_ptr(),
                                    ws.numel(), None)
        assert st == 0, lib.tg_last_error_string()
        torch.cuda.synchronize()
        outs.append(H.bf16_host_bits(out))
    for o in outs[1:]:
        np.testing.assert_array_equal(o, outs[0])
    rows = np.unique(np.concatenate([np.arange(0, M, 97), [M - 1]])).astype(np.int64)
    ref, _ = oracle.gated_attention(ai["q"], ai["k"], ai["v"], ck, comp["pos"], comp["rank"],
                                    comp["gls"].astype(np.float32), ai["g"], ai["c"], rows=rows, want_lse=False)
    from workloads import bf16_bits_to_f32
    H.assert_attention_close(bf16_bits_to_f32(outs[0][rows]), ref, name)
