"""tg_gated_attention_noalloc: the attention entry point for callers that
cannot allocate device memory where they run it (for example a serving
engine that reserves all of HBM at start-up and hands out only fixed
buffers).  Its scratch is a fixed array inside the library, so these tests
check that it gives the same results as tg_gated_attention with a caller
workspace, call after call, and that the array covers every scratch size the
causal split can ask for on this device.

The file is named to run last, so that a run stopping at the first failure
has already run every other test; it also passes alone in a fresh process.
"""

import math

import numpy as np
import pytest
import torch

import oracle
from tests import helpers as H
from workloads import get_config, make_attention_inputs, make_scores

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from learned_token_pruning_rmsnorm_b200 import _lib
    return _lib.load()


def _inputs(name, seed_scores=3):
    w = get_config(name)
    cu, span, k = w.cu_seqlens(), w.span_array(), w.budget_array()
    s = make_scores(w.T, std=2.0, seed=seed_scores)
    keep = oracle.select_topk(s, cu, span, k)
    comp = oracle.compact(None, s, keep, cu, span)
    M = int(comp["cu_kept"][-1])
    ai = make_attention_inputs(w, M)
    t = {
        "q": H.bf16_dev(ai["q"]), "k": H.bf16_dev(ai["k"]), "v": H.bf16_dev(ai["v"]),
        "pos": H.i32_dev(comp["pos"]), "rank": H.i32_dev(comp["rank"]),
        "gls": H.f32_dev(comp["gls"]), "g": H.f32_dev(ai["g"]), "c": H.f32_dev(ai["c"]),
        "cu_kept": H.i32_dev(comp["cu_kept"]),
    }
    max_M = int(np.max(np.diff(comp["cu_kept"])))
    return w, t, M, max_M


def _args(w, t, M, max_M, out, lse):
    return [t["q"].data_ptr(), t["k"].data_ptr(), t["v"].data_ptr(), t["cu_kept"].data_ptr(), w.B, M, max_M,
            w.Hq, w.Hkv, w.d, t["pos"].data_ptr(), t["rank"].data_ptr(), t["gls"].data_ptr(), t["g"].data_ptr(),
            t["c"].data_ptr(), 1.0 / math.sqrt(w.d), out.data_ptr(), lse.data_ptr()]


@pytest.mark.parametrize("name", ["c2_32k_k2000", "c1_16k", "c0_tiny"])
def test_noalloc_matches_workspace_entry_point(lib, name):
    from learned_token_pruning_rmsnorm_b200 import _lib
    w, t, M, max_M = _inputs(name)
    st = torch.cuda.current_stream().cuda_stream
    need = lib.tg_gated_attention_workspace_size(w.B, max_M, w.Hq, w.Hkv, w.d)
    if name != "c0_tiny":
        assert need > 0, "these sizes use the causal split, so the scratch is exercised"
    ws = torch.zeros(max(int(need), 256), dtype=torch.uint8, device="cuda")
    out_ref = torch.empty((M, w.Hq, w.d), dtype=torch.bfloat16, device="cuda")
    lse_ref = torch.empty((M, w.Hq), dtype=torch.float32, device="cuda")
    _lib.check(lib.tg_gated_attention(*_args(w, t, M, max_M, out_ref, lse_ref), ws.data_ptr(), ws.numel(), st))
    torch.cuda.synchronize()
    ref = out_ref.float().cpu().numpy().astype(np.float64)
    ref_lse = lse_ref.cpu().numpy()
    for call in range(2):  # the array keeps the previous call's contents
        out = torch.full((M, w.Hq, w.d), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((M, w.Hq), float("nan"), dtype=torch.float32, device="cuda")
        _lib.check(lib.tg_gated_attention_noalloc(*_args(w, t, M, max_M, out, lse), st))
        torch.cuda.synchronize()
        H.assert_attention_close(out.float().cpu().numpy(), ref, f"{name} no-alloc call {call}")
        assert np.max(np.abs(lse.cpu().numpy() - ref_lse)) <= H.LSE_ABS


def test_noalloc_scratch_bounds_the_split_on_this_device(lib):
    """The causal split is only considered while tiles * (n_qt + 1) < 4 * SMs, where
    tiles = B * Hq / 2 is the number of (sequence, head pair) instances and n_qt the
    number of 128-row query tiles (beyond that every SM's share is at least twice the
    longest unit and no tile is split).  Every such shape is checked here against the
    fixed array, for the SM count of this device; on 148 SMs the largest need is about
    18 MB (head_dim 128, one head pair, n_qt = 144).  Larger needs, possible on devices
    with more SMs, are refused by the entry point with TG_ERR_UNSUPPORTED."""
    import math
    limit = 32 * 1024 * 1024
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    worst = 0
    for d in (64, 128):
        for Hq, Hkv in ((2, 1), (4, 2), (16, 8), (8, 2)):
            for B in (1, 2, 4):
                tiles = B * (Hq // 2)
                for n_qt in range(1, math.ceil(4 * sms / tiles) + 2):
                    need = lib.tg_gated_attention_workspace_size(B, 128 * n_qt, Hq, Hkv, d)
                    worst = max(worst, need)
                    assert need <= limit, (d, Hq, Hkv, B, n_qt, need)
    assert worst > 0
