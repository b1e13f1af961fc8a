"""GPU parity of the multi-gate path (several stacked gate modules; TokenGate
AI summary, "Future Directions") against the fp64 oracle, through the C ABI.

Bars as for one gate: maps (positions, ranks, kept indices) bit-exact,
scores within 1e-4 relative, logsigmoids within 1e-5, attention within
max-abs 2e-2 and mean-abs 2e-3.
"""

import dataclasses
import functools

import numpy as np
import pytest
import torch

import oracle
from tests import helpers as H
from workloads import CONFIGS, f32_to_bf16_bits, make_attention_inputs, make_gate_inputs, make_scores

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import learned_token_pruning_rmsnorm_b200 as tg
    tg.load()
    return tg


@functools.lru_cache(maxsize=None)
def gates_case(name, n_gates, rows_step=None):
    """One gate's compaction of the config, plus n_gates - 1 more logsigmoid rows
    (seeded scores on the rows the first gate could prune) and per-gate gains."""
    w = CONFIGS[name]
    cu, span, k = w.cu_seqlens(), w.span_array(), w.budget_array()
    s1 = make_scores(w.T, std=2.0, seed=w.seed)
    keep = oracle.select_topk(s1, cu, span, k)
    comp = oracle.compact(None, s1, keep, cu, span)
    M = int(comp["cu_kept"][-1])
    ai = make_attention_inputs(w, M, layer=0)
    prunable = comp["gls"] != 0
    gls = [comp["gls"].astype(np.float32)]
    gains = [ai["g"]]
    for i in range(1, n_gates):
        s = make_scores(M, std=2.0, seed=w.seed + 11 * i)
        ls = np.minimum(s, 0) - np.log1p(np.exp(-np.abs(s.astype(np.float64))))
        gls.append(np.where(prunable, ls, 0.0).astype(np.float32))
        gains.append(make_attention_inputs(w, 1, layer=i)["g"])
    gls = np.stack(gls)
    gains = np.stack(gains)
    rows = None
    if rows_step:
        rows = np.unique(np.concatenate([np.arange(0, M, rows_step), np.arange(max(0, M - 128), M)])).astype(np.int64)
    out_ref, lse_ref = oracle.gated_attention(ai["q"], ai["k"], ai["v"], comp["cu_kept"], comp["pos"], comp["rank"],
                                              gls, gains, ai["c"], rows=rows)
    return w, comp, ai, gls, gains, rows, out_ref, lse_ref


def _run_gates(tg, comp, ai, gls, gains, want_lse=True):
    cu_kept = comp["cu_kept"]
    max_M = int(np.max(np.diff(cu_kept)))
    res = tg.tg_gated_attention_gates(H.bf16_dev(ai["q"]), H.bf16_dev(ai["k"]), H.bf16_dev(ai["v"]), cu_kept, max_M,
                                      H.i32_dev(comp["pos"]), H.i32_dev(comp["rank"]),
                                      [H.f32_dev(x) for x in gls], [H.f32_dev(x) for x in gains],
                                      H.f32_dev(ai["c"]), want_lse=want_lse)
    torch.cuda.synchronize()
    out, lse = res
    return out.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("name,n_gates,rows_step", [("c0_tiny", 2, None), ("c0_tiny", 3, None),
                                                    ("c0_tiny", 4, None), ("c1_16k", 2, 3),
                                                    ("c2_32k_k2000", 4, 9)])
def test_gates_attention_matches_oracle(tg, name, n_gates, rows_step):
    w, comp, ai, gls, gains, rows, out_ref, lse_ref = gates_case(name, n_gates, rows_step)
    out, lse = _run_gates(tg, comp, ai, gls, gains)
    if rows is not None:
        out, lse = out[rows], lse[rows]
    H.assert_attention_close(out, out_ref, f"{name} x{n_gates} gates")
    assert np.max(np.abs(lse - lse_ref)) <= H.LSE_ABS


@pytest.mark.parametrize("name", ["c0_tiny", "c2_32k_k2000"])
def test_zero_second_gate_is_bitwise_one_gate(tg, name):
    """A second gate whose logsigmoids are all 0 adds exact zeros to every logit."""
    w, comp, ai, gls, gains, _, _, _ = gates_case(name, 2)
    cu_kept = comp["cu_kept"]
    max_M = int(np.max(np.diff(cu_kept)))
    one = tg.tg_gated_attention(H.bf16_dev(ai["q"]), H.bf16_dev(ai["k"]), H.bf16_dev(ai["v"]), cu_kept, max_M,
                                H.i32_dev(comp["pos"]), H.i32_dev(comp["rank"]), H.f32_dev(gls[0]),
                                H.f32_dev(gains[0]), H.f32_dev(ai["c"]))
    two, _ = _run_gates(tg, comp, ai, np.stack([gls[0], np.zeros_like(gls[0])]), gains)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(two, one.float().cpu().numpy())


@pytest.mark.parametrize("d", [64, 128])
def test_gates_odd_group_kernel(tg, d):
    """Odd GQA groups (three query heads per KV head) take the one-head kernel,
    whose softmax sums the gates' biases itself."""
    rng = np.random.default_rng(60 + d)
    seqlens = [300, 1, 129]
    Hq, Hkv = 6, 2
    M = sum(seqlens)
    q = f32_to_bf16_bits((rng.standard_normal((M, Hq, d)) * 0.5).astype(np.float32))
    k = f32_to_bf16_bits((rng.standard_normal((M, Hkv, d)) * 0.5).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((M, Hkv, d)).astype(np.float32))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    rank = np.concatenate([np.arange(1, n + 1) for n in seqlens]).astype(np.int32)
    pos = (rank + np.concatenate([np.sort(rng.integers(0, 500, n)) for n in seqlens])).astype(np.int32)
    gls = -np.abs(rng.standard_normal((3, M)) * 2).astype(np.float32)
    gls[:, :10] = 0
    gains = rng.standard_normal((3, Hq)).astype(np.float32)
    c = (0.5 * rng.random(Hq)).astype(np.float32)
    ai = {"q": q, "k": k, "v": v, "c": c}
    comp = {"cu_kept": cu, "pos": pos, "rank": rank}
    out, lse = _run_gates(tg, comp, ai, gls, gains)
    out_ref, lse_ref = oracle.gated_attention(q, k, v, cu, pos, rank, gls, gains, c)
    H.assert_attention_close(out, out_ref, f"odd group d={d}")
    assert np.max(np.abs(lse - lse_ref)) <= H.LSE_ABS


def test_gates_refused_outside_one_to_four(tg):
    w, comp, ai, gls, gains, _, _, _ = gates_case("c0_tiny", 4)
    five = np.concatenate([gls, gls[:1]])
    with pytest.raises(tg.TokenGateError):
        _run_gates(tg, comp, ai, five, np.concatenate([gains, gains[:1]]))
    with pytest.raises(tg.TokenGateError):
        _run_gates(tg, comp, ai, gls[:0], gains[:0])


@pytest.mark.parametrize("name,k2", [("c0_tiny", 20), ("c1_16k", 500)])
def test_two_gate_pipeline_matches_oracle(tg, name, k2):
    """Gate 1 scores, selects and compacts; gate 2 scores the kept rows' hidden
    states at its own layer (seeded, standing in for the layers between the
    gates), selects inside the kept part of the span, and the composed map
    (original positions, final ranks, both gates' logsigmoids) feeds the
    two-gate attention."""
    w = CONFIGS[name]
    cu, span, k1 = w.cu_seqlens(), w.span_array(), w.budget_array()
    gi1 = make_gate_inputs(w)
    Wg1 = oracle.gate_fold(gi1["gamma"], gi1["W1"])
    # ---- oracle pipeline on the oracle's own scores
    s1_ref = oracle.score(gi1["hidden"], cu, span, Wg1, gi1["b1"], gi1["w2"], gi1["b2"], w.eps)
    s1_ref32 = np.where(np.isnan(s1_ref), 0.0, s1_ref).astype(np.float32)
    keep1_ref = oracle.select_topk(s1_ref32, cu, span, k1)
    first = oracle.compact(None, s1_ref32, keep1_ref, cu, span)
    span2 = oracle.next_gate_span(first, cu, span)
    cu1 = first["cu_kept"]
    k2a = np.full(w.B, k2, np.int32)
    w2 = dataclasses.replace(w, name=name + "_gate2", seqlens=tuple(int(x) for x in np.diff(cu1)),
                             spans=tuple(tuple(int(y) for y in r) for r in span2), budgets=tuple(k2a.tolist()),
                             seed=w.seed + 1)
    gi2 = make_gate_inputs(w2)
    Wg2 = oracle.gate_fold(gi2["gamma"], gi2["W1"])
    s2_ref = oracle.score(gi2["hidden"], cu1, span2, Wg2, gi2["b1"], gi2["w2"], gi2["b2"], w.eps)
    s2_ref32 = np.where(np.isnan(s2_ref), 0.0, s2_ref).astype(np.float32)
    keep2_ref = oracle.select_topk(s2_ref32, cu1, span2, k2a)
    second = oracle.compact(None, s2_ref32, keep2_ref, cu1, span2)
    comp = oracle.compose_gates(first, second)
    M2 = int(comp["cu_kept"][-1])
    ai = make_attention_inputs(w, M2, layer=0)
    gains = np.stack([ai["g"], make_attention_inputs(w, 1, layer=1)["g"]])
    out_ref, lse_ref = oracle.gated_attention(ai["q"], ai["k"], ai["v"], comp["cu_kept"], comp["pos"], comp["rank"],
                                              comp["gls"].astype(np.float32), gains, ai["c"])
    # ---- GPU pipeline through the C ABI
    s1 = tg.tg_score(H.bf16_dev(gi1["hidden"]), cu, span, H.bf16_dev(Wg1), H.f32_dev(gi1["b1"]),
                     H.f32_dev(gi1["w2"]), gi1["b2"], w.eps)
    M1, cu_kept1 = tg.tg_kept_count(cu, span, k1)
    keep1, map1 = tg.tg_select_topk(s1, cu, span, k1, cu_kept=cu_kept1, M_total=M1)
    span2_gpu = tg.tg_next_gate_span(span, k1)
    np.testing.assert_array_equal(span2_gpu, span2)
    s2 = tg.tg_score(H.bf16_dev(gi2["hidden"]), cu_kept1, span2_gpu, H.bf16_dev(Wg2), H.f32_dev(gi2["b1"]),
                     H.f32_dev(gi2["w2"]), gi2["b2"], w.eps)
    M2g, cu_kept2 = tg.tg_kept_count(cu_kept1, span2_gpu, k2a)
    keep2, map2 = tg.tg_select_topk(s2, cu_kept1, span2_gpu, k2a, cu_kept=cu_kept2, M_total=M2g)
    pos = tg.tg_gather_rows(map1["pos"], map2["kept_idx"])
    gls1 = tg.tg_gather_rows(map1["gls"], map2["kept_idx"])
    src = tg.tg_gather_rows(map1["kept_idx"], map2["kept_idx"])
    out, lse = tg.tg_gated_attention_gates(H.bf16_dev(ai["q"]), H.bf16_dev(ai["k"]), H.bf16_dev(ai["v"]),
                                           cu_kept2, int(np.max(np.diff(cu_kept2))), pos, map2["rank"],
                                           [gls1, map2["gls"]], [H.f32_dev(x) for x in gains],
                                           H.f32_dev(ai["c"]), want_lse=True)
    torch.cuda.synchronize()
    # ---- compare
    m1 = H.prunable_mask(w)
    assert H.score_error(s1.cpu().numpy()[m1], s1_ref[m1]) <= H.SCORE_REL
    assert H.check_selection_swaps(keep1.cpu().numpy(), keep1_ref, np.where(m1, s1_ref, 0.0)) == 0
    m2 = H.prunable_mask(w2)
    assert H.score_error(s2.cpu().numpy()[m2], s2_ref[m2]) <= H.SCORE_REL
    assert H.check_selection_swaps(keep2.cpu().numpy(), keep2_ref, np.where(m2, s2_ref, 0.0)) == 0
    assert M2g == M2
    np.testing.assert_array_equal(cu_kept2, comp["cu_kept"])
    np.testing.assert_array_equal(pos.cpu().numpy(), comp["pos"])
    np.testing.assert_array_equal(map2["rank"].cpu().numpy(), comp["rank"])
    np.testing.assert_array_equal(src.cpu().numpy(), comp["src"])
    gls_gpu = np.stack([gls1.cpu().numpy(), map2["gls"].cpu().numpy()]).astype(np.float64)
    assert np.max(np.abs(gls_gpu - comp["gls"])) <= 1e-5
    assert ((gls_gpu == 0) == (comp["gls"] == 0)).all()
    H.assert_attention_close(out.float().cpu().numpy(), out_ref, f"{name} two gates")
    assert np.max(np.abs(lse.cpu().numpy() - lse_ref)) <= H.LSE_ABS


def test_gather_narrow_rows_matches_indexing(tg):
    """4- and 8-byte rows (positions, logsigmoids, 64-bit ids) gathered by a map,
    with entries outside the source skipped."""
    rng = np.random.default_rng(70)
    T, M = 5000, 1777
    idx = rng.integers(0, T, M).astype(np.int32)
    idx[::97] = T + 3  # outside: the row keeps its old content
    a32 = rng.integers(-2**31, 2**31 - 1, T).astype(np.int32)
    a64 = rng.integers(-2**62, 2**62, T).astype(np.int64)
    for a in (a32, a64):
        src = torch.from_numpy(a).cuda()
        dst = torch.full((M,), 7, dtype=src.dtype, device="cuda")
        tg.tg_gather_rows(src, H.i32_dev(idx), dst)
        torch.cuda.synchronize()
        want = np.where(idx < T, a[np.minimum(idx, T - 1)], 7)
        np.testing.assert_array_equal(dst.cpu().numpy(), want)
