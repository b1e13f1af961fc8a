"""CPU pins of the oracle's multi-gate parts (several gate modules stacked at
increasing layers, each selecting from what the lower one kept and each adding
its own bias term to the token-gated attention above it; TokenGate AI summary,
"Future Directions").

Pinned by reductions to the single gate (an absent or zero gate changes
nothing; two gates with equal gains add like one gate with the summed
logsigmoid; gate order is irrelevant), by nested top-K (a second gate that
re-ranks by the same scores keeps exactly the single-gate top-K2), by the
identity of a full second budget, and by the map invariants.
"""

import numpy as np
import pytest

from workloads import f32_to_bf16_bits


def _bf16(x):
    return f32_to_bf16_bits(np.asarray(x, np.float32))


def _attn_inputs(rng, seqlens, Hq, Hkv, d):
    M = sum(seqlens)
    q = _bf16(rng.standard_normal((M, Hq, d)) * 0.7)
    k = _bf16(rng.standard_normal((M, Hkv, d)) * 0.7)
    v = _bf16(rng.standard_normal((M, Hkv, d)))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    rank = np.concatenate([np.arange(1, n + 1) for n in seqlens]).astype(np.int32)
    pos = (rank + np.concatenate([np.sort(rng.integers(0, 40, n)) for n in seqlens])).astype(np.int32)
    g = rng.standard_normal(Hq).astype(np.float32)
    c = (0.5 * rng.random(Hq)).astype(np.float32)
    return q, k, v, cu, pos, rank, g, c


def test_zero_second_gate_equals_one_gate(oracle_mod):
    rng = np.random.default_rng(31)
    q, k, v, cu, pos, rank, g, c = _attn_inputs(rng, [40, 17], 4, 2, 16)
    M = int(cu[-1])
    gls = -np.abs(rng.standard_normal(M) * 3).astype(np.float32)
    out1, lse1 = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, g, c)
    g2 = np.stack([g, rng.standard_normal(4).astype(np.float32)])
    out2, lse2 = oracle_mod.gated_attention(q, k, v, cu, pos, rank, np.stack([gls, np.zeros(M, np.float32)]), g2, c)
    np.testing.assert_array_equal(out2, out1)
    np.testing.assert_array_equal(lse2, lse1)


def test_gates_with_equal_gains_add_like_one_gate(oracle_mod):
    """softplus(g) * a + softplus(g) * b = softplus(g) * (a + b): two gates with the
    same gains act as one gate carrying the summed logsigmoid (sums exact in fp32)."""
    rng = np.random.default_rng(32)
    q, k, v, cu, pos, rank, g, c = _attn_inputs(rng, [33], 4, 1, 8)
    M = int(cu[-1])
    a = -(rng.integers(0, 4096, M) / 1024.0).astype(np.float32)
    b = -(rng.integers(0, 4096, M) / 1024.0).astype(np.float32)
    assert ((a + b).astype(np.float64) == a.astype(np.float64) + b.astype(np.float64)).all()
    out1, _ = oracle_mod.gated_attention(q, k, v, cu, pos, rank, (a + b).astype(np.float32), g, c)
    out2, _ = oracle_mod.gated_attention(q, k, v, cu, pos, rank, np.stack([a, b]), np.stack([g, g]), c)
    np.testing.assert_allclose(out2, out1, rtol=1e-12, atol=1e-13)
    # a gate with a different gain is a different function
    out3, _ = oracle_mod.gated_attention(q, k, v, cu, pos, rank, np.stack([a, b]), np.stack([g, g + 2]), c)
    assert np.abs(out3 - out1).max() > 1e-4


def test_gate_order_is_irrelevant(oracle_mod):
    rng = np.random.default_rng(33)
    q, k, v, cu, pos, rank, g, c = _attn_inputs(rng, [25, 30], 6, 3, 8)
    M = int(cu[-1])
    G = 4
    gls = -np.abs(rng.standard_normal((G, M)) * 2).astype(np.float32)
    gg = rng.standard_normal((G, 6)).astype(np.float32)
    out, lse = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, gg, c)
    perm = [2, 0, 3, 1]
    outp, lsep = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls[perm], gg[perm], c)
    np.testing.assert_allclose(outp, out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lsep, lse, rtol=1e-12, atol=1e-13)


def _two_gates(oracle_mod, rng, seqlens, spans, k1, k2, s2=None):
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    span = np.asarray(spans, np.int32)
    T = int(cu[-1])
    s1 = (2 * rng.standard_normal(T)).astype(np.float32)
    keep1 = oracle_mod.select_topk(s1, cu, span, k1)
    first = oracle_mod.compact(None, s1, keep1, cu, span)
    cu1 = first["cu_kept"]
    span2 = oracle_mod.next_gate_span(first, cu, span)
    M1 = int(cu1[-1])
    if s2 is None:
        s2 = (2 * rng.standard_normal(M1)).astype(np.float32)
    keep2 = oracle_mod.select_topk(s2, cu1, span2, k2)
    second = oracle_mod.compact(None, s2, keep2, cu1, span2)
    return cu, span, s1, first, span2, s2, second, oracle_mod.compose_gates(first, second)


def test_next_span_is_the_kept_part_of_the_span(oracle_mod):
    rng = np.random.default_rng(34)
    seqlens = [60, 1, 45, 30]
    spans = [[10, 50], [0, 0], [0, 45], [5, 5]]
    k1 = [12, 3, 100, 0]
    cu, span, s1, first, span2, _, _, _ = _two_gates(oracle_mod, rng, seqlens, spans, k1, [4, 1, 7, 2])
    for b, (p0, p1) in enumerate(spans):
        kept = min(k1[b], p1 - p0) if k1[b] >= 0 else p1 - p0
        assert tuple(span2[b]) == (p0, p0 + kept)
        # the rows inside the next span are exactly the first gate's kept span tokens
        a0 = first["cu_kept"][b]
        rows = first["pos"][a0 + span2[b, 0]:a0 + span2[b, 1]] - 1
        assert ((rows >= p0) & (rows < p1)).all()


def test_second_gate_keeping_everything_is_identity(oracle_mod):
    rng = np.random.default_rng(35)
    cu, span, s1, first, span2, s2, second, comp = _two_gates(oracle_mod, rng, [80, 50], [[8, 70], [0, 40]],
                                                              [20, 9], [-1, 100])
    np.testing.assert_array_equal(comp["pos"], first["pos"])
    np.testing.assert_array_equal(comp["rank"], first["rank"])
    np.testing.assert_array_equal(comp["src"], first["src"])
    np.testing.assert_array_equal(comp["gls"][0], first["gls"])
    inside = np.zeros(len(first["pos"]), bool)
    for b in range(2):
        a0 = first["cu_kept"][b]
        inside[a0 + span2[b, 0]:a0 + span2[b, 1]] = True
    assert (comp["gls"][1][~inside] == 0).all()
    assert (comp["gls"][1][inside] < 0).all()


@pytest.mark.parametrize("seed", range(3))
def test_nested_topk_equals_single_gate(oracle_mod, seed):
    """A second gate that ranks by the first gate's own scores keeps the single-gate
    top-K2: the composed map equals one gate at budget K2 (ties by index on both)."""
    rng = np.random.default_rng(40 + seed)
    seqlens = [90, 64]
    spans = [[6, 80], [0, 64]]
    k1, k2 = [30, 40], [11, 40]
    cu = np.array([0, 90, 154], np.int32)
    span = np.asarray(spans, np.int32)
    s1 = np.round(2 * rng.standard_normal(154), 1).astype(np.float32)  # plenty of ties
    keep1 = oracle_mod.select_topk(s1, cu, span, k1)
    first = oracle_mod.compact(None, s1, keep1, cu, span)
    span2 = oracle_mod.next_gate_span(first, cu, span)
    s2 = s1[first["src"]]
    keep2 = oracle_mod.select_topk(s2, first["cu_kept"], span2, k2)
    second = oracle_mod.compact(None, s2, keep2, first["cu_kept"], span2)
    comp = oracle_mod.compose_gates(first, second)
    keep_single = oracle_mod.select_topk(s1, cu, span, k2)
    single = oracle_mod.compact(None, s1, keep_single, cu, span)
    np.testing.assert_array_equal(comp["pos"], single["pos"])
    np.testing.assert_array_equal(comp["rank"], single["rank"])
    np.testing.assert_array_equal(comp["src"], single["src"])
    np.testing.assert_array_equal(comp["cu_kept"], single["cu_kept"])
    # both gates' logsigmoids are the same function of the same score here
    np.testing.assert_array_equal(comp["gls"][0], comp["gls"][1])
    assert len(seqlens) == 2


def test_composed_map_invariants(oracle_mod):
    rng = np.random.default_rng(36)
    seqlens = [120, 3, 70]
    spans = [[10, 110], [0, 3], [2, 68]]
    cu, span, s1, first, span2, s2, second, comp = _two_gates(oracle_mod, rng, seqlens, spans, [40, 2, 30],
                                                              [9, 0, 12])
    cu2 = comp["cu_kept"]
    for b in range(3):
        a0, a1 = cu2[b], cu2[b + 1]
        pos, rank = comp["pos"][a0:a1], comp["rank"][a0:a1]
        assert (np.diff(pos) > 0).all()
        np.testing.assert_array_equal(rank, np.arange(1, a1 - a0 + 1))
        assert (pos >= rank).all()
        np.testing.assert_array_equal(comp["src"][a0:a1], cu[b] + pos - 1)
        # every token the first gate could not prune survives the second gate too
        p0, p1 = spans[b]
        fixed = [t for t in range(seqlens[b]) if not (p0 <= t < p1)]
        assert set(fixed) <= set((pos - 1).tolist())
        n_span = int(np.sum((pos - 1 >= p0) & (pos - 1 < p1)))
        assert n_span == min([9, 0, 12][b], span2[b, 1] - span2[b, 0])
    # the tokens the second gate keeps are among those the first kept
    assert set(comp["src"].tolist()) <= set(first["src"].tolist())
    assert comp["gls"].shape == (2, int(cu2[-1]))


def test_library_next_span_helper_matches_oracle(oracle_mod):
    """The library's host helper (closed form) against the oracle's count."""
    from learned_token_pruning_rmsnorm_b200 import build
    build.build()
    import learned_token_pruning_rmsnorm_b200 as tg
    rng = np.random.default_rng(37)
    seqlens = [50, 8, 77, 1]
    spans = [[4, 44], [0, 8], [10, 77], [0, 1]]
    for k1 in ([5, 8, -1, 0], [0, 0, 0, 0], [100, 3, 20, 1]):
        cu, span, s1, first, span2, _, _, _ = _two_gates(oracle_mod, rng, seqlens, spans, k1, [1, 1, 1, 1])
        np.testing.assert_array_equal(tg.tg_next_gate_span(span, k1), span2)
