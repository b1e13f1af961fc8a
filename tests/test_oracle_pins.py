"""Pins of the fp64 oracle against things other than itself.

Each test fixes one part of the oracle with a closed form, a brute force, an
invariant or an independent library routine (PyTorch CPU in fp64), chosen so
that a plausible slip in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a sum instead of a mean) fails at least one of them.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from workloads import bf16_bits_to_f32, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def _t_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


# ---------------------------------------------------------------- gate fold

def test_gate_fold_matches_torch_rounding(oracle_mod):
    rng = np.random.default_rng(1)
    D, I = 48, 24
    gamma = _bf16(1 + 0.3 * rng.standard_normal(D))
    W1 = _bf16(rng.standard_normal((D, I)))
    Wg = oracle_mod.gate_fold(gamma, W1)
    ref = (_t_bf16(gamma).float()[:, None] * _t_bf16(W1).float()).to(torch.bfloat16).T.contiguous()
    assert Wg.shape == (I, D)
    np.testing.assert_array_equal(Wg, ref.view(torch.int16).numpy().view(np.uint16))


def test_gate_fold_ties_round_to_even(oracle_mod):
    # products of two bf16 mantissas that land exactly half-way between two
    # bf16 values; both neighbours are checked against round-half-to-even
    ties = []
    for ma in range(128, 256):
        for mb in range(128, 256):
            p = np.float32(ma / 128.0) * np.float32(mb / 128.0)
            u = int(np.array(p, dtype=np.float32).view(np.uint32))
            if (u & 0xFFFF) == 0x8000:
                ties.append((ma / 128.0, mb / 128.0, u))
    assert len(ties) > 10
    gamma = _bf16([t[0] for t in ties])
    W1 = _bf16(np.diag([t[1] for t in ties]))  # [D, I] diagonal
    Wg = oracle_mod.gate_fold(gamma, W1)
    for j, (_, _, u) in enumerate(ties):
        hi = u >> 16
        want = hi + (hi & 1)          # ties to even
        assert int(Wg[j, j]) == want


# ---------------------------------------------------------------- RMSNorm / score

def _identity_gate(D):
    gamma = _bf16(np.ones(D))
    W1 = _bf16(np.eye(D))
    return gamma, W1


@pytest.mark.parametrize("a", [0.5, 3.0, -2.0, 1e-3])
def test_rmsnorm_constant_row_closed_form(oracle_mod, a):
    D = 16
    gamma, W1 = _identity_gate(D)
    Wg = oracle_mod.gate_fold(gamma, W1)
    a_b = float(bf16_bits_to_f32(_bf16([a]))[0])
    hidden = _bf16(np.full((1, D), a_b))
    eps = 1e-6
    for kch in (0, 7, 15):
        w2 = np.zeros(D, np.float32)
        w2[kch] = 1.0
        s = oracle_mod.score(hidden, [0, 1], [[0, 1]], Wg, np.zeros(D, np.float32), w2, 0.0, eps)[0]
        z = a_b / math.sqrt(a_b * a_b + eps)          # every channel equals a
        assert s == pytest.approx(z / (1 + math.exp(-z)), rel=1e-13, abs=1e-15)


@pytest.mark.parametrize("a", [2.0, -5.0])
def test_rmsnorm_one_hot_row_uses_mean(oracle_mod, a):
    D = 32
    gamma, W1 = _identity_gate(D)
    Wg = oracle_mod.gate_fold(gamma, W1)
    x = np.zeros((1, D))
    x[0, 5] = a
    eps = 1e-6
    w2 = np.zeros(D, np.float32)
    w2[5] = 1.0
    s = oracle_mod.score(_bf16(x), [0, 1], [[0, 1]], Wg, np.zeros(D, np.float32), w2, 0.0, eps)[0]
    z = a / math.sqrt(a * a / D + eps)            # mean over D channels, not the sum
    assert s == pytest.approx(z / (1 + math.exp(-z)), rel=1e-13)


def test_zero_row_gives_bias_path(oracle_mod):
    D, I = 16, 8
    rng = np.random.default_rng(3)
    Wg = oracle_mod.gate_fold(_bf16(np.ones(D)), _bf16(rng.standard_normal((D, I))))
    b1 = rng.standard_normal(I).astype(np.float32)
    w2 = rng.standard_normal(I).astype(np.float32)
    s = oracle_mod.score(_bf16(np.zeros((1, D))), [0, 1], [[0, 1]], Wg, b1, w2, 0.25, 1e-6)[0]
    b1d, w2d = b1.astype(np.float64), w2.astype(np.float64)
    want = 0.25 + float(np.sum(w2d * b1d / (1 + np.exp(-b1d))))
    assert s == pytest.approx(want, rel=1e-13)


def test_score_matches_torch_composition(oracle_mod):
    rng = np.random.default_rng(4)
    T, D, I = 40, 64, 24
    hidden = _bf16(rng.standard_normal((T, D)) * np.where(np.arange(D) == 3, 8.0, 1.0))
    gamma = _bf16(1 + 0.1 * rng.standard_normal(D))
    W1 = _bf16(rng.standard_normal((D, I)) / math.sqrt(D))
    b1 = (0.1 * rng.standard_normal(I)).astype(np.float32)
    w2 = (rng.standard_normal(I) / math.sqrt(I)).astype(np.float32)
    b2 = float(np.float32(0.05))   # b2 crosses the interface as fp32
    cu = np.array([0, 17, 40], np.int32)
    span = np.array([[2, 15], [0, 23]], np.int32)
    eps = 1e-6
    s = oracle_mod.score(hidden, cu, span, oracle_mod.gate_fold(gamma, W1), b1, w2, b2, eps)

    x = _t_bf16(hidden).double()
    Wg_t = (_t_bf16(gamma).float()[:, None] * _t_bf16(W1).float()).to(torch.bfloat16).double()  # [D, I]
    r = torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + eps)
    z = F.linear(x * r, Wg_t.T, torch.from_numpy(b1).double())
    ref = (F.linear(F.silu(z), torch.from_numpy(w2).double()[None, :]) + b2)[:, 0].numpy()
    prunable = np.zeros(T, bool)
    prunable[2:15] = True
    prunable[17:40] = True
    np.testing.assert_allclose(s[prunable], ref[prunable], rtol=1e-12, atol=1e-12)
    assert np.isnan(s[~prunable]).all()

    # the unfolded mode is RMSNorm(gamma) then Linear, exactly
    su = oracle_mod.score_unfolded(hidden, cu, span, gamma, W1, b1, w2, b2, eps)
    u = x * r * _t_bf16(gamma).double()
    zu = F.linear(u, _t_bf16(W1).double().T, torch.from_numpy(b1).double())
    refu = (F.linear(F.silu(zu), torch.from_numpy(w2).double()[None, :]) + b2)[:, 0].numpy()
    np.testing.assert_allclose(su[prunable], refu[prunable], rtol=1e-12, atol=1e-12)
    # the bf16 fold of gamma into W1 moves scores only at bf16 resolution
    assert np.max(np.abs(su[prunable] - s[prunable])) < 2e-2


# ---------------------------------------------------------------- top-K

def _dominates(s, i, j):
    """True when token i must be kept before token j (score desc, index asc;
    NaN below everything; -0 == +0)."""
    si, sj = s[i], s[j]
    if np.isnan(si) or np.isnan(sj):
        if np.isnan(si) and np.isnan(sj):
            return i < j
        return not np.isnan(si)
    if si != sj:
        return si > sj
    return i < j


def _brute_force_topk(s, K):
    n = len(s)
    good = []
    for sub in itertools.combinations(range(n), K):
        inside = set(sub)
        if all(_dominates(s, i, j) for i in inside for j in range(n) if j not in inside):
            good.append(inside)
    assert len(good) == 1, "the order (score desc, index asc) must single out one set"
    return good[0]


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_small(oracle_mod, seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 11))
    pool = np.array([0.0, -0.0, 1.0, 1.0, -1.0, 2.5, np.inf, -np.inf, np.nan, 0.5], np.float32)
    s = rng.choice(pool, size=n).astype(np.float32) if seed % 2 else \
        rng.integers(-2, 3, size=n).astype(np.float32)
    for K in range(0, n + 1):
        keep = oracle_mod.select_topk(s, [0, n], [[0, n]], [K])
        kept = set(np.nonzero(keep)[0].tolist())
        assert kept == _brute_force_topk(s, K)


def test_topk_partition_and_budgets(oracle_mod):
    # two sequences; non-prunable tokens are always kept; K<0 and K>|P| keep all
    rng = np.random.default_rng(7)
    cu = np.array([0, 20, 50], np.int32)
    span = np.array([[3, 17], [0, 30]], np.int32)
    s = rng.standard_normal(50).astype(np.float32)
    for k in ([0, 0], [5, 11], [-1, 100], [14, 30]):
        keep = oracle_mod.select_topk(s, cu, span, k)
        assert keep[0:3].all() and keep[17:20].all()
        for b, (p0, p1) in enumerate(span):
            base = cu[b]
            P = p1 - p0
            want = P if (k[b] < 0 or k[b] > P) else k[b]
            got = int(keep[base + p0:base + p1].sum())
            assert got == want
            kept = [t for t in range(base + p0, base + p1) if keep[t]]
            dropped = [t for t in range(base + p0, base + p1) if not keep[t]]
            for i in kept:
                for j in dropped:
                    assert _dominates(s, i, j)


def test_topk_equals_full_sort_medium(oracle_mod):
    rng = np.random.default_rng(8)
    n = 3000
    s = np.round(rng.standard_normal(n) * 4).astype(np.float32)  # many ties
    K = 777
    keep = oracle_mod.select_topk(s, [0, n], [[0, n]], [K])
    order = sorted(range(n), key=lambda t: (-s[t], t))
    assert set(np.nonzero(keep)[0].tolist()) == set(order[:K])


# ---------------------------------------------------------------- kept count

def test_kept_count_formula(oracle_mod):
    cu = np.array([0, 10, 10, 25, 40], np.int32)
    span = np.array([[2, 8], [0, 0], [0, 15], [5, 5]], np.int32)
    k = np.array([3, 4, -1, 0], np.int32)
    tot, cu_kept = oracle_mod.kept_count(cu, span, k)
    # (10-6)+3, (0-0)+0, (15-15)+15, (15-0)+0
    assert cu_kept.tolist() == [0, 7, 7, 22, 37]
    assert tot == 37


def test_kept_count_readme_demo_golden(oracle_mod):
    """The README demo keeps 144 of 32,191 prompt tokens at K=100: every token
    outside the `{state}` document is kept, plus K document tokens."""
    with open(os.path.join(GOLDEN, "readme_niah_kept_tokens.json")) as f:
        g = json.load(f)
    n, k, kept = g["prompt_tokens"], g["K"], g["kept_tokens"]
    n_np = kept - k
    span = [[n_np // 2, n - (n_np - n_np // 2)]]   # any placement of the document span
    tot, _ = oracle_mod.kept_count([0, n], span, [k])
    assert tot == kept
    assert round(100.0 * kept / n, 1) == g["kept_percent"]
    tot_all, _ = oracle_mod.kept_count([0, n], span, [-1])
    assert tot_all == n


# ---------------------------------------------------------------- compaction

def test_compaction_invariants(oracle_mod):
    rng = np.random.default_rng(9)
    cu = np.array([0, 64, 64, 160], np.int32)
    span = np.array([[8, 50], [0, 0], [0, 90]], np.int32)
    D = 8
    hidden = rng.integers(0, 65536, size=(160, D)).astype(np.uint16)
    s = rng.standard_normal(160).astype(np.float32) * 3
    k = np.array([10, 5, 40], np.int32)
    keep = oracle_mod.select_topk(s, cu, span, k)
    res = oracle_mod.compact(hidden, s, keep, cu, span)
    tot, cu_kept = oracle_mod.kept_count(cu, span, k)
    np.testing.assert_array_equal(res["cu_kept"], cu_kept)
    assert len(res["pos"]) == tot
    for b in range(3):
        a0, a1 = cu_kept[b], cu_kept[b + 1]
        pos, rank = res["pos"][a0:a1], res["rank"][a0:a1]
        assert (np.diff(pos) > 0).all()
        np.testing.assert_array_equal(rank, np.arange(1, a1 - a0 + 1))
        assert (pos >= rank).all()
        src = res["src"][a0:a1]
        np.testing.assert_array_equal(src, cu[b] + pos - 1)
        np.testing.assert_array_equal(res["hidden_kept"][a0:a1], hidden[src])
        p0, p1 = span[b]
        prunable = (pos - 1 >= p0) & (pos - 1 < p1)
        gls_ref = F.logsigmoid(torch.from_numpy(s[src].astype(np.float64))).numpy()
        np.testing.assert_allclose(res["gls"][a0:a1][prunable], gls_ref[prunable], rtol=1e-14, atol=1e-300)
        assert (res["gls"][a0:a1][~prunable] == 0).all()
        # every non-prunable token of the sequence is present
        np_tokens = [t for t in range(cu[b + 1] - cu[b]) if not (p0 <= t < p1)]
        assert set(np_tokens) <= set((pos - 1).tolist())


def test_compaction_full_budget_is_identity(oracle_mod):
    rng = np.random.default_rng(10)
    n, D = 70, 4
    hidden = rng.integers(0, 65536, size=(n, D)).astype(np.uint16)
    s = rng.standard_normal(n).astype(np.float32)
    span = [[5, 60]]
    keep = oracle_mod.select_topk(s, [0, n], span, [55])
    assert keep.all()
    res = oracle_mod.compact(hidden, s, keep, [0, n], span)
    np.testing.assert_array_equal(res["pos"], res["rank"])
    np.testing.assert_array_equal(res["hidden_kept"], hidden)


def test_logsigmoid_extremes(oracle_mod):
    s = np.array([-100.0, -30.0, 0.0, 30.0, 100.0, -0.0], np.float32)
    keep = np.ones(6, np.uint8)
    res = oracle_mod.compact(None, s, keep, [0, 6], [[0, 6]])
    want = np.array([-100.0, -30.0 - math.log1p(math.exp(-30.0)), -math.log(2.0),
                     -math.log1p(math.exp(-30.0)), -math.log1p(math.exp(-100.0)), -math.log(2.0)])
    np.testing.assert_allclose(res["gls"], want, rtol=1e-15, atol=0)


# ---------------------------------------------------------------- attention

def _attn_case(rng, seqlens, Hq, Hkv, d, std=0.5):
    M = sum(seqlens)
    q = _bf16(rng.standard_normal((M, Hq, d)) * std)
    k = _bf16(rng.standard_normal((M, Hkv, d)) * std)
    v = _bf16(rng.standard_normal((M, Hkv, d)))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    return q, k, v, cu


def _sdpa_causal_gqa(q, k, v, cu, scale=None):
    """PyTorch fp64 scaled_dot_product_attention(is_causal=True), per sequence,
    with KV heads repeated for GQA."""
    qt, kt, vt = (_t_bf16(a).double() for a in (q, k, v))
    Hq, Hkv = qt.shape[1], kt.shape[1]
    outs = []
    for b in range(len(cu) - 1):
        a0, a1 = int(cu[b]), int(cu[b + 1])
        qb = qt[a0:a1].transpose(0, 1)
        kb = kt[a0:a1].transpose(0, 1).repeat_interleave(Hq // Hkv, dim=0)
        vb = vt[a0:a1].transpose(0, 1).repeat_interleave(Hq // Hkv, dim=0)
        ob = F.scaled_dot_product_attention(qb, kb, vb, is_causal=True, scale=scale)
        outs.append(ob.transpose(0, 1))
    return torch.cat(outs).numpy()


def test_attention_reduces_to_causal_gqa(oracle_mod):
    """bias 0, tau 1 and a full budget give ordinary causal GQA attention."""
    rng = np.random.default_rng(11)
    seqlens = [37, 1, 20]
    Hq, Hkv, d = 4, 2, 16
    q, k, v, cu = _attn_case(rng, seqlens, Hq, Hkv, d)
    M = cu[-1]
    pos = np.concatenate([np.arange(1, n + 1) for n in seqlens]).astype(np.int32)
    rank = pos.copy()
    gls = np.zeros(M, np.float32)
    g = rng.standard_normal(Hq).astype(np.float32)
    c = rng.random(Hq).astype(np.float32)   # tau is 1 anyway since pos == rank
    out, lse = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, g, c)
    ref = _sdpa_causal_gqa(q, k, v, cu)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_attention_temperature_and_bias_against_sdpa_rows(oracle_mod):
    """Each query row equals SDPA with scale sm_scale/tau and additive mask
    bias/tau: the temperature divides the whole logit."""
    rng = np.random.default_rng(12)
    seqlens = [30]
    Hq, Hkv, d = 4, 1, 8
    q, k, v, cu = _attn_case(rng, seqlens, Hq, Hkv, d, std=1.0)
    M = 30
    pos = np.sort(rng.choice(np.arange(1, 200), size=M, replace=False)).astype(np.int32)
    rank = np.arange(1, M + 1, dtype=np.int32)
    gls = np.minimum(0, rng.standard_normal(M) * 3).astype(np.float32)
    gls[:4] = 0.0
    g = rng.standard_normal(Hq).astype(np.float32)
    c = (0.5 * rng.random(Hq)).astype(np.float32)
    out, lse = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, g, c)
    qt, kt, vt = (_t_bf16(a).double() for a in (q, k, v))
    sm = 1 / math.sqrt(d)
    for i in range(M):
        for h in range(Hq):
            tau = 1 + float(c[h]) * math.log(pos[i] / rank[i])
            gain = float(F.softplus(torch.tensor(float(g[h]), dtype=torch.float64)))
            bias = torch.from_numpy(gls[: i + 1].astype(np.float64)) * gain / tau
            o = F.scaled_dot_product_attention(qt[i:i + 1, h][None], kt[: i + 1, 0][None], vt[: i + 1, 0][None],
                                               attn_mask=bias[None, None, :], scale=sm / tau)
            np.testing.assert_allclose(out[i, h], o[0, 0].numpy(), rtol=1e-11, atol=1e-12)
            logits = (qt[i, h] @ kt[: i + 1, 0].T * sm + torch.from_numpy(gls[: i + 1].astype(np.float64)) * gain) / tau
            assert lse[i, h] == pytest.approx(float(torch.logsumexp(logits, 0)), rel=1e-12)
    # the other reading (tau on q.k only) is a different function
    out2, _ = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, g, c, tau_on_qk_only=True)
    assert np.max(np.abs(out2 - out)) > 1e-6


def test_attention_bias_only_closed_form(oracle_mod):
    """With q = 0 the weights are softmax(b_j / tau) over the causal keys."""
    rng = np.random.default_rng(13)
    M, d = 12, 8
    q = _bf16(np.zeros((M, 1, d)))
    k = _bf16(rng.standard_normal((M, 1, d)))
    v = _bf16(rng.standard_normal((M, 1, d)))
    pos = (np.arange(M) * 3 + 1).astype(np.int32)
    rank = np.arange(1, M + 1, dtype=np.int32)
    gls = -np.abs(rng.standard_normal(M)).astype(np.float32)
    g = np.array([0.7], np.float32)
    c = np.array([0.3], np.float32)
    out, _ = oracle_mod.gated_attention(q, k, v, [0, M], pos, rank, gls, g, c)
    vv = bf16_bits_to_f32(v).astype(np.float64)[:, 0]
    gain = math.log1p(math.exp(float(g[0])))    # g and c cross the interface as fp32
    for i in range(M):
        tau = 1 + float(c[0]) * math.log(pos[i] / rank[i])
        w = np.exp(gain * gls[: i + 1].astype(np.float64) / tau)
        w /= w.sum()
        np.testing.assert_allclose(out[i, 0], w @ vv[: i + 1], rtol=1e-12, atol=1e-13)


def test_attention_tau_is_one_where_pos_equals_rank(oracle_mod):
    rng = np.random.default_rng(14)
    M, Hq, Hkv, d = 40, 2, 1, 16
    q, k, v, cu = _attn_case(rng, [M], Hq, Hkv, d)
    pos = np.arange(1, M + 1, dtype=np.int32)
    pos[20:] += 7          # a pruned gap: rows from 20 on have pos > rank
    rank = np.arange(1, M + 1, dtype=np.int32)
    gls = -np.abs(rng.standard_normal(M)).astype(np.float32)
    g = rng.standard_normal(Hq).astype(np.float32)
    c = (0.5 + rng.random(Hq)).astype(np.float32)
    out, _ = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, g, c)
    out0, _ = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, g, np.zeros_like(c))
    np.testing.assert_array_equal(out[:20], out0[:20])
    assert np.max(np.abs(out[20:] - out0[20:])) > 1e-6


def test_attention_uniform_values_and_first_row(oracle_mod):
    rng = np.random.default_rng(15)
    M, Hq, Hkv, d = 25, 4, 2, 8
    q, k, _, cu = _attn_case(rng, [M], Hq, Hkv, d, std=2.0)
    row = _bf16(rng.standard_normal((1, Hkv, d)))
    v = np.repeat(row, M, axis=0)
    pos = np.arange(1, M + 1, dtype=np.int32) * 2
    rank = np.arange(1, M + 1, dtype=np.int32)
    gls = -np.abs(rng.standard_normal(M)).astype(np.float32) * 4
    g = rng.standard_normal(Hq).astype(np.float32)
    c = rng.random(Hq).astype(np.float32)
    out, lse = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, g, c)
    vr = bf16_bits_to_f32(row)[0].astype(np.float64)
    for h in range(Hq):
        np.testing.assert_allclose(out[:, h], np.broadcast_to(vr[h // 2], (M, d)), rtol=1e-14, atol=1e-15)
    # the first query of a sequence sees only itself
    k0 = bf16_bits_to_f32(k).astype(np.float64)
    q0 = bf16_bits_to_f32(q).astype(np.float64)
    for h in range(Hq):
        gain = math.log1p(math.exp(float(g[h])))
        tau = 1 + float(c[h]) * math.log(2.0)
        l0 = (q0[0, h] @ k0[0, h // 2] / math.sqrt(d) + gain * float(gls[0])) / tau
        assert lse[0, h] == pytest.approx(l0, rel=1e-13)


def test_compacted_equals_masked_full_length(oracle_mod):
    """Running the upper layers on the compacted kept tokens equals running
    the full sequence with dropped keys masked out (the training-time form)."""
    rng = np.random.default_rng(16)
    seqlens = [50, 33]
    cu = np.array([0, 50, 83], np.int32)
    span = np.array([[5, 45], [3, 33]], np.int32)
    Hq, Hkv, d = 4, 2, 8
    T = 83
    q = _bf16(rng.standard_normal((T, Hq, d)))
    k = _bf16(rng.standard_normal((T, Hkv, d)))
    v = _bf16(rng.standard_normal((T, Hkv, d)))
    s = (2 * rng.standard_normal(T)).astype(np.float32)
    g = rng.standard_normal(Hq).astype(np.float32)
    c = (0.5 * rng.random(Hq)).astype(np.float32)
    keep = oracle_mod.select_topk(s, cu, span, [12, 7])
    comp = oracle_mod.compact(None, s, keep, cu, span)
    src = comp["src"]
    out_c, _ = oracle_mod.gated_attention(q[src], k[src], v[src], comp["cu_kept"], comp["pos"], comp["rank"],
                                          comp["gls"].astype(np.float32), g, c)
    out_m = oracle_mod.masked_gated_attention(q, k, v, cu, span, keep, s, g, c)
    np.testing.assert_allclose(out_m[src], out_c, rtol=1e-6, atol=1e-7)
    assert (out_m[keep == 0] == 0).all()
    assert len(seqlens) == 2


def test_row_subset_matches_full(oracle_mod):
    rng = np.random.default_rng(17)
    q, k, v, cu = _attn_case(rng, [30, 20], 2, 1, 8)
    M = 50
    pos = np.concatenate([np.arange(1, 31) * 2, np.arange(1, 21) + 3]).astype(np.int32)
    rank = np.concatenate([np.arange(1, 31), np.arange(1, 21)]).astype(np.int32)
    gls = -np.abs(rng.standard_normal(M)).astype(np.float32)
    g = rng.standard_normal(2).astype(np.float32)
    c = rng.random(2).astype(np.float32)
    full, lse = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, g, c)
    rows = np.array([0, 29, 30, 49, 7], np.int64)
    part, lsep = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, g, c, rows=rows)
    np.testing.assert_array_equal(part, full[rows])
    np.testing.assert_array_equal(lsep, lse[rows])
