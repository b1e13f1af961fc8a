"""CPU pins of the oracle's backward of the token-gated attention.

Pinned against things other than its own chain rule: PyTorch fp64 autograd
through the forward written as library calls (per-row scaled_dot_product_
attention of the query scaled by sm/tau with additive mask softplus(g) gls / tau -- the
composition the forward pins already tie to the oracle's forward), central
differences of the oracle's own forward for g, c and gls, and the closed form
of uniform values (the output no longer depends on any logit).
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from workloads import bf16_bits_to_f32, f32_to_bf16_bits


def _case(seed, seqlens, Hq, Hkv, d, std=0.8):
    rng = np.random.default_rng(seed)
    M = sum(seqlens)
    q = f32_to_bf16_bits((rng.standard_normal((M, Hq, d)) * std).astype(np.float32))
    k = f32_to_bf16_bits((rng.standard_normal((M, Hkv, d)) * std).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((M, Hkv, d)).astype(np.float32))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    rank = np.concatenate([np.arange(1, n + 1) for n in seqlens]).astype(np.int32)
    pos = (rank + np.concatenate([np.sort(rng.integers(0, 30, n)) for n in seqlens])).astype(np.int32)
    gls = -np.abs(rng.standard_normal(M) * 2).astype(np.float32)
    gls[:3] = 0.0
    g = rng.standard_normal(Hq).astype(np.float32)
    c = (0.6 * rng.random(Hq)).astype(np.float32)
    dout = rng.standard_normal((M, Hq, d))
    return q, k, v, cu, pos, rank, gls, g, c, dout


def _autograd(q, k, v, cu, pos, rank, gls, g, c, dout):
    Hq, Hkv, d = q.shape[1], k.shape[1], q.shape[2]
    qt = torch.tensor(bf16_bits_to_f32(q), dtype=torch.float64, requires_grad=True)
    kt = torch.tensor(bf16_bits_to_f32(k), dtype=torch.float64, requires_grad=True)
    vt = torch.tensor(bf16_bits_to_f32(v), dtype=torch.float64, requires_grad=True)
    gl = torch.tensor(gls, dtype=torch.float64, requires_grad=True)
    gt = torch.tensor(g, dtype=torch.float64, requires_grad=True)
    ct = torch.tensor(c, dtype=torch.float64, requires_grad=True)
    sm = 1.0 / math.sqrt(d)
    outs = []
    for b in range(len(cu) - 1):
        for i in range(cu[b], cu[b + 1]):
            row = []
            for h in range(Hq):
                hk = h // (Hq // Hkv)
                tau = 1 + ct[h] * math.log(pos[i] / rank[i])
                mask = F.softplus(gt[h]) * gl[cu[b]:i + 1] / tau
                # SDPA's scale is a plain number: sm / tau enters through the query instead
                o = F.scaled_dot_product_attention((qt[i, h] * (sm / tau))[None, None, None],
                                                   kt[cu[b]:i + 1, hk][None, None], vt[cu[b]:i + 1, hk][None, None],
                                                   attn_mask=mask[None, None, None], scale=1.0)
                row.append(o[0, 0, 0])
            outs.append(torch.stack(row))
    out = torch.stack(outs)
    (out * torch.from_numpy(dout)).sum().backward()
    return {"dq": qt.grad.numpy(), "dk": kt.grad.numpy(), "dv": vt.grad.numpy(), "dgls": gl.grad.numpy(),
            "dg": gt.grad.numpy(), "dc": ct.grad.numpy()}


@pytest.mark.parametrize("seed,seqlens,Hq,Hkv,d", [(1, [13, 9], 4, 2, 8), (2, [1, 17], 3, 1, 4),
                                                   (3, [20], 2, 2, 16)])
def test_backward_matches_autograd_of_library_forward(oracle_mod, seed, seqlens, Hq, Hkv, d):
    q, k, v, cu, pos, rank, gls, g, c, dout = _case(seed, seqlens, Hq, Hkv, d)
    ref = _autograd(q, k, v, cu, pos, rank, gls, g, c, dout)
    got = oracle_mod.gated_attention_backward(q, k, v, cu, pos, rank, gls, g, c, dout)
    for key in ("dq", "dk", "dv", "dgls", "dg", "dc"):
        np.testing.assert_allclose(got[key], ref[key], rtol=1e-9, atol=1e-11, err_msg=key)


def _loss(oracle_mod, q, k, v, cu, pos, rank, gls, g, c, dout):
    out, _ = oracle_mod.gated_attention(q, k, v, cu, pos, rank, gls, g, c)
    return float(np.sum(out * dout))


def test_backward_matches_central_differences(oracle_mod):
    """Gain, temperature and one logsigmoid perturbed by +-2^-12 (exact in fp32)."""
    q, k, v, cu, pos, rank, gls, g, c, dout = _case(4, [15, 10], 4, 2, 8)
    got = oracle_mod.gated_attention_backward(q, k, v, cu, pos, rank, gls, g, c, dout)
    eps = 2.0 ** -12
    for h in range(4):
        gp, gm = g.copy(), g.copy()
        gp[h] += eps
        gm[h] -= eps
        fd = (_loss(oracle_mod, q, k, v, cu, pos, rank, gls, gp, c, dout) -
              _loss(oracle_mod, q, k, v, cu, pos, rank, gls, gm, c, dout)) / (2 * eps)
        assert got["dg"][h] == pytest.approx(fd, rel=1e-4, abs=1e-8)
        cp, cm = c.copy(), c.copy()
        cp[h] += eps
        cm[h] -= eps
        fd = (_loss(oracle_mod, q, k, v, cu, pos, rank, gls, g, cp, dout) -
              _loss(oracle_mod, q, k, v, cu, pos, rank, gls, g, cm, dout)) / (2 * eps)
        assert got["dc"][h] == pytest.approx(fd, rel=1e-4, abs=1e-8)
    for j in (3, 7, 14, 20):
        lp, lm = gls.copy(), gls.copy()
        lp[j] += eps
        lm[j] -= eps
        fd = (_loss(oracle_mod, q, k, v, cu, pos, rank, lp, g, c, dout) -
              _loss(oracle_mod, q, k, v, cu, pos, rank, lm, g, c, dout)) / (2 * eps)
        assert got["dgls"][j] == pytest.approx(fd, rel=1e-4, abs=1e-8)


def test_uniform_values_give_no_logit_gradient(oracle_mod):
    """With every value row equal the output is that row whatever the logits: all
    gradients through the logits vanish, and the value gradient sums to the
    output gradient (the weights of each row sum to one)."""
    q, k, v, cu, pos, rank, gls, g, c, dout = _case(5, [12, 8], 4, 2, 8)
    v = np.repeat(v[:1], len(v), axis=0)
    got = oracle_mod.gated_attention_backward(q, k, v, cu, pos, rank, gls, g, c, dout)
    for key in ("dq", "dk", "dgls", "dg", "dc"):
        assert np.max(np.abs(got[key])) < 1e-12, key
    for hk in range(2):
        want = dout[:, 2 * hk:2 * hk + 2].sum(axis=(0, 1))
        np.testing.assert_allclose(got["dv"][:, hk].sum(axis=0), want, rtol=1e-12, atol=1e-12)


def test_temperature_gradient_vanishes_where_pos_equals_rank(oracle_mod):
    """ln(pos/rank) = 0 rows carry no temperature gradient: with every pos equal to
    its rank, dc is exactly 0 while dg is not."""
    q, k, v, cu, pos, rank, gls, g, c, dout = _case(6, [16], 2, 1, 8)
    got = oracle_mod.gated_attention_backward(q, k, v, cu, rank.copy(), rank, gls, g, c, dout)
    assert (got["dc"] == 0).all()
    assert np.abs(got["dg"]).max() > 1e-6


def _logsigmoid(s):
    s = np.asarray(s, dtype=np.float64)
    return np.minimum(s, 0.0) - np.log1p(np.exp(-np.abs(s)))


def test_score_gradient_matches_central_differences(oracle_mod):
    """d loss / d s_j, pinned by differencing the oracle's forward in the gate score
    itself: s_j is moved by +-2^-6 and gls_j = logsigmoid(s_j) recomputed, so a sign,
    a missing factor or sigmoid(s) in place of sigmoid(-s) in dscore fails by O(1).
    Rows the gate cannot prune (gls = 0, no bias) get 0."""
    q, k, v, cu, pos, rank, gls, g, c, dout = _case(7, [14, 11], 4, 2, 8)
    rng = np.random.default_rng(70)
    s = (2.0 * rng.standard_normal(len(gls))).astype(np.float32)
    s[[5, 12]] = [9.0, -9.0]  # saturated ends of the sigmoid
    prunable = np.ones(len(gls), dtype=bool)
    prunable[:3] = False
    gls = np.where(prunable, _logsigmoid(s), 0.0).astype(np.float32)
    got = oracle_mod.gated_attention_backward(q, k, v, cu, pos, rank, gls, g, c, dout, scores=s, prunable=prunable)
    assert (got["dscore"][~prunable] == 0).all()
    eps = 2.0 ** -6
    for j in (3, 5, 8, 12, 16, 24):
        sp, sm = s.astype(np.float64), s.astype(np.float64)
        sp = sp.copy()
        sm = sm.copy()
        sp[j] += eps
        sm[j] -= eps
        lp = np.where(prunable, _logsigmoid(sp), 0.0).astype(np.float32)
        lm = np.where(prunable, _logsigmoid(sm), 0.0).astype(np.float32)
        fd = (_loss(oracle_mod, q, k, v, cu, pos, rank, lp, g, c, dout) -
              _loss(oracle_mod, q, k, v, cu, pos, rank, lm, g, c, dout)) / (2 * eps)
        assert got["dscore"][j] == pytest.approx(fd, rel=2e-3, abs=1e-7), j


def test_two_gate_backward_matches_central_differences(oracle_mod):
    """Several gates: each gate's logsigmoids and gains, perturbed by +-2^-12 in the
    oracle's two-gate forward, give its dgls and dg."""
    q, k, v, cu, pos, rank, gls, g, c, dout = _case(8, [12, 9], 4, 2, 8)
    rng = np.random.default_rng(80)
    gls2 = np.stack([gls, -np.abs(rng.standard_normal(len(gls)) * 1.5).astype(np.float32)])
    gls2[1, :2] = 0.0
    g2 = np.stack([g, rng.standard_normal(4).astype(np.float32)])
    got = oracle_mod.gated_attention_backward(q, k, v, cu, pos, rank, gls2, g2, c, dout)
    assert got["dgls"].shape == (2, len(gls)) and got["dg"].shape == (2, 4)
    eps = 2.0 ** -12
    for gi in range(2):
        for j in (2, 6, 15, 20):
            lp, lm = gls2.copy(), gls2.copy()
            lp[gi, j] += eps
            lm[gi, j] -= eps
            fd = (_loss(oracle_mod, q, k, v, cu, pos, rank, lp, g2, c, dout) -
                  _loss(oracle_mod, q, k, v, cu, pos, rank, lm, g2, c, dout)) / (2 * eps)
            assert got["dgls"][gi, j] == pytest.approx(fd, rel=1e-4, abs=1e-8), (gi, j)
        for h in range(4):
            gp, gm = g2.copy(), g2.copy()
            gp[gi, h] += eps
            gm[gi, h] -= eps
            fd = (_loss(oracle_mod, q, k, v, cu, pos, rank, gls2, gp, c, dout) -
                  _loss(oracle_mod, q, k, v, cu, pos, rank, gls2, gm, c, dout)) / (2 * eps)
            assert got["dg"][gi, h] == pytest.approx(fd, rel=1e-4, abs=1e-8), (gi, h)


def test_split_gate_backward_equals_one_gate(oracle_mod):
    """Two gates with the same gains whose logsigmoids add up to one gate's give that
    gate's dq, dk, dv, dc; each of them gets the one gate's dgls (same gain), and their
    dg add up to the one gate's."""
    q, k, v, cu, pos, rank, gls, g, c, dout = _case(9, [10, 7], 2, 1, 8)
    # a keeps the top 12 significand bits of gls, b the rest: both exact, a + b == gls in fp32
    a = (gls.view(np.uint32) & np.uint32(0xFFFFF800)).view(np.float32)
    b = (gls - a).astype(np.float32)
    assert np.array_equal(a + b, gls) and np.abs(b).max() > 0
    one = oracle_mod.gated_attention_backward(q, k, v, cu, pos, rank, a + b, g, c, dout)
    two = oracle_mod.gated_attention_backward(q, k, v, cu, pos, rank, np.stack([a, b]), np.stack([g, g]), c, dout)
    for key in ("dq", "dk", "dv", "dc"):
        np.testing.assert_allclose(two[key], one[key], rtol=1e-9, atol=1e-12, err_msg=key)
    for gi in range(2):
        np.testing.assert_allclose(two["dgls"][gi], one["dgls"], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(two["dg"].sum(axis=0), one["dg"], rtol=1e-9, atol=1e-12)
