"""GPU parity of the backward of the token-gated attention against the fp64
oracle, through the C ABI.

Bars, relative to each gradient's own scale (the tensor cores take P and G as
bf16 operands, 2^-9 relative, and dq/dk/dv are returned in bf16):
  dq, dk, dv      max-abs <= 3e-2 * max|ref|, mean-abs <= 6e-3 * mean|ref|
  dgls, dscore    max-abs <= 1e-2 * max|ref|
  dg, dc          max-abs <= 1e-2 * max|ref|
dscore is compared with the oracle's, which takes it from the kept rows' gate
scores themselves (sigmoid(-s) times d gls), not from the kernel's identity.
"""

import functools

import numpy as np
import pytest
import torch

import oracle
from tests import helpers as H
from workloads import CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, make_attention_inputs, make_scores

pytestmark = pytest.mark.gpu

GRAD_MAX_REL = 3e-2
GRAD_MEAN_REL = 6e-3
SUM_MAX_REL = 1e-2


@pytest.fixture(scope="module")
def tg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import learned_token_pruning_rmsnorm_b200 as tg
    tg.load()
    return tg


def _rand_case(seed, seqlens, Hq, Hkv, d, std=0.5):
    rng = np.random.default_rng(seed)
    M = sum(seqlens)
    q = f32_to_bf16_bits((rng.standard_normal((M, Hq, d)) * std).astype(np.float32))
    k = f32_to_bf16_bits((rng.standard_normal((M, Hkv, d)) * std).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((M, Hkv, d)).astype(np.float32))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    rank = np.concatenate([np.arange(1, n + 1) for n in seqlens]).astype(np.int32)
    pos = (rank + np.concatenate([np.sort(rng.integers(0, 400, n)) for n in seqlens])).astype(np.int32)
    s = (2 * rng.standard_normal(M)).astype(np.float32)
    prunable = np.arange(M) >= 24  # the first 24 rows are ones the gate cannot prune
    gls = np.where(prunable, np.minimum(s, 0) - np.log1p(np.exp(-np.abs(s.astype(np.float64)))), 0.0)
    gls = gls.astype(np.float32)
    g = rng.standard_normal(Hq).astype(np.float32)
    c = (0.5 * rng.random(Hq)).astype(np.float32)
    dout = f32_to_bf16_bits(rng.standard_normal((M, Hq, d)).astype(np.float32))
    return {"q": q, "k": k, "v": v, "cu": cu, "pos": pos, "rank": rank, "gls": gls, "g": g, "c": c, "dout": dout,
            "s": s, "prunable": prunable}


def _gpu_backward(tg, cs):
    cu = cs["cu"]
    max_M = int(np.max(np.diff(cu)))
    q, k, v = H.bf16_dev(cs["q"]), H.bf16_dev(cs["k"]), H.bf16_dev(cs["v"])
    pos, rank, gls = H.i32_dev(cs["pos"]), H.i32_dev(cs["rank"]), H.f32_dev(cs["gls"])
    g, c = H.f32_dev(cs["g"]), H.f32_dev(cs["c"])
    out, lse = tg.tg_gated_attention(q, k, v, cu, max_M, pos, rank, gls, g, c, want_lse=True)
    res = tg.tg_gated_attention_backward(q, k, v, out, H.bf16_dev(cs["dout"]), lse, cu, max_M, pos, rank, gls, g, c)
    torch.cuda.synchronize()
    return {key: (None if t is None else (t.float().cpu().numpy())) for key, t in res.items()}


def _check(got, ref, cs, what):
    for key in ("dq", "dk", "dv"):
        err = np.abs(got[key] - ref[key])
        scale = np.abs(ref[key])
        assert err.max() <= GRAD_MAX_REL * scale.max(), f"{what} {key}: max {err.max():.3e} vs {scale.max():.3e}"
        assert err.mean() <= GRAD_MEAN_REL * scale.mean(), f"{what} {key}: mean {err.mean():.3e} vs {scale.mean():.3e}"
    for key in ("dgls", "dscore", "dg", "dc"):
        err = np.abs(got[key] - ref[key])
        assert err.max() <= SUM_MAX_REL * np.abs(ref[key]).max(), f"{what} {key}: {err.max():.3e}"
    assert (got["dscore"][~cs["prunable"]] == 0).all()


def _in_span(src, cu, span):
    """Kept rows whose source token lies in its sequence's prunable span."""
    b = np.searchsorted(cu, src, side="right") - 1
    local = src - cu[b]
    return (local >= span[b, 0]) & (local < span[b, 1])


def _oracle_backward(cs):
    return oracle.gated_attention_backward(cs["q"], cs["k"], cs["v"], cs["cu"], cs["pos"], cs["rank"], cs["gls"],
                                           cs["g"], cs["c"], bf16_bits_to_f32(cs["dout"]).astype(np.float64),
                                           scores=cs["s"], prunable=cs["prunable"])


# GQA groups of 2, 4 and 8 heads reduce dK / dV inside a thread-block cluster; a group of 3
# goes through fp32 partials; a group of 1 writes directly
@pytest.mark.parametrize("seed,seqlens,Hq,Hkv,d", [(1, [192], 4, 2, 64), (2, [300, 1, 129], 4, 2, 64),
                                                   (3, [700, 1, 1000], 4, 2, 128), (4, [257, 130], 3, 1, 64),
                                                   (5, [400], 4, 4, 128), (6, [333, 200], 8, 2, 128),
                                                   (7, [260], 8, 1, 64)])
def test_backward_matches_oracle(tg, seed, seqlens, Hq, Hkv, d):
    cs = _rand_case(seed, seqlens, Hq, Hkv, d)
    got = _gpu_backward(tg, cs)
    ref = _oracle_backward(cs)
    _check(got, ref, cs, f"seed {seed}")


def test_backward_at_the_bench_workload(tg):
    """N=32768, K=2000 (M=2256), 16 query / 8 KV heads, head_dim 128."""
    w = CONFIGS["c2_32k_k2000"]
    cu, span, kb = w.cu_seqlens(), w.span_array(), w.budget_array()
    s = make_scores(w.T, std=2.0, seed=w.seed)
    keep = oracle.select_topk(s, cu, span, kb)
    comp = oracle.compact(None, s, keep, cu, span)
    M = int(comp["cu_kept"][-1])
    ai = make_attention_inputs(w, M, layer=0, qkv_std=0.5)
    rng = np.random.default_rng(8)
    cs = {"q": ai["q"], "k": ai["k"], "v": ai["v"], "cu": comp["cu_kept"], "pos": comp["pos"], "rank": comp["rank"],
          "gls": comp["gls"].astype(np.float32), "g": ai["g"], "c": ai["c"],
          "dout": f32_to_bf16_bits(rng.standard_normal((M, w.Hq, w.d)).astype(np.float32)),
          "s": s[comp["src"]], "prunable": _in_span(comp["src"], cu, span)}
    got = _gpu_backward(tg, cs)
    ref = _oracle_backward(cs)
    _check(got, ref, cs, "c2_32k_k2000")


def test_backward_is_deterministic(tg):
    cs = _rand_case(9, [600, 333], 4, 2, 128)
    a = _gpu_backward(tg, cs)
    b = _gpu_backward(tg, cs)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)


@pytest.mark.parametrize("seed,seqlens,Hq,Hkv", [(10, [64], 2, 1), (14, [300, 129], 4, 2), (15, [257], 2, 2),
                                                (16, [513], 8, 2), (17, [200, 77], 3, 1)])
def test_backward_head_dim_256_matches_oracle(tg, seed, seqlens, Hq, Hkv):
    """head_dim 256: the dQ kernel streams K/V as single-buffered 64-key half tiles, and dV
    and dK come from two launches over the same keys (P^T then G^T), reduced over the
    group's query heads through fp32 partials (a group of one writes bf16 directly).
    Ragged sequences, a partial query tile, several tiles, odd and even groups."""
    cs = _rand_case(seed, seqlens, Hq, Hkv, 256)
    got = _gpu_backward(tg, cs)
    ref = _oracle_backward(cs)
    _check(got, ref, cs, f"d=256 seed {seed}")


def test_backward_head_dim_256_at_c5(tg):
    """The head_dim-256 workload: N=16384, K=2000 (M=2384), 8 query / 2 KV heads."""
    w = CONFIGS["c5_hd256_16k"]
    cu, span, kb = w.cu_seqlens(), w.span_array(), w.budget_array()
    s = make_scores(w.T, std=2.0, seed=w.seed)
    keep = oracle.select_topk(s, cu, span, kb)
    comp = oracle.compact(None, s, keep, cu, span)
    M = int(comp["cu_kept"][-1])
    ai = make_attention_inputs(w, M, layer=0, qkv_std=0.5)
    rng = np.random.default_rng(18)
    cs = {"q": ai["q"], "k": ai["k"], "v": ai["v"], "cu": comp["cu_kept"], "pos": comp["pos"], "rank": comp["rank"],
          "gls": comp["gls"].astype(np.float32), "g": ai["g"], "c": ai["c"],
          "dout": f32_to_bf16_bits(rng.standard_normal((M, w.Hq, w.d)).astype(np.float32)),
          "s": s[comp["src"]], "prunable": _in_span(comp["src"], cu, span)}
    got = _gpu_backward(tg, cs)
    ref = _oracle_backward(cs)
    _check(got, ref, cs, "c5_hd256_16k")


def test_backward_head_dim_256_is_deterministic(tg):
    cs = _rand_case(19, [400, 150], 4, 2, 256)
    a = _gpu_backward(tg, cs)
    b = _gpu_backward(tg, cs)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key], err_msg=key)


@pytest.mark.parametrize("seed,seqlens,Hq,Hkv,d,n_gates", [(11, [300, 129], 4, 2, 128, 2), (12, [260], 8, 2, 64, 4),
                                                           (13, [200, 77], 3, 1, 64, 3), (20, [300], 4, 2, 256, 2)])
def test_backward_with_several_gates_matches_oracle(tg, seed, seqlens, Hq, Hkv, d, n_gates):
    """Several gate modules: the forward's logits carry sum_i softplus(g_i) gls_i; the
    backward returns each gate's dgls, dscore and dg (R24 bars per gate) and the same dq,
    dk, dv, dc bars as one gate."""
    cs = _rand_case(seed, seqlens, Hq, Hkv, d)
    rng = np.random.default_rng(seed + 100)
    M = sum(seqlens)
    scores, gls = [cs["s"]], [cs["gls"]]
    for _ in range(n_gates - 1):
        sc = (2 * rng.standard_normal(M)).astype(np.float32)
        x = np.where(cs["prunable"], np.minimum(sc, 0) - np.log1p(np.exp(-np.abs(sc.astype(np.float64)))), 0.0)
        scores.append(sc)
        gls.append(x.astype(np.float32))
    gains = [cs["g"]] + [rng.standard_normal(Hq).astype(np.float32) for _ in range(n_gates - 1)]
    cu = cs["cu"]
    max_M = int(np.max(np.diff(cu)))
    q, k, v = H.bf16_dev(cs["q"]), H.bf16_dev(cs["k"]), H.bf16_dev(cs["v"])
    pos, rank = H.i32_dev(cs["pos"]), H.i32_dev(cs["rank"])
    gls_d, g_d, c = [H.f32_dev(x) for x in gls], [H.f32_dev(x) for x in gains], H.f32_dev(cs["c"])
    out, lse = tg.tg_gated_attention_gates(q, k, v, cu, max_M, pos, rank, gls_d, g_d, c, want_lse=True)
    res = tg.tg_gated_attention_backward_gates(q, k, v, out, H.bf16_dev(cs["dout"]), lse, cu, max_M, pos, rank,
                                               gls_d, g_d, c)
    torch.cuda.synchronize()
    ref = oracle.gated_attention_backward(cs["q"], cs["k"], cs["v"], cu, cs["pos"], cs["rank"], np.stack(gls),
                                          np.stack(gains), cs["c"], bf16_bits_to_f32(cs["dout"]).astype(np.float64),
                                          scores=np.stack(scores), prunable=cs["prunable"])
    for key in ("dq", "dk", "dv"):
        got = res[key].float().cpu().numpy()
        err, scale = np.abs(got - ref[key]), np.abs(ref[key])
        assert err.max() <= GRAD_MAX_REL * scale.max(), key
        assert err.mean() <= GRAD_MEAN_REL * scale.mean(), key
    got_dc = res["dc"].cpu().numpy()
    assert np.abs(got_dc - ref["dc"]).max() <= SUM_MAX_REL * np.abs(ref["dc"]).max()
    for i in range(n_gates):
        for key in ("dgls", "dscore", "dg"):
            got = res[key][i].cpu().numpy()
            assert np.abs(got - ref[key][i]).max() <= SUM_MAX_REL * np.abs(ref[key][i]).max(), (key, i)
