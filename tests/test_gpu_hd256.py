"""GPU parity at head_dim 256 and for odd GQA groups (the one-head attention
kernel, P kept in tensor memory) against the fp64 oracle, through the C ABI.

The pages' key-bias attention kernel serves head dimensions 128 and 256
(TokenGate AI summary, "Main Findings": kernel overhead).  Bars: attention
within max-abs 2e-2 and mean-abs 2e-3, LSE within 1e-3.
"""

import functools

import numpy as np
import pytest
import torch

import oracle
from tests import helpers as H
from workloads import CONFIGS, f32_to_bf16_bits, make_attention_inputs, make_scores

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import learned_token_pruning_rmsnorm_b200 as tg
    tg.load()
    return tg


def _rand_case(seed, seqlens, Hq, Hkv, d, std=0.5, gap=500):
    rng = np.random.default_rng(seed)
    M = sum(seqlens)
    q = f32_to_bf16_bits((rng.standard_normal((M, Hq, d)) * std).astype(np.float32))
    k = f32_to_bf16_bits((rng.standard_normal((M, Hkv, d)) * std).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((M, Hkv, d)).astype(np.float32))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    rank = np.concatenate([np.arange(1, n + 1) for n in seqlens]).astype(np.int32)
    pos = (rank + np.concatenate([np.sort(rng.integers(0, gap, n)) for n in seqlens])).astype(np.int32)
    gls = -np.abs(rng.standard_normal(M) * 2).astype(np.float32)
    gls[:16] = 0.0
    g = rng.standard_normal(Hq).astype(np.float32)
    c = (0.5 * rng.random(Hq)).astype(np.float32)
    return q, k, v, cu, pos, rank, gls, g, c


def _run(tg, q, k, v, cu, pos, rank, gls, g, c):
    out, lse = tg.tg_gated_attention(H.bf16_dev(q), H.bf16_dev(k), H.bf16_dev(v), cu, int(np.max(np.diff(cu))),
                                     H.i32_dev(pos), H.i32_dev(rank), H.f32_dev(gls), H.f32_dev(g), H.f32_dev(c),
                                     want_lse=True)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("d,Hq,Hkv", [(256, 8, 2), (256, 6, 2), (256, 4, 4), (64, 6, 2), (128, 3, 1), (128, 4, 4)])
def test_one_head_kernel_matches_oracle(tg, d, Hq, Hkv):
    """Ragged varlen batch (a one-token sequence, tails that are not a tile multiple)."""
    q, k, v, cu, pos, rank, gls, g, c = _rand_case(80 + d + Hq, [300, 1, 129, 520], Hq, Hkv, d)
    out, lse = _run(tg, q, k, v, cu, pos, rank, gls, g, c)
    out_ref, lse_ref = oracle.gated_attention(q, k, v, cu, pos, rank, gls, g, c)
    H.assert_attention_close(out, out_ref, f"d={d} Hq={Hq} Hkv={Hkv}")
    assert np.max(np.abs(lse - lse_ref)) <= H.LSE_ABS


def test_hd256_peaked_logits(tg):
    q, k, v, cu, pos, rank, gls, g, c = _rand_case(91, [400, 257], 8, 2, 256, std=1.0)
    out, lse = _run(tg, q, k, v, cu, pos, rank, gls, g, c)
    out_ref, lse_ref = oracle.gated_attention(q, k, v, cu, pos, rank, gls, g, c)
    H.assert_attention_close(out, out_ref, "d=256 peaked")
    assert np.max(np.abs(lse - lse_ref)) <= H.LSE_ABS * 10


@functools.lru_cache(maxsize=None)
def hd256_case(rows_step=5):
    w = CONFIGS["c5_hd256_16k"]
    cu, span, kb = w.cu_seqlens(), w.span_array(), w.budget_array()
    s = make_scores(w.T, std=2.0, seed=w.seed)
    keep = oracle.select_topk(s, cu, span, kb)
    comp = oracle.compact(None, s, keep, cu, span)
    M = int(comp["cu_kept"][-1])
    ai = make_attention_inputs(w, M, layer=0)
    gls = comp["gls"].astype(np.float32)
    rows = np.unique(np.concatenate([np.arange(0, M, rows_step), np.arange(M - 128, M)])).astype(np.int64)
    out_ref, lse_ref = oracle.gated_attention(ai["q"], ai["k"], ai["v"], comp["cu_kept"], comp["pos"],
                                              comp["rank"], gls, ai["g"], ai["c"], rows=rows)
    return w, comp, ai, gls, rows, out_ref, lse_ref


def test_hd256_workload_matches_oracle(tg):
    """N=16384, K=2000 (M=2384), 8 query / 2 KV heads, head_dim 256, sampled rows."""
    w, comp, ai, gls, rows, out_ref, lse_ref = hd256_case()
    out, lse = _run(tg, ai["q"], ai["k"], ai["v"], comp["cu_kept"], comp["pos"], comp["rank"], gls, ai["g"],
                    ai["c"])
    H.assert_attention_close(out[rows], out_ref, "c5_hd256_16k")
    assert np.max(np.abs(lse[rows] - lse_ref)) <= H.LSE_ABS


def test_hd256_tau_one_rows_bitwise(tg):
    """Rows with pos == rank have tau exactly 1: bit-equal to a run with c = 0."""
    w, comp, ai, gls, _, _, _ = hd256_case()
    a, _ = _run(tg, ai["q"], ai["k"], ai["v"], comp["cu_kept"], comp["pos"], comp["rank"], gls, ai["g"], ai["c"])
    b, _ = _run(tg, ai["q"], ai["k"], ai["v"], comp["cu_kept"], comp["pos"], comp["rank"], gls, ai["g"],
                np.zeros_like(ai["c"]))
    eq = comp["pos"] == comp["rank"]
    np.testing.assert_array_equal(a[eq], b[eq])
    assert np.abs(a[~eq] - b[~eq]).max() > 0


def test_hd256_reduces_to_causal_sdpa(tg):
    """bias 0, tau 1: ordinary causal GQA attention (PyTorch fp64 SDPA)."""
    rng = np.random.default_rng(93)
    seqlens = [333, 130]
    Hq, Hkv, d = 8, 2, 256
    M = sum(seqlens)
    q = f32_to_bf16_bits((rng.standard_normal((M, Hq, d)) * 0.4).astype(np.float32))
    k = f32_to_bf16_bits((rng.standard_normal((M, Hkv, d)) * 0.4).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((M, Hkv, d)).astype(np.float32))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    pos = np.concatenate([np.arange(1, n + 1) for n in seqlens]).astype(np.int32)
    out, _ = _run(tg, q, k, v, cu, pos, pos, np.zeros(M, np.float32), rng.standard_normal(Hq).astype(np.float32),
                  rng.random(Hq).astype(np.float32))
    qt, kt, vt = (H.bf16_dev(a, "cpu").double() for a in (q, k, v))
    ref = []
    for b in range(len(seqlens)):
        a0, a1 = cu[b], cu[b + 1]
        qb = qt[a0:a1].transpose(0, 1)
        kb = kt[a0:a1].transpose(0, 1).repeat_interleave(Hq // Hkv, 0)
        vb = vt[a0:a1].transpose(0, 1).repeat_interleave(Hq // Hkv, 0)
        ref.append(torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, is_causal=True).transpose(0, 1))
    H.assert_attention_close(out, torch.cat(ref).numpy(), "sdpa d=256")


def test_hd256_masked_full_length(tg):
    """The full-length masked form at a sampled budget, head_dim 256, all rows."""
    rng = np.random.default_rng(94)
    seqlens = [700, 300]
    cu = np.array([0, 700, 1000], np.int32)
    span = np.array([[50, 650], [0, 300]], np.int32)
    kbud = np.array([37, 120], np.int32)
    Hq, Hkv, d = 8, 2, 256
    T = 1000
    q = f32_to_bf16_bits((rng.standard_normal((T, Hq, d)) * 0.3).astype(np.float32))
    k = f32_to_bf16_bits((rng.standard_normal((T, Hkv, d)) * 0.3).astype(np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((T, Hkv, d)).astype(np.float32))
    s = (2 * rng.standard_normal(T)).astype(np.float32)
    g = rng.standard_normal(Hq).astype(np.float32)
    c = (0.5 * rng.random(Hq)).astype(np.float32)
    out, keep = tg.tg_masked_gated_attention(H.bf16_dev(q), H.bf16_dev(k), H.bf16_dev(v), H.f32_dev(s), cu, span,
                                             kbud, H.f32_dev(g), H.f32_dev(c))
    torch.cuda.synchronize()
    keep_ref = oracle.select_topk(s, cu, span, kbud)
    np.testing.assert_array_equal(keep.cpu().numpy(), keep_ref)
    ref = oracle.masked_gated_attention(q, k, v, cu, span, keep_ref, s, g, c)
    H.assert_attention_close(out.float().cpu().numpy(), ref, "masked d=256")
    assert len(seqlens) == 2


def test_hd256_two_gates(tg):
    q, k, v, cu, pos, rank, gls, g, c = _rand_case(95, [600, 200], 8, 2, 256)
    rng = np.random.default_rng(96)
    gls2 = np.where(gls != 0, -np.abs(rng.standard_normal(len(gls))), 0.0).astype(np.float32)
    g2 = rng.standard_normal(8).astype(np.float32)
    out, lse = tg.tg_gated_attention_gates(H.bf16_dev(q), H.bf16_dev(k), H.bf16_dev(v), cu, 600, H.i32_dev(pos),
                                           H.i32_dev(rank), [H.f32_dev(gls), H.f32_dev(gls2)],
                                           [H.f32_dev(g), H.f32_dev(g2)], H.f32_dev(c), want_lse=True)
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle.gated_attention(q, k, v, cu, pos, rank, np.stack([gls, gls2]), np.stack([g, g2]), c)
    H.assert_attention_close(out.float().cpu().numpy(), out_ref, "d=256 two gates")
    assert np.max(np.abs(lse.cpu().numpy() - lse_ref)) <= H.LSE_ABS
