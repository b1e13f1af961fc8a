// Backward of stage 4, the token-gated causal GQA attention (TokenGate AI
// summary, "Key Contributions" 2 and 3: the gate bias is what carries the task
// loss's gradient back to the scoring network, and the gain and temperature
// are learned).  One gate.  With
//   l_ij = (sm q_i.k_j + beta_h gls_j) / tau_ih,   beta_h = softplus(g_h),
//   P = softmax_j(l),   out_i = sum_j P_ij v_j,
// and the upstream gradient dout:
//   dP_ij = dout_i.v_j,  D_i = dout_i.out_i,  dl_ij = P_ij (dP_ij - D_i),
//   G_ij = dl_ij / tau_ih,
//   dq_i = sm sum_j G_ij k_j,  dk_j = sm sum_i G_ij q_i,  dv_j = sum_i P_ij dout_i,
//   dgls_j = sum_h beta_h sum_i G_ij,  dbeta_h = sum_ij G_ij gls_j,
//   dtau_ih = -sum_j dl_ij l_ij / tau_ih,
//   dg_h = dbeta_h sigmoid(g_h),  dc_h = sum_i dtau_ih ln(pos_i / rank_i),
//   d score_j = dgls_j sigmoid(-score_j) = dgls_j (1 - exp(gls_j)).
//
// Three or four launches in this order, no atomics (results do not depend on
// scheduling):
//   dq       one CTA per (query head, 128-query tile), the forward's layout:
//            S = Q K^T and dP = dO V^T, G as bf16 over S, dQ += G K.  It forms
//            D_ih = dout_i.out_i for its rows; the per-query sums for dtau run
//            along each thread's row, which also yields the exact
//            D'_i = sum_j P_ij dP_ij.  It leaves each row's factors (with D' in
//            place of D) for the dkv kernel.
//   dkv      one CTA per (query head, 128-key tile): for every half (64
//            queries) of every causal query tile, S^T = K Q^T and dP^T = V dO^T
//            on the tensor core (TMEM lanes = keys), then P^T and G^T as bf16
//            over the first 32 columns of S^T and dP^T, and dV += P^T dO,
//            dK += G^T Q read from TMEM.  The per-key sums of G (the gate
//            bias's gradient, per head) are sums along each thread's own row.
//            The query heads of a GQA group leave fp32 partials of dK / dV (a
//            group of one writes bf16 itself).
//   kv_reduce sums those partials in head order (groups of two or more only).
//   finish   dgls / d score per key, dg and dc per head (dbeta from the per-key
//            sums of G; the dq kernel leaves one partial sum of the dc terms per
//            query tile).
// Every row of P is rebuilt from the forward's log-sum-exp.

#include "tg_sm100.cuh"

namespace tg {
namespace {

using namespace sm100;

constexpr int BT = 128;  // rows of a query or key tile (= TMEM lanes)
constexpr float LOG2E_B = 1.4426950408889634f;
constexpr float LN2_B = 0.6931471805599453f;

__device__ __forceinline__ float softplus_b(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }

// The gains beta_i = softplus(g_i[h]) of every gate for query head h (0 past the last gate).
struct GateGains {
    float b0, b1, b2, b3;
};
__device__ __forceinline__ GateGains gate_gains(const GateSet& gs, int h) {
    GateGains r;
    r.b0 = softplus_b(gs.g[0][h]);
    r.b1 = gs.n > 1 ? softplus_b(gs.g[1][h]) : 0.f;
    r.b2 = gs.n > 2 ? softplus_b(gs.g[2][h]) : 0.f;
    r.b3 = gs.n > 3 ? softplus_b(gs.g[3][h]) : 0.f;
    return r;
}
// The bias of kept row `row` for that head: sum_i beta_i gls_i[row] (loads through L2: the
// compaction map may have been written during this kernel's lifetime).
__device__ __forceinline__ float gate_bias(const GateSet& gs, const GateGains& w, int64_t row) {
    float acc = w.b0 * __ldcg(gs.gls[0] + row);
    if (gs.n > 1) acc = fmaf(w.b1, __ldcg(gs.gls[1] + row), acc);
    if (gs.n > 2) acc = fmaf(w.b2, __ldcg(gs.gls[2] + row), acc);
    if (gs.n > 3) acc = fmaf(w.b3, __ldcg(gs.gls[3] + row), acc);
    return acc;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ bool drain_wait_b(uint32_t bar, uint32_t parity, int* status) {
    volatile int never = 0;
    return mbar_wait(bar, parity, &never, status, TG_WHERE_DRAIN);
}

// ---------------------------------------------------------------------------
// dK, dV and the per-key sums of G: one CTA per (query head, 128-key tile, sequence).
//
// 320 threads: warps 0-7 compute, warp 8 TMA producer, warp 9 MMA issuer.  The K
// and V tiles stay resident; the (Q, dO) tiles of the causal query tiles stream
// through a two-stage ring.  TMEM (512 columns): two (S^T | dP^T) buffers of half a
// query tile (64 queries, 64 + 64 columns), then dV and dK.  Per half step u the
// issuer puts out S^T = K Q^T and dP^T = V dO^T into buffer u & 1, then, once the
// compute warps have turned half u - 1 into P^T and G^T, accumulates dV += P^T dO
// and dK += G^T Q from TMEM: the tensor core computes one half while the compute
// warps work on the other (tcgen05 operations of one thread execute in issue
// order, so a buffer is overwritten only after the products that read it).
// Warps w and w + 4 share key rows 32 (w & 3) .. + 31 (the TMEM lanes of that
// quarter) and split each half's 64 queries.  Each element of P^T is rebuilt from
// the query's log-sum-exp; the per-query factors (left by the dQ kernel, one
// float4 per query row and head) go through a small table of each warp's own.
constexpr int DKV_THREADS = 320;

// bar.red.or over the two compute warps of one row group (named barrier 2 + q4, 64 threads)
__device__ __forceinline__ bool pair_red_or(int id, bool pred) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, 64, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"(static_cast<uint32_t>(pred)), "r"(id)
        : "memory");
    return res != 0;
}

// PASS 0 computes dV and dK together (head_dim <= 128).  At head_dim 256 the two fp32
// accumulators alone would fill TMEM, so the work runs as two launches over the same keys:
// PASS 1 forms P^T and accumulates dV = P^T dO, PASS 2 forms G^T and accumulates dK = G^T Q
// (and the per-key sums of G); there the (Q, dO) rows stream as half query tiles (64 rows),
// in two stages for PASS 1 (no V needed) and one for PASS 2 (K and V resident).
template <int HD, int PASS = 0>
struct DkvSmem {
    static constexpr bool QD_HALF = PASS != 0;
    static constexpr bool HAS_V = PASS != 1;  // dP^T = V dO^T is not needed for dV alone
    static constexpr int TILE = BT * HD * 2;
    static constexpr int QD_ROWS = QD_HALF ? 64 : BT;
    static constexpr int QD_STAGE = QD_ROWS * HD * 2;  // the Q (or dO) rows of one stage
    static constexpr int QD_STAGES = PASS == 2 ? 1 : 2;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + TILE;
    static constexpr int OFF_Q = OFF_V + (HAS_V ? TILE : 0);          // [QD_STAGES]
    static constexpr int OFF_DO = OFF_Q + QD_STAGES * QD_STAGE;        // [QD_STAGES]
    static constexpr int OFF_TAB = OFF_DO + QD_STAGES * QD_STAGE;      // [8 warps][2][4][32] fp32 query factors
    static constexpr int OFF_XCH = OFF_TAB + 8 * 2 * 4 * 32 * 4;  // [BT] fp32: the second query half's key sums
    static constexpr int OFF_BAR = OFF_XCH + BT * 4;
    static constexpr int NUM_BARS = 12;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(ALLOC <= 227 * 1024, "shared memory");
    static_assert(2 * BT + (PASS == 0 ? 2 : 1) * HD <= 512, "TMEM columns");
    static_assert(PASS != 0 || HD <= 128, "head_dim 256 runs as two passes");
};

enum : int {
    D_KV_FULL = 0,
    D_QD_FULL = 1,   // [2]
    D_QD_EMPTY = 3,  // [2]
    D_SDP_FULL = 5,  // [2]
    D_PG_FULL = 7,   // [2]
    D_ACC_DONE = 9,
    D_DRAIN = 10
};

template <int HD, int PASS = 0>
__global__ void __launch_bounds__(DKV_THREADS, 1)
gated_attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                          const int32_t* __restrict__ cu_kept, const GateSet gates,
                          const float4* __restrict__ fac, float sm_scale, int Hq,
                          int Hkv, int64_t M_total,
                          uint16_t* __restrict__ dk, uint16_t* __restrict__ dv, float* __restrict__ part_k,
                          float* __restrict__ part_v, float* __restrict__ colsum, int* __restrict__ status,
                          int cl) {
    using L = DkvSmem<HD, PASS>;
    constexpr bool DO_DV = PASS != 2, DO_DK = PASS != 1;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // One query head per CTA.  The heads of a GQA group of 2, 4 or 8 run as one cluster
    // (cl = the group size, cluster rank = head within the group): at the end the other
    // heads' fp32 dK / dV go into their own shared memory and rank 0 adds them in head
    // order and writes bf16.  Other groups of two or more leave fp32 partials that
    // bwd_kv_reduce_kernel sums in head order; a group of one writes bf16 directly.  A
    // cluster's CTAs share kt and b, so they return here together or not at all.
    const int h = blockIdx.x, kt = blockIdx.y, b = blockIdx.z;
    // Early start: every input but the dQ kernel's factor records was complete before the dQ
    // kernel (this kernel's predecessor) passed its own wait, and this kernel starts only
    // after that, so the set-up and the tile loads go ahead while the dQ kernel drains; only
    // the compute warps wait, before their first factor record.
    pdl_trigger();
    const int seq0 = cu_kept[b];
    const int Mb = cu_kept[b + 1] - seq0;
    if (kt * BT >= Mb) return;
    const int n_qt = (Mb + BT - 1) / BT;
    const int grp = Hq / Hkv;
    const int hk = h / grp, hh = h - hk * grp;
    const int nq = n_qt - kt;  // causal query tiles
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t sK = sbase + L::OFF_K, sV = sbase + L::OFF_V, sQ = sbase + L::OFF_Q, sDO = sbase + L::OFF_DO;
    auto bar = [&](int i) { return sbase + L::OFF_BAR + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar(D_KV_FULL), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(D_QD_FULL + s), 1);
            mbar_init(bar(D_QD_EMPTY + s), 1);
            mbar_init(bar(D_SDP_FULL + s), 1);
            mbar_init(bar(D_PG_FULL + s), 256);  // every thread of the eight compute warps
        }
        mbar_init(bar(D_ACC_DONE), 1);
        mbar_init(bar(D_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // half buffer hb: S^T of 64 queries at columns [128 hb, +64), dP^T at [128 hb + 64, +64);
    // P^T and G^T (bf16 pairs) go over the first 32 columns of each
    const uint32_t tDV = tmem + 2 * BT, tDK = tmem + 2 * BT + (PASS == 0 ? HD : 0);

    bool epi_ok = false;  // a compute thread's accumulators are complete
    if (warp == 8) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmDO);
            mbar_expect_tx(bar(D_KV_FULL), (L::HAS_V ? 2 : 1) * L::TILE);
#pragma unroll
            for (int hf = 0; hf < HD / 64; ++hf) {
                tma_load_2d(sK + hf * BT * 128, &tmK, hk * HD + hf * 64, seq0 + kt * BT, bar(D_KV_FULL));
                if (L::HAS_V)
                    tma_load_2d(sV + hf * BT * 128, &tmV, hk * HD + hf * 64, seq0 + kt * BT, bar(D_KV_FULL));
            }
            int issued[2] = {0, 0};
            if constexpr (L::QD_HALF) {
                // half query tile u (64 rows: tile kt + u / 2, rows 64 (u & 1) ..) into stage u % S
                constexpr int S = L::QD_STAGES;
                for (int u = 0; u < 2 * nq; ++u) {
                    const int s = u % S;
                    if (u >= S && !mbar_wait(bar(D_QD_EMPTY + s), ((u / S) - 1) & 1, abort_flag, status,
                                             TG_WHERE_PRODUCER))
                        break;
                    mbar_expect_tx(bar(D_QD_FULL + s), 2 * L::QD_STAGE);
                    const int row = seq0 + kt * BT + u * 64;
#pragma unroll
                    for (int hf = 0; hf < HD / 64; ++hf) {
                        tma_load_2d(sQ + s * L::QD_STAGE + hf * 64 * 128, &tmQ, h * HD + hf * 64, row,
                                    bar(D_QD_FULL + s));
                        tma_load_2d(sDO + s * L::QD_STAGE + hf * 64 * 128, &tmDO, h * HD + hf * 64, row,
                                    bar(D_QD_FULL + s));
                    }
                    ++issued[s];
                }
            } else {
                for (int t = 0; t < nq; ++t) {
                    const int s = t & 1;
                    const int i = kt + t;
                    if (t >= 2 && !mbar_wait(bar(D_QD_EMPTY + s), ((t - 2) >> 1) & 1, abort_flag, status,
                                             TG_WHERE_PRODUCER))
                        break;
                    mbar_expect_tx(bar(D_QD_FULL + s), 2 * L::TILE);
#pragma unroll
                    for (int hf = 0; hf < HD / 64; ++hf) {
                        tma_load_2d(sQ + s * L::TILE + hf * BT * 128, &tmQ, h * HD + hf * 64, seq0 + i * BT,
                                    bar(D_QD_FULL + s));
                        tma_load_2d(sDO + s * L::TILE + hf * BT * 128, &tmDO, h * HD + hf * 64, seq0 + i * BT,
                                    bar(D_QD_FULL + s));
                    }
                    ++issued[s];
                }
            }
            if (*abort_flag) {
                drain_wait_b(bar(D_KV_FULL), 0, status);
                for (int s = 0; s < 2; ++s)
                    if (issued[s]) drain_wait_b(bar(D_QD_FULL + s), (issued[s] - 1) & 1, status);
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(BT, 64, false);
            constexpr uint32_t idesc_acc = idesc_bf16_f32(BT, HD, true);
            // Matrix descriptors are built once per stage; an operand at a byte offset is the
            // same descriptor with offset / 16 added to its start-address field (shared-memory
            // addresses stay below 2^18, so the 14-bit field never carries).
            // (half-tile stages hold only half u: no offset for hb, and the rows' 64-column boxes
            // are QD_ROWS * 128 bytes apart)
            constexpr int QS = L::QD_HALF ? L::QD_STAGE : L::TILE;  // bytes between stages
            constexpr uint32_t QBOX = L::QD_ROWS * 128;
            const uint64_t kd = smem_desc_sw128(sK, 16, 1024), vd = smem_desc_sw128(sV, 16, 1024);
            const uint64_t qd0 = smem_desc_sw128(sQ, 16, 1024), qd1 = smem_desc_sw128(sQ + QS, 16, 1024);
            const uint64_t dd0 = smem_desc_sw128(sDO, 16, 1024), dd1 = smem_desc_sw128(sDO + QS, 16, 1024);
            const uint64_t qm0 = smem_desc_sw128(sQ, QBOX, 1024), qm1 = smem_desc_sw128(sQ + QS, QBOX, 1024);
            const uint64_t dm0 = smem_desc_sw128(sDO, QBOX, 1024), dm1 = smem_desc_sw128(sDO + QS, QBOX, 1024);
            auto stage_of = [&](int u) { return L::QD_HALF ? u % L::QD_STAGES : (u >> 1) & 1; };
            auto hoff_of = [&](int u) {
                return L::QD_HALF ? 0u : static_cast<uint32_t>(((u & 1) * 64 * 128) >> 4);
            };
            // Half step u: query tile u >> 1, queries 64 (u & 1) .. +63 (64 rows = 8 KB into
            // each swizzled box of the stage), TMEM buffer u & 1.
            auto issue_sdp = [&](int u) {
                const int hb = u & 1, s = stage_of(u);
                const uint32_t tb = tmem + hb * 128;
                const uint64_t qb = (s ? qd1 : qd0) + hoff_of(u);
                const uint64_t db = (s ? dd1 : dd0) + hoff_of(u);
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * (BT * 128) + (kk & 3) * 32) >> 4;
                    const uint32_t offq = ((kk >> 2) * QBOX + (kk & 3) * 32) >> 4;
                    mma_bf16_ss(tb, kd + off, qb + offq, idesc_s, kk > 0 ? 1u : 0u);
                }
                if (DO_DK) {
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk) {
                        const uint32_t off = ((kk >> 2) * (BT * 128) + (kk & 3) * 32) >> 4;
                        const uint32_t offq = ((kk >> 2) * QBOX + (kk & 3) * 32) >> 4;
                        mma_bf16_ss(tb + 64, vd + off, db + offq, idesc_s, kk > 0 ? 1u : 0u);
                    }
                }
                mma_commit(bar(D_SDP_FULL + hb));
            };
            // dV += P^T dO(half), dK += G^T Q(half): A from TMEM (16 queries = 8 columns per
            // k-step), B the (query x head_dim) rows read MN-major
            auto issue_acc = [&](int u) {
                const int hb = u & 1, s = stage_of(u);
                const uint32_t tb = tmem + hb * 128;
                const uint64_t db = (s ? dm1 : dm0) + hoff_of(u);
                const uint64_t qb = (s ? qm1 : qm0) + hoff_of(u);
                if (DO_DV) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(tDV, tb + kk * 8, db + ((kk * 16 * 128) >> 4), idesc_acc,
                                    (u > 0 || kk > 0) ? 1u : 0u);
                }
                if (DO_DK) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16_ts(tDK, tb + 64 + kk * 8, qb + ((kk * 16 * 128) >> 4), idesc_acc,
                                    (u > 0 || kk > 0) ? 1u : 0u);
                }
                if (L::QD_HALF || hb == 1) mma_commit(bar(D_QD_EMPTY + s));  // the stage is no longer read
            };
            const int n_u = 2 * nq;
            bool ok = mbar_wait(bar(D_KV_FULL), 0, abort_flag, status, TG_WHERE_MMA);
            for (int u = 0; ok && u < n_u; ++u) {
                if constexpr (L::QD_HALF && L::QD_STAGES == 1) {
                    // one stage: the products of half u - 1 read it and must go out (releasing it)
                    // before half u can land, so they precede S(u) here
                    if (u >= 1) {
                        ok = mbar_wait(bar(D_PG_FULL + ((u - 1) & 1)), ((u - 1) >> 1) & 1, abort_flag, status,
                                       TG_WHERE_MMA);
                        if (!ok) break;
                        tc_fence_after();
                        issue_acc(u - 1);
                    }
                    ok = mbar_wait(bar(D_QD_FULL), u & 1, abort_flag, status, TG_WHERE_MMA);
                    if (!ok) break;
                    tc_fence_after();
                    issue_sdp(u);
                } else {
                    if (L::QD_HALF || (u & 1) == 0) {
                        const int s = stage_of(u);
                        const int use = L::QD_HALF ? u / L::QD_STAGES : u >> 2;
                        ok = mbar_wait(bar(D_QD_FULL + s), use & 1, abort_flag, status, TG_WHERE_MMA);
                        if (!ok) break;
                    }
                    tc_fence_after();
                    issue_sdp(u);
                    if (u >= 1) {
                        ok = mbar_wait(bar(D_PG_FULL + ((u - 1) & 1)), ((u - 1) >> 1) & 1, abort_flag, status,
                                       TG_WHERE_MMA);
                        if (!ok) break;
                        tc_fence_after();
                        issue_acc(u - 1);
                    }
                }
            }
            if (ok) ok = mbar_wait(bar(D_PG_FULL + ((n_u - 1) & 1)), ((n_u - 1) >> 1) & 1, abort_flag, status,
                                   TG_WHERE_MMA);
            if (ok) {
                tc_fence_after();
                issue_acc(n_u - 1);
                mma_commit(bar(D_ACC_DONE));
            }
            mma_commit(bar(D_DRAIN));
            drain_wait_b(bar(D_DRAIN), 0, status);
        }
    } else {
        // ---------------------------------------------------------------- compute warps 0-7
        const int q4 = warp & 3, cs = warp >> 2;
        const int r = q4 * 32 + lane;  // key row of the tile == TMEM lane
        const int key_local = kt * BT + r;
        const bool valid_key = key_local < Mb;
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        // kgl = (sum_i beta_i gls_ij) / sm, the key's bias in units of the score, so that the
        // log2 of P is tt = fa (s + kgl) - lse log2(e) with the query's fa = sm log2(e) / tau
        const float kgl = valid_key ? gate_bias(gates, gate_gains(gates, h), seq0 + key_local) / sm_scale : 0.f;
        // this warp's own table of its 32 queries' factors (fa, -lse log2(e), 1/tau, -D'/tau),
        // [2 half steps][4][32]; only __syncwarp orders it
        float* wtab = reinterpret_cast<float*>(smem + L::OFF_TAB) + warp * (2 * 4 * 32);
        bool ok = true;
        float csum = 0.f;
        const int n_u = 2 * nq;
        // lane's query of half step u: query tile kt + (u >> 1), column 64 (u & 1) + 32 cs + lane;
        // its factors are loaded one half step ahead
        auto load_fac = [&](int u) {
            const int qrow = (kt + (u >> 1)) * BT + (u & 1) * 64 + cs * 32 + lane;
            return qrow < Mb ? __ldcg(fac + static_cast<size_t>(seq0 + qrow) * Hq + h)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        };
        // The dQ kernel's factor records are complete from here on.  This wait must stay
        // unconditional for every CTA with work: bwd_finish_kernel waits only for this grid
        // (its direct predecessor) and reads tileT, which the dQ kernel writes, so it is
        // ordered after the dQ kernel only through these waits (a non-empty batch always
        // has key tile 0 of some sequence with work).
        pdl_wait();
        float4 fnext = load_fac(0);
        for (int u = 0; u < n_u; ++u) {
            const int t = u >> 1, hb = u & 1, i = kt + t;
            float* tab = wtab + hb * 128;
            tab[0 * 32 + lane] = fnext.x;
            tab[1 * 32 + lane] = fnext.y;
            tab[2 * 32 + lane] = fnext.z;
            tab[3 * 32 + lane] = fnext.w;
            __syncwarp();
            if (u + 1 < n_u) fnext = load_fac(u + 1);
            const int c0 = hb * 64 + cs * 32;  // first query column of this warp
            const bool okw = mbar_wait_warp(bar(D_SDP_FULL + hb), t & 1, abort_flag, status, TG_WHERE_SOFTMAX);
            const uint32_t tb = tmem + lane_addr + hb * 128;
            float sx[32], dpx[32];
            if (okw) {
                tc_fence_after();
                tmem_ld32(tb + cs * 32, sx);
                if (DO_DK) tmem_ld32(tb + 64 + cs * 32, dpx);
                tmem_wait_ld();
            }
            if (!DO_DK) {
#pragma unroll
                for (int x = 0; x < 32; ++x) dpx[x] = 0.f;  // (not used: the dV pass forms no G)
            }
            // both warps of the row group have read their columns (the P^T / G^T stores
            // below overwrite some of the partner's); an abort is decided by the pair
            if (pair_red_or(2 + q4, !okw)) {
                ok = false;
                break;
            }
            // columns c0 + k with lo <= c0 + k < col_lim are live: inside the sequence and, on
            // the diagonal tile, not before the key
            const int col_lim = min(BT, Mb - i * BT);
            const int lo = (i == kt) ? r : 0;
            const int a = lo - c0, e = col_lim - c0;
            const uint32_t live = (a >= 32 || e <= 0 || a >= e)
                                      ? 0u
                                      : ((e >= 32 ? 0xFFFFFFFFu : ((1u << e) - 1u)) &
                                         (a <= 0 ? 0xFFFFFFFFu : ~((1u << a) - 1u)));
            uint32_t pp[16], gg[16];
#pragma unroll
            for (int k4 = 0; k4 < 32; k4 += 4) {
                const float4 fa4 = *reinterpret_cast<const float4*>(tab + 0 * 32 + k4);
                const float4 fl4 = *reinterpret_cast<const float4*>(tab + 1 * 32 + k4);
                const float4 fi4 = *reinterpret_cast<const float4*>(tab + 2 * 32 + k4);
                const float4 fd4 = *reinterpret_cast<const float4*>(tab + 3 * 32 + k4);
                const float fav[4] = {fa4.x, fa4.y, fa4.z, fa4.w}, flv[4] = {fl4.x, fl4.y, fl4.z, fl4.w};
                const float fiv[4] = {fi4.x, fi4.y, fi4.z, fi4.w}, fdv[4] = {fd4.x, fd4.y, fd4.z, fd4.w};
                float pv[4], gv[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int k = k4 + x;
                    const float tt = fmaf(fav[x], sx[k] + kgl, flv[x]);
                    const float p = (live >> k) & 1u ? ex2_approx(tt) : 0.f;
                    const float G = DO_DK ? p * fmaf(fiv[x], dpx[k], fdv[x]) : 0.f;
                    if (DO_DK) csum += G;
                    pv[x] = p;
                    gv[x] = G;
                }
                pp[k4 / 2] = pack2_bf16(pv[0], pv[1]);
                pp[k4 / 2 + 1] = pack2_bf16(pv[2], pv[3]);
                gg[k4 / 2] = pack2_bf16(gv[0], gv[1]);
                gg[k4 / 2 + 1] = pack2_bf16(gv[2], gv[3]);
            }
            if (DO_DV) tmem_st16u(tb + cs * 16, pp);       // P^T of these 32 queries over S^T
            if (DO_DK) tmem_st16u(tb + 64 + cs * 16, gg);  // G^T over dP^T
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(D_PG_FULL + hb));
        }
        // the second query half's key sums join the first's (all eight warps, abort or not)
        float* xch = reinterpret_cast<float*>(smem + L::OFF_XCH);
        if (cs == 1) xch[r] = csum;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (DO_DK && cs == 0 && ok && valid_key) colsum[static_cast<size_t>(seq0 + key_local) * Hq + h] = csum + xch[r];
        // ---------------------------------------------------------------- epilogue
        if (ok) ok = mbar_wait_warp(bar(D_ACC_DONE), 0, abort_flag, status, TG_WHERE_SOFTMAX);
        epi_ok = ok;
        if (PASS == 0 && cl > 1) {
            // heads 1 .. cl-1 of the group: this head's fp32 dV and dK into the exchange area
            // (the Q/dO stages, idle now), [dV|dK][HD/4 column quads][128 rows] float4s
            if (ok && hh != 0) {
                tc_fence_after();
                float4* xa = reinterpret_cast<float4*>(smem + L::OFF_Q);
#pragma unroll 1
                for (int which = 0; which < 2; ++which) {
#pragma unroll
                    for (int ch = 0; ch < HD / 64; ++ch) {
                        float o[32];
                        tmem_ld32((which ? tDK : tDV) + cs * (HD / 2) + lane_addr + ch * 32, o);
                        tmem_wait_ld();
                        const int c4 = (cs * (HD / 2) + ch * 32) / 4;
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            xa[(which * (HD / 4) + c4 + q) * BT + r] =
                                make_float4(o[q * 4], o[q * 4 + 1], o[q * 4 + 2], o[q * 4 + 3]);
                    }
                }
            }
        } else if (ok && part_k) {
            // partials of this head: [head in group][row][KV head][d] fp32, unscaled; warp cs
            // writes head_dim columns cs HD/2 .. + HD/2 - 1 of its rows
            tc_fence_after();
            const size_t row = ((static_cast<size_t>(hh) * M_total + seq0 + key_local) * Hkv + hk) * HD + cs * (HD / 2);
#pragma unroll 1
            for (int which = DO_DV ? 0 : 1; which < (DO_DK ? 2 : 1); ++which) {
                const uint32_t src = (which ? tDK : tDV) + cs * (HD / 2);
                float* dst = (which ? part_k : part_v) + row;
#pragma unroll
                for (int ch = 0; ch < HD / 64; ++ch) {
                    float o[32];
                    tmem_ld32(src + lane_addr + ch * 32, o);
                    tmem_wait_ld();
                    if (valid_key) {
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<float4*>(dst + ch * 32 + q * 4) =
                                make_float4(o[q * 4], o[q * 4 + 1], o[q * 4 + 2], o[q * 4 + 3]);
                    }
                }
            }
        } else if (ok) {
            tc_fence_after();
            const size_t row = (static_cast<size_t>(seq0 + key_local) * Hkv + hk) * HD + cs * (HD / 2);
#pragma unroll 1
            for (int which = DO_DV ? 0 : 1; which < (DO_DK ? 2 : 1); ++which) {
                const uint32_t src = (which ? tDK : tDV) + cs * (HD / 2);
                const float scale = which ? sm_scale : 1.0f;
                uint16_t* dst = (which ? dk : dv) + row;
#pragma unroll
                for (int ch = 0; ch < HD / 64; ++ch) {
                    float o[32];
                    tmem_ld32(src + lane_addr + ch * 32, o);
                    tmem_wait_ld();
                    if (valid_key) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 w;
                            w.x = pack2_bf16(o[q * 8 + 0] * scale, o[q * 8 + 1] * scale);
                            w.y = pack2_bf16(o[q * 8 + 2] * scale, o[q * 8 + 3] * scale);
                            w.z = pack2_bf16(o[q * 8 + 4] * scale, o[q * 8 + 5] * scale);
                            w.w = pack2_bf16(o[q * 8 + 6] * scale, o[q * 8 + 7] * scale);
                            *reinterpret_cast<uint4*>(dst + ch * 32 + q * 8) = w;
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (PASS == 0 && cl > 1) {
        // every thread of the cluster, abort or not
        cluster_sync_all();  // the other heads' copies are in their shared memory
        if (hh == 0 && warp < 8 && epi_ok) {
            // rank 0: dK = sm (dK_0 + dK_1 + ...), dV = dV_0 + dV_1 + ... in head order, to bf16
            tc_fence_after();
            const int q4 = warp & 3, cs = warp >> 2;
            const int r = q4 * 32 + lane;
            const int key_local = kt * BT + r;
            const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
            const uint32_t xa_local = sbase + L::OFF_Q;
            const size_t row = (static_cast<size_t>(seq0 + key_local) * Hkv + hk) * HD + cs * (HD / 2);
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                const float scale = which ? sm_scale : 1.0f;
                uint16_t* dst = (which ? dk : dv) + row;
#pragma unroll 1
                for (int ch = 0; ch < HD / 64; ++ch) {
                    float o[32];
                    tmem_ld32((which ? tDK : tDV) + cs * (HD / 2) + lane_addr + ch * 32, o);
                    tmem_wait_ld();
                    const int c4 = (cs * (HD / 2) + ch * 32) / 4;
                    for (int rk = 1; rk < cl; ++rk) {
                        const uint32_t base = mapa_shared(xa_local, static_cast<uint32_t>(rk));
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 v = ld_dsmem_f4(base + static_cast<uint32_t>(((which * (HD / 4) + c4 + q) * BT + r) * 16));
                            o[q * 4] += v.x;
                            o[q * 4 + 1] += v.y;
                            o[q * 4 + 2] += v.z;
                            o[q * 4 + 3] += v.w;
                        }
                    }
                    if (key_local < Mb) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint4 w;
                            w.x = pack2_bf16(o[q * 8 + 0] * scale, o[q * 8 + 1] * scale);
                            w.y = pack2_bf16(o[q * 8 + 2] * scale, o[q * 8 + 3] * scale);
                            w.z = pack2_bf16(o[q * 8 + 4] * scale, o[q * 8 + 5] * scale);
                            w.w = pack2_bf16(o[q * 8 + 6] * scale, o[q * 8 + 7] * scale);
                            *reinterpret_cast<uint4*>(dst + ch * 32 + q * 8) = w;
                        }
                    }
                }
            }
        }
        cluster_sync_all();  // rank 0 has read the other heads' shared memory
    }
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// dQ and the per-query sums: one CTA per (query head, 128-query tile, sequence),
// heaviest causal tiles first.
//
// 320 threads: warps 0-7 compute (warps w and w + 4 share query rows 32 w .. + 31,
// the TMEM lanes of that quarter, and split each half tile's keys), warp 8 TMA
// producer (Q and dO once, K/V tiles through a two-stage ring), warp 9 MMA issuer.
// TMEM: two (S | dP) buffers of half a KV tile (64 keys) and dQ.  The issuer puts
// out S and dP of one half while the compute warps turn the other half into G,
// then accumulates dQ += G K from TMEM.  The compute warps rebuild P from the
// log-sum-exp, form tau G = P (dP - D) (1/tau scales dQ's rows at the end), store
// it as bf16 over the first 32 columns of the half's S and sum, along their own
// row, dl l (for dtau).
template <int HD>
struct DqSmem {
    // head_dim 256: K and V stream as single-buffered half tiles (64 keys), so that they fit
    // beside the resident Q and dO; otherwise whole tiles in two stages
    static constexpr bool KV_HALF = HD > 128;
    static constexpr int TILE = BT * HD * 2;
    static constexpr int KV_ROWS = KV_HALF ? 64 : BT;
    static constexpr int KV_STAGE = KV_ROWS * HD * 2;
    static constexpr int KV_STAGES = KV_HALF ? 1 : 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_DO = OFF_Q + TILE;
    static constexpr int OFF_K = OFF_DO + TILE;                     // [KV_STAGES]
    static constexpr int OFF_V = OFF_K + KV_STAGES * KV_STAGE;      // [KV_STAGES]
    static constexpr int OFF_GLS = OFF_V + KV_STAGES * KV_STAGE;    // [8 warps][2][BT] fp32, a private copy per warp
    static constexpr int OFF_XCH = OFF_GLS + 8 * 2 * BT * 4;  // [6][BT] fp32: row sums [0..3], D halves [4..5]
    static constexpr int OFF_BAR = OFF_XCH + 6 * BT * 4;
    static constexpr int NUM_BARS = 16;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;  // tmem slot, abort flag, then 8 fp32
    static constexpr int BYTES = OFF_MISC + 16 + 32;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(ALLOC <= 227 * 1024, "shared memory");
    static_assert(2 * BT + HD <= 512, "TMEM columns");
};

enum : int {
    Q_QD_FULL = 0, Q_K_FULL = 1, Q_K_EMPTY = 3, Q_V_FULL = 5, Q_V_EMPTY = 7, Q_SDP_FULL = 9, Q_G_FULL = 11,
    Q_DQ_DONE = 13, Q_DRAIN = 14
};

constexpr int DQ_THREADS = 320;  // warps 0-7 compute, 8 TMA producer, 9 MMA issuer

template <int HD>
__global__ void __launch_bounds__(DQ_THREADS, 1)
gated_attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const int32_t* __restrict__ cu_kept, const int32_t* __restrict__ pos,
                         const int32_t* __restrict__ rank, const GateSet gates,
                         const float* __restrict__ c, const float* __restrict__ lse,
                         const uint16_t* __restrict__ out_fwd, float4* __restrict__ fac, float sm_scale, int Hq,
                         int Hkv, int n_qt_max, uint16_t* __restrict__ dq, float* __restrict__ tileT,
                         int* __restrict__ status) {
    using L = DqSmem<HD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int h = blockIdx.x;
    const int qt = n_qt_max - 1 - static_cast<int>(blockIdx.y);
    const int b = blockIdx.z;
    pdl_wait();  // global memory is read only from here on
    pdl_trigger();
    const int seq0 = cu_kept[b];
    const int Mb = cu_kept[b + 1] - seq0;
    if (qt * BT >= Mb) return;
    const int n_kv = qt + 1;  // the diagonal tile is the last one
    const int hk = h / (Hq / Hkv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + L::OFF_Q, sDO = sbase + L::OFF_DO, sK = sbase + L::OFF_K, sV = sbase + L::OFF_V;
    auto bar = [&](int i) { return sbase + L::OFF_BAR + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar(Q_QD_FULL), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(Q_K_FULL + s), 1);
            mbar_init(bar(Q_K_EMPTY + s), 1);
            mbar_init(bar(Q_V_FULL + s), 1);
            mbar_init(bar(Q_V_EMPTY + s), 1);
        }
        for (int hb = 0; hb < 2; ++hb) {
            mbar_init(bar(Q_SDP_FULL + hb), 1);
            mbar_init(bar(Q_G_FULL + hb), 256);  // every thread of the eight compute warps
        }
        mbar_init(bar(Q_DQ_DONE), 1);
        mbar_init(bar(Q_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // two half-tile buffers: half hb of a KV tile (keys 64 hb .. 64 hb + 63) keeps S at
    // columns [128 hb, +64) and dP at [128 hb + 64, +64); dQ follows
    const uint32_t tDQ = tmem + 2 * BT;

    if (warp == 8) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            prefetch_tmap(&tmDO);
            mbar_expect_tx(bar(Q_QD_FULL), 2 * L::TILE);
#pragma unroll
            for (int hf = 0; hf < HD / 64; ++hf) {
                tma_load_2d(sQ + hf * BT * 128, &tmQ, h * HD + hf * 64, seq0 + qt * BT, bar(Q_QD_FULL));
                tma_load_2d(sDO + hf * BT * 128, &tmDO, h * HD + hf * 64, seq0 + qt * BT, bar(Q_QD_FULL));
            }
            int k_issued[2] = {0, 0}, v_issued[2] = {0, 0};
            if constexpr (L::KV_HALF) {
                // one half tile (64 keys) per step u, one stage: the next half's K loads once the
                // previous half's dQ product has read K, its V once that half's dP has read V
                for (int u = 0; u < 2 * n_kv; ++u) {
                    if (u >= 1 && !mbar_wait(bar(Q_K_EMPTY), (u - 1) & 1, abort_flag, status, TG_WHERE_PRODUCER))
                        break;
                    mbar_expect_tx(bar(Q_K_FULL), L::KV_STAGE);
#pragma unroll
                    for (int hf = 0; hf < HD / 64; ++hf)
                        tma_load_2d(sK + hf * 64 * 128, &tmK, hk * HD + hf * 64, seq0 + u * 64, bar(Q_K_FULL));
                    ++k_issued[0];
                    if (u >= 1 && !mbar_wait(bar(Q_V_EMPTY), (u - 1) & 1, abort_flag, status, TG_WHERE_PRODUCER))
                        break;
                    mbar_expect_tx(bar(Q_V_FULL), L::KV_STAGE);
#pragma unroll
                    for (int hf = 0; hf < HD / 64; ++hf)
                        tma_load_2d(sV + hf * 64 * 128, &tmV, hk * HD + hf * 64, seq0 + u * 64, bar(Q_V_FULL));
                    ++v_issued[0];
                }
            } else {
                for (int j = 0; j < n_kv; ++j) {
                    const int s = j & 1;
                    if (j >= 2 && !mbar_wait(bar(Q_K_EMPTY + s), ((j - 2) >> 1) & 1, abort_flag, status,
                                             TG_WHERE_PRODUCER))
                        break;
                    mbar_expect_tx(bar(Q_K_FULL + s), L::TILE);
#pragma unroll
                    for (int hf = 0; hf < HD / 64; ++hf)
                        tma_load_2d(sK + s * L::TILE + hf * BT * 128, &tmK, hk * HD + hf * 64, seq0 + j * BT,
                                    bar(Q_K_FULL + s));
                    ++k_issued[s];
                    if (j >= 2 && !mbar_wait(bar(Q_V_EMPTY + s), ((j - 2) >> 1) & 1, abort_flag, status,
                                             TG_WHERE_PRODUCER))
                        break;
                    mbar_expect_tx(bar(Q_V_FULL + s), L::TILE);
#pragma unroll
                    for (int hf = 0; hf < HD / 64; ++hf)
                        tma_load_2d(sV + s * L::TILE + hf * BT * 128, &tmV, hk * HD + hf * 64, seq0 + j * BT,
                                    bar(Q_V_FULL + s));
                    ++v_issued[s];
                }
            }
            if (*abort_flag) {
                drain_wait_b(bar(Q_QD_FULL), 0, status);
                for (int s = 0; s < 2; ++s) {
                    if (k_issued[s]) drain_wait_b(bar(Q_K_FULL + s), (k_issued[s] - 1) & 1, status);
                    if (v_issued[s]) drain_wait_b(bar(Q_V_FULL + s), (v_issued[s] - 1) & 1, status);
                }
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(BT, 64, false);
            constexpr uint32_t idesc_acc = idesc_bf16_f32(BT, HD, true);
            // Half step u: KV tile u >> 1, keys 64 (u & 1) .. +63 (64 rows = 8 KB into each
            // swizzled box), TMEM buffer u & 1.  S(u) and dP(u) go out before dQ(u - 1), so the
            // tensor core computes half u while the compute warps turn half u - 1 into G; the
            // buffer S(u) overwrites last held G(u - 2), which dQ(u - 2) -- issued earlier by this
            // thread, so executed earlier -- has read.
            // Descriptors built once, as in the dK/dV kernel.
            const uint64_t qd = smem_desc_sw128(sQ, 16, 1024), dd = smem_desc_sw128(sDO, 16, 1024);
            const uint64_t kd0 = smem_desc_sw128(sK, 16, 1024), kd1 = smem_desc_sw128(sK + L::KV_STAGE, 16, 1024);
            const uint64_t vd0 = smem_desc_sw128(sV, 16, 1024), vd1 = smem_desc_sw128(sV + L::KV_STAGE, 16, 1024);
            const uint64_t km0 = smem_desc_sw128(sK, L::KV_ROWS * 128, 1024),
                           km1 = smem_desc_sw128(sK + L::KV_STAGE, L::KV_ROWS * 128, 1024);
            // (with half-tile stages the K/V stage holds only half u, so there is no offset for hb,
            // and the K/V rows' 64-column boxes are KV_ROWS * 128 bytes apart instead of BT * 128)
            auto issue_sdp = [&](int u) {
                const int hb = u & 1, s = L::KV_HALF ? 0 : (u >> 1) & 1;
                const uint32_t tb = tmem + hb * 128;
                const uint32_t hoff = L::KV_HALF ? 0u : static_cast<uint32_t>((hb * 64 * 128) >> 4);
                const uint64_t kb = (s ? kd1 : kd0) + hoff;
                const uint64_t vb = (s ? vd1 : vd0) + hoff;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * (BT * 128) + (kk & 3) * 32) >> 4;
                    const uint32_t offk = ((kk >> 2) * (L::KV_ROWS * 128) + (kk & 3) * 32) >> 4;
                    mma_bf16_ss(tb, qd + off, kb + offk, idesc_s, kk > 0 ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * (BT * 128) + (kk & 3) * 32) >> 4;
                    const uint32_t offk = ((kk >> 2) * (L::KV_ROWS * 128) + (kk & 3) * 32) >> 4;
                    mma_bf16_ss(tb + 64, dd + off, vb + offk, idesc_s, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar(Q_SDP_FULL + hb));
                if (L::KV_HALF || hb == 1) mma_commit(bar(Q_V_EMPTY + s));  // V of this stage is no longer read
            };
            // dQ += G(u) K(half of u): A from TMEM (16 keys = 8 columns per k-step), B the K rows MN-major
            auto issue_dq = [&](int u) {
                const int hb = u & 1, s = L::KV_HALF ? 0 : (u >> 1) & 1;
                const uint32_t hoff = L::KV_HALF ? 0u : static_cast<uint32_t>((hb * 64 * 128) >> 4);
                const uint64_t kb = (s ? km1 : km0) + hoff;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16_ts(tDQ, tmem + hb * 128 + kk * 8, kb + ((kk * 16 * 128) >> 4), idesc_acc,
                                (u > 0 || kk > 0) ? 1u : 0u);
                if (L::KV_HALF || hb == 1) mma_commit(bar(Q_K_EMPTY + s));  // K of this stage is no longer read
            };
            const int n_u = 2 * n_kv;
            bool ok = mbar_wait(bar(Q_QD_FULL), 0, abort_flag, status, TG_WHERE_MMA);
            for (int u = 0; ok && u < n_u; ++u) {
                const int j = u >> 1, s = j & 1;
                if constexpr (L::KV_HALF) {
                    // one stage: dQ(u - 1) reads K(u - 1) and must go out (releasing the stage)
                    // before K(u) can land, so it precedes S(u) here
                    if (u >= 1) {
                        ok = mbar_wait(bar(Q_G_FULL + ((u - 1) & 1)), ((u - 1) >> 1) & 1, abort_flag, status,
                                       TG_WHERE_MMA);
                        if (!ok) break;
                        tc_fence_after();
                        issue_dq(u - 1);
                    }
                    ok = mbar_wait(bar(Q_K_FULL), u & 1, abort_flag, status, TG_WHERE_MMA);
                    if (ok) ok = mbar_wait(bar(Q_V_FULL), u & 1, abort_flag, status, TG_WHERE_MMA);
                    if (!ok) break;
                    tc_fence_after();
                    issue_sdp(u);
                } else {
                    if ((u & 1) == 0) {
                        ok = mbar_wait(bar(Q_K_FULL + s), (j >> 1) & 1, abort_flag, status, TG_WHERE_MMA);
                        if (ok) ok = mbar_wait(bar(Q_V_FULL + s), (j >> 1) & 1, abort_flag, status, TG_WHERE_MMA);
                        if (!ok) break;
                    }
                    tc_fence_after();
                    issue_sdp(u);
                    if (u >= 1) {
                        ok = mbar_wait(bar(Q_G_FULL + ((u - 1) & 1)), ((u - 1) >> 1) & 1, abort_flag, status,
                                       TG_WHERE_MMA);
                        if (!ok) break;
                        tc_fence_after();
                        issue_dq(u - 1);
                    }
                }
            }
            if (ok) ok = mbar_wait(bar(Q_G_FULL + ((n_u - 1) & 1)), ((n_u - 1) >> 1) & 1, abort_flag, status,
                                   TG_WHERE_MMA);
            if (ok) {
                tc_fence_after();
                issue_dq(n_u - 1);
                mma_commit(bar(Q_DQ_DONE));
            }
            mma_commit(bar(Q_DRAIN));
            drain_wait_b(bar(Q_DRAIN), 0, status);
        }
    } else {
        // ---------------------------------------------------------------- compute warps 0-7
        // Warp w owns query rows 32 (w & 3) .. + 31 (TMEM lanes) and the keys
        // 32 (w >> 2) .. + 31 of each 64-key half step; the two warps of a row group meet
        // at a 64-thread reducing barrier once per half step (each stores G over S columns
        // the other reads) and combine their row sums once at the end.
        const int q4 = warp & 3, cs = warp >> 2;
        const int r = q4 * 32 + lane;  // query row of the tile == TMEM lane
        const int q_local = qt * BT + r;
        const bool valid_row = q_local < Mb;
        const int qg = seq0 + q_local;
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        // D = dout . out of this row, each warp of the row group taking half of head_dim:
        // out (the forward's output) is read from global memory while Q and dout arrive,
        // dout from the staged tile (128-byte swizzled boxes of 64 columns)
        constexpr int NCH = HD / 16;  // 8-column chunks per warp
        uint4 ov[NCH];
        if (valid_row) {
            const uint16_t* orow = out_fwd + (static_cast<size_t>(qg) * Hq + h) * HD + cs * (HD / 2);
#pragma unroll
            for (int m = 0; m < NCH; ++m) ov[m] = __ldcg(reinterpret_cast<const uint4*>(orow + m * 8));
        }
        float fa = 0.f, fb = 0.f, fl = 0.f, fi = 0.f, lr = 0.f;
        if (valid_row) {
            lr = logf(static_cast<float>(__ldcg(pos + qg)) / static_cast<float>(__ldcg(rank + qg)));
            fi = 1.0f / (1.0f + c[h] * lr);
            fa = sm_scale * LOG2E_B * fi;
            fb = LOG2E_B * fi;  // multiplies the key's whole bias sum_i beta_i gls_ij
            fl = __ldcg(lse + static_cast<size_t>(qg) * Hq + h) * LOG2E_B;
        }
        float* xch = reinterpret_cast<float*>(smem + L::OFF_XCH);
        bool ok = mbar_wait_warp(bar(Q_QD_FULL), 0, abort_flag, status, TG_WHERE_SOFTMAX);
        {
            float acc = 0.f;
            if (ok && valid_row) {
#pragma unroll
                for (int m = 0; m < NCH; ++m) {
                    const int col = cs * (HD / 2) + m * 8;  // first head_dim column of the chunk
                    const int hf = col / 64, cch = (col % 64) / 8;
                    const uint4 dv = *reinterpret_cast<const uint4*>(smem + L::OFF_DO + hf * (BT * 128) + r * 128 +
                                                                     ((cch ^ (r & 7)) << 4));
                    const uint32_t a[4] = {dv.x, dv.y, dv.z, dv.w}, o4[4] = {ov[m].x, ov[m].y, ov[m].z, ov[m].w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        acc = fmaf(__uint_as_float(a[e] << 16), __uint_as_float(o4[e] << 16), acc);
                        acc = fmaf(__uint_as_float(a[e] & 0xFFFF0000u), __uint_as_float(o4[e] & 0xFFFF0000u), acc);
                    }
                }
            }
            xch[(4 + cs) * BT + r] = acc;
        }
        ok = !pair_red_or(2 + q4, !ok);
        const float fd = xch[4 * BT + r] + xch[5 * BT + r];  // the same order in both warps
        float* wgls = reinterpret_cast<float*>(smem + L::OFF_GLS) + warp * (2 * BT);
        // Row sums for dtau, formed with the row's exact D' = sum_j P dP (the D above comes
        // from the bf16 output; dtau = -sum_j dl l / tau cancels to a small number and would
        // amplify its rounding):  sum_j dl x = sum P dP x - D' sum P x.
        float aPdPt = 0.f, aPt = 0.f, aPdP = 0.f, aP = 0.f;
        // the bias sum_i beta_i gls_ij of the next KV tile's keys is loaded one tile ahead (its
        // latency hides behind a tile of work)
        const GateGains gw = gate_gains(gates, h);
        float gnext[BT / 32];
#pragma unroll
        for (int e = 0; e < BT / 32; ++e) gnext[e] = e * 32 + lane < Mb ? gate_bias(gates, gw, seq0 + e * 32 + lane) : 0.f;
        for (int j = 0; ok && j < n_kv; ++j) {
            const int s = j & 1;
            // the tile's gls into this warp's own copy (only __syncwarp orders it)
#pragma unroll
            for (int e = 0; e < BT / 32; ++e) wgls[s * BT + e * 32 + lane] = gnext[e];
            __syncwarp();
            if (j + 1 < n_kv) {
#pragma unroll
                for (int e = 0; e < BT / 32; ++e) {
                    const int key_local = (j + 1) * BT + e * 32 + lane;
                    gnext[e] = key_local < Mb ? gate_bias(gates, gw, seq0 + key_local) : 0.f;
                }
            }
            const bool diag = (j == n_kv - 1);
            const int lim = q_local - j * BT;  // on the diagonal tile, columns > lim are future keys
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                const int c0 = half * 64 + cs * 32;  // first key column of this warp
                const bool okw = mbar_wait_warp(bar(Q_SDP_FULL + half), j & 1, abort_flag, status, TG_WHERE_SOFTMAX);
                const uint32_t tb = tmem + lane_addr + half * 128;
                float sx[32], dpx[32];
                if (okw) {
                    tc_fence_after();
                    tmem_ld32(tb + cs * 32, sx);
                    tmem_ld32(tb + 64 + cs * 32, dpx);
                    tmem_wait_ld();
                }
                // both warps of the row group have read their columns of S (the G stores below
                // overwrite some of the partner's); an abort is decided by the pair together
                if (pair_red_or(2 + q4, !okw)) {
                    ok = false;
                    break;
                }
                // live columns c0 + k: the row exists and, on the diagonal tile, c0 + k <= lim
                const int nlive = diag ? lim - c0 + 1 : 32;
                const uint32_t live = !valid_row || nlive <= 0 ? 0u : (nlive >= 32 ? 0xFFFFFFFFu : (1u << nlive) - 1u);
                const float* bl = wgls + s * BT + c0;
                uint32_t gg[16];
#pragma unroll
                for (int k4 = 0; k4 < 32; k4 += 4) {
                    const float4 g4 = *reinterpret_cast<const float4*>(bl + k4);
                    const float glv[4] = {g4.x, g4.y, g4.z, g4.w};
                    float gv[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const int k = k4 + x;
                        const float tt = fmaf(fa, sx[k], fmaf(fb, glv[x], -fl));
                        // masked and padded entries have p = 0 and finite tt: they add nothing
                        const float p = (live >> k) & 1u ? ex2_approx(tt) : 0.f;
                        const float pdp = p * dpx[k];
                        aPdPt = fmaf(pdp, tt, aPdPt);
                        aPt = fmaf(p, tt, aPt);
                        aPdP += pdp;
                        aP += p;
                        gv[x] = fmaf(-p, fd, pdp);  // G tau = P (dP - D); 1/tau is applied to dQ's rows
                    }
                    gg[k4 / 2] = pack2_bf16(gv[0], gv[1]);
                    gg[k4 / 2 + 1] = pack2_bf16(gv[2], gv[3]);
                }
                tmem_st16u(tb + cs * 16, gg);  // G of these 32 keys as bf16 pairs over S
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(Q_G_FULL + half));
            }
        }
        // ---------------------------------------------------------------- epilogue
        if (ok) ok = mbar_wait_warp(bar(Q_DQ_DONE), 0, abort_flag, status, TG_WHERE_SOFTMAX);
        if (ok) {
            tc_fence_after();
            const float rs = sm_scale * fi;
            uint16_t* dst = dq + (static_cast<size_t>(qg) * Hq + h) * HD + cs * (HD / 2);
#pragma unroll
            for (int ch = 0; ch < HD / 64; ++ch) {
                float o[32];
                tmem_ld32(tDQ + lane_addr + cs * (HD / 2) + ch * 32, o);
                tmem_wait_ld();
                if (valid_row) {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        uint4 w;
                        w.x = pack2_bf16(o[q8 * 8 + 0] * rs, o[q8 * 8 + 1] * rs);
                        w.y = pack2_bf16(o[q8 * 8 + 2] * rs, o[q8 * 8 + 3] * rs);
                        w.z = pack2_bf16(o[q8 * 8 + 4] * rs, o[q8 * 8 + 5] * rs);
                        w.w = pack2_bf16(o[q8 * 8 + 6] * rs, o[q8 * 8 + 7] * rs);
                        *reinterpret_cast<uint4*>(dst + ch * 32 + q8 * 8) = w;
                    }
                }
            }
        }
        // the second column half's row sums join the first's (all eight warps, abort or not)
        if (cs == 1) {
            xch[0 * BT + r] = aPdPt;
            xch[1 * BT + r] = aPt;
            xch[2 * BT + r] = aPdP;
            xch[3 * BT + r] = aP;
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        // this tile's terms of dc_h (sum_i ln(pos/rank) dtau), summed over its rows in a fixed
        // order and stored at the tile's first row
        float eT = 0.f;
        if (cs == 0) {
            aPdPt += xch[0 * BT + r];
            aPt += xch[1 * BT + r];
            aPdP += xch[2 * BT + r];
            aP += xch[3 * BT + r];
            if (ok && valid_row) {
                const float Dx = aPdP;
                // tt = l log2(e) - lse log2(e):  sum dl l = ln2 (sum dl tt + lse log2(e) sum dl)
                const float sum_dl_t = aPdPt - Dx * aPt + fl * (aPdP - Dx * aP);
                eT = lr * (-LN2_B * fi * sum_dl_t);
                // the row's factors for the dK/dV kernel, with the exact D'
                fac[static_cast<size_t>(qg) * Hq + h] = make_float4(fa, -fl, fi, -fi * Dx);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) eT += __shfl_xor_sync(0xffffffffu, eT, o);
        }
        float* red = reinterpret_cast<float*>(smem + L::OFF_MISC + 16);
        if (cs == 0 && lane == 0) red[q4] = eT;
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (threadIdx.x == 0 && ok) {
            const size_t slot = (static_cast<size_t>(seq0) + static_cast<size_t>(qt) * BT) * Hq + h;
            tileT[slot] = (red[0] + red[1]) + (red[2] + red[3]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// dK = sm * sum_h part_k[h], dV = sum_h part_v[h] over the query heads of each group, in
// head order, to bf16 (8 consecutive elements per thread).
__global__ void __launch_bounds__(256)
bwd_kv_reduce_kernel(const float* __restrict__ part_k, const float* __restrict__ part_v, int grp, int64_t n,
                     float sm_scale, uint16_t* __restrict__ dk, uint16_t* __restrict__ dv) {
    pdl_wait();
    pdl_trigger();
    for (int64_t e = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 8; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x * 8) {
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
            const float* src = which ? part_v : part_k;
            float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int q = 0; q < grp; ++q) {
                const float4 x = __ldcg(reinterpret_cast<const float4*>(src + q * n + e));
                const float4 y = __ldcg(reinterpret_cast<const float4*>(src + q * n + e + 4));
                a[0] += x.x; a[1] += x.y; a[2] += x.z; a[3] += x.w;
                a[4] += y.x; a[5] += y.y; a[6] += y.z; a[7] += y.w;
            }
            const float sc = which ? 1.0f : sm_scale;
            uint4 w;
            w.x = pack2_bf16(a[0] * sc, a[1] * sc);
            w.y = pack2_bf16(a[2] * sc, a[3] * sc);
            w.z = pack2_bf16(a[4] * sc, a[5] * sc);
            w.w = pack2_bf16(a[6] * sc, a[7] * sc);
            *reinterpret_cast<uint4*>((which ? dv : dk) + e) = w;
        }
    }
}

// ---------------------------------------------------------------------------
// The last step, one launch, for gates i < n:
//   blocks (i, h), i * Hq + h:  dg_ih = sigmoid(g_ih) sum_j gls_ij colsum[j, h]  (dbeta_ih
//                               = sum_qj G_qj gls_ij, by keys); the blocks of gate 0 also
//                               dc_h = sum_tiles tileT[., h]  (fixed order);
//   the other blocks, per key:  dgls_ij = sum_h softplus(g_ih) colsum[j, h] and
//                               d score_ij = dgls_ij (1 - exp(gls_ij)).
struct BwdGateOut {
    float* dgls[kMaxGates];
    float* dscore[kMaxGates];  // entries may be null
    float* dg[kMaxGates];
};

__global__ void __launch_bounds__(256)
bwd_finish_kernel(const float* __restrict__ colsum, const float* __restrict__ tileT, const GateSet gates,
                  const int32_t* __restrict__ cu_kept, int B, int64_t M, int Hq, const BwdGateOut go,
                  float* __restrict__ dc) {
    // Waits for the dK/dV grid (colsum).  tileT comes from the dQ kernel, one launch
    // earlier: it is complete because every dK/dV CTA with work waits for the dQ kernel
    // before it finishes, and a non-empty batch has at least one such CTA.
    pdl_wait();
    pdl_trigger();
    const int n = gates.n;
    if (static_cast<int>(blockIdx.x) < n * Hq) {
        const int gi = static_cast<int>(blockIdx.x) / Hq, h = static_cast<int>(blockIdx.x) % Hq;
        // (a select chain, not gates.gls[gi]: a run-time index into the parameter block would
        // copy it to local memory)
        const float* gls = gi == 0 ? gates.gls[0] : (gi == 1 ? gates.gls[1] : (gi == 2 ? gates.gls[2] : gates.gls[3]));
        const float* g = gi == 0 ? gates.g[0] : (gi == 1 ? gates.g[1] : (gi == 2 ? gates.g[2] : gates.g[3]));
        float* dg = gi == 0 ? go.dg[0] : (gi == 1 ? go.dg[1] : (gi == 2 ? go.dg[2] : go.dg[3]));
        float e = 0.f, t = 0.f;
        // thread x takes keys x, x + 256, ... and tiles x, x + 256, ... (running tile number)
        for (int64_t j = threadIdx.x; j < M; j += 256) e = fmaf(__ldcg(gls + j), __ldcg(colsum + j * Hq + h), e);
        if (gi == 0) {
            int k = 0;
            for (int b = 0; b < B; ++b) {
                const int s0 = cu_kept[b], n_qt = (cu_kept[b + 1] - s0 + BT - 1) / BT;
                for (int qt = 0; qt < n_qt; ++qt, ++k)
                    if ((k & 255) == static_cast<int>(threadIdx.x))
                        t += __ldcg(tileT + (static_cast<size_t>(s0) + static_cast<size_t>(qt) * BT) * Hq + h);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            e += __shfl_xor_sync(0xffffffffu, e, o);
            t += __shfl_xor_sync(0xffffffffu, t, o);
        }
        __shared__ float red[2][8];
        const int w = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) {
            red[0][w] = e;
            red[1][w] = t;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            const float se = ((red[0][0] + red[0][1]) + (red[0][2] + red[0][3])) +
                             ((red[0][4] + red[0][5]) + (red[0][6] + red[0][7]));
            const float st = ((red[1][0] + red[1][1]) + (red[1][2] + red[1][3])) +
                             ((red[1][4] + red[1][5]) + (red[1][6] + red[1][7]));
            dg[h] = se / (1.0f + expf(-g[h]));
            if (gi == 0) dc[h] = st;
        }
        return;
    }
    const int64_t nb = static_cast<int64_t>(gridDim.x) - n * Hq;
    for (int64_t j = static_cast<int64_t>(blockIdx.x - n * Hq) * blockDim.x + threadIdx.x; j < M;
         j += nb * blockDim.x) {
#pragma unroll 1
        for (int gi = 0; gi < n; ++gi) {
            const float* gls = gi == 0 ? gates.gls[0] : (gi == 1 ? gates.gls[1] : (gi == 2 ? gates.gls[2] : gates.gls[3]));
            const float* g = gi == 0 ? gates.g[0] : (gi == 1 ? gates.g[1] : (gi == 2 ? gates.g[2] : gates.g[3]));
            float* dgls = gi == 0 ? go.dgls[0] : (gi == 1 ? go.dgls[1] : (gi == 2 ? go.dgls[2] : go.dgls[3]));
            float* dscore =
                gi == 0 ? go.dscore[0] : (gi == 1 ? go.dscore[1] : (gi == 2 ? go.dscore[2] : go.dscore[3]));
            float acc = 0.f;
            for (int h = 0; h < Hq; ++h) acc = fmaf(softplus_b(g[h]), __ldcg(colsum + j * Hq + h), acc);
            dgls[j] = acc;
            if (dscore) dscore[j] = acc * -expm1f(__ldcg(gls + j));
        }
    }
}

// GQA groups of 2, 4 or 8 heads run their dK/dV CTAs as one cluster (portable sizes).
inline int bwd_cluster_size(int grp) { return grp == 2 || grp == 4 || grp == 8 ? grp : 0; }

template <int HD>
cudaError_t launch_bwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* out,
                       const uint16_t* dout, const float* lse, const int32_t* cu_kept, int B, int64_t M_total,
                       int max_M, int Hq, int Hkv, const int32_t* pos, const int32_t* rank, const GateSet& gates,
                       const float* c, float sm_scale, uint16_t* dq, uint16_t* dk, uint16_t* dv,
                       const BwdGateOut& gout, float* dc, void* ws, cudaStream_t st) {
    constexpr bool TWO_PASS = HD > 128;  // dV and dK in two launches (see DkvSmem)
    constexpr int P1 = TWO_PASS ? 1 : 0;
    static std::atomic<uint64_t> set_dkv{0}, set_dkv2{0}, set_dq{0};
    if (cudaError_t e = ensure_smem_limit(gated_attn_bwd_dkv_kernel<HD, P1>, DkvSmem<HD, P1>::ALLOC, set_dkv);
        e != cudaSuccess)
        return e;
    if constexpr (TWO_PASS) {
        if (cudaError_t e = ensure_smem_limit(gated_attn_bwd_dkv_kernel<HD, 2>, DkvSmem<HD, 2>::ALLOC, set_dkv2);
            e != cudaSuccess)
            return e;
    }
    if (cudaError_t e = ensure_smem_limit(gated_attn_bwd_dq_kernel<HD>, DqSmem<HD>::ALLOC, set_dq); e != cudaSuccess)
        return e;
    const size_t rows = static_cast<size_t>(M_total) * Hq;
    // every section starts on a 16-byte boundary (the partials are written as float4)
    const size_t rows4 = (rows + 3) & ~static_cast<size_t>(3);
    float4* fac = static_cast<float4*>(ws);  // per query row and head: fa, -lse log2(e), 1/tau, -D'/tau
    float* colsum = reinterpret_cast<float*>(fac + rows);
    float* tileT = colsum + rows4;  // per query tile, at its first row
    const int grp = Hq / Hkv;
    // the group's heads as one cluster (its exchange area holds a head's fp32 dV and dK only at
    // head_dim <= 128), else partials
    const int cl = TWO_PASS ? 0 : bwd_cluster_size(grp);
    const int64_t nkv = M_total * Hkv * HD;
    float* part_k = grp > 1 && cl == 0 ? tileT + rows4 : nullptr;  // [grp][M][Hkv][HD] each
    float* part_v = part_k ? part_k + grp * nkv : nullptr;
    // tensor maps: whole 128-row tiles, and (head_dim 256) 64-row half tiles for the rows
    // that stream: K/V in the dQ kernel, Q/dO in the dK/dV passes
    constexpr uint32_t HR = TWO_PASS ? 64 : BT;
    CUtensorMap tq, tk, tv, tdo, tq_s, tk_s, tv_s, tdo_s;
    auto enc = [&](CUtensorMap* m, const uint16_t* p, int H, uint32_t rows) {
        return encode_tmap_2d_bf16(m, p, static_cast<uint64_t>(H) * HD, static_cast<uint64_t>(M_total),
                                   static_cast<uint64_t>(H) * HD * 2, 64, rows);
    };
    if (!enc(&tq, q, Hq, BT) || !enc(&tdo, dout, Hq, BT) || !enc(&tk, k, Hkv, BT) || !enc(&tv, v, Hkv, BT) ||
        !enc(&tq_s, q, Hq, HR) || !enc(&tdo_s, dout, Hq, HR) || !enc(&tk_s, k, Hkv, HR) || !enc(&tv_s, v, Hkv, HR))
        return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int* status = device_status_ptr();
    const int n_t = (max_M + BT - 1) / BT;
    // dq first: it forms each row's D = dout . out for its own use and leaves the exact
    // D' = sum_j P dP for the dK/dV kernel
    cudaError_t e = launch_pdl(gated_attn_bwd_dq_kernel<HD>, dim3(Hq, n_t, B), dim3(DQ_THREADS),
                               static_cast<size_t>(DqSmem<HD>::ALLOC), st, tq, tk_s, tv_s, tdo, cu_kept, pos, rank,
                               gates, c, lse, out, fac, sm_scale, Hq, Hkv, n_t, dq, tileT, status);
    if (e != cudaSuccess) return e;
    if constexpr (TWO_PASS) {
        e = launch_pdl(gated_attn_bwd_dkv_kernel<HD, 1>, dim3(Hq, n_t, B), dim3(DKV_THREADS),
                       static_cast<size_t>(DkvSmem<HD, 1>::ALLOC), st, tq_s, tk, tv, tdo_s, cu_kept, gates,
                       static_cast<const float4*>(fac), sm_scale, Hq, Hkv, M_total, dk, dv, part_k, part_v, colsum,
                       status, 0);
        if (e == cudaSuccess)
            e = launch_pdl(gated_attn_bwd_dkv_kernel<HD, 2>, dim3(Hq, n_t, B), dim3(DKV_THREADS),
                           static_cast<size_t>(DkvSmem<HD, 2>::ALLOC), st, tq_s, tk, tv, tdo_s, cu_kept, gates,
                           static_cast<const float4*>(fac), sm_scale, Hq, Hkv, M_total, dk, dv, part_k, part_v,
                           colsum, status, 0);
    } else if (cl > 1)
        e = launch_pdl_cluster(gated_attn_bwd_dkv_kernel<HD>, dim3(Hq, n_t, B), dim3(DKV_THREADS),
                               static_cast<size_t>(DkvSmem<HD>::ALLOC), st, static_cast<unsigned>(cl), tq, tk, tv, tdo,
                               cu_kept, gates, static_cast<const float4*>(fac), sm_scale, Hq, Hkv, M_total, dk, dv,
                               part_k, part_v, colsum, status, cl);
    else
        e = launch_pdl(gated_attn_bwd_dkv_kernel<HD>, dim3(Hq, n_t, B), dim3(DKV_THREADS),
                       static_cast<size_t>(DkvSmem<HD>::ALLOC), st, tq, tk, tv, tdo, cu_kept, gates,
                       static_cast<const float4*>(fac), sm_scale, Hq, Hkv, M_total, dk, dv, part_k, part_v, colsum,
                       status, 0);
    if (e != cudaSuccess) return e;
    if (part_k) {
        const int64_t rb = (nkv / 8 + 255) / 256;
        e = launch_pdl(bwd_kv_reduce_kernel, dim3(static_cast<unsigned>(rb < sms * 8 ? rb : sms * 8)), dim3(256), 0, st,
                       static_cast<const float*>(part_k), static_cast<const float*>(part_v), grp, nkv, sm_scale, dk,
                       dv);
        if (e != cudaSuccess) return e;
    }
    const int64_t kb = (M_total + 255) / 256;
    const int key_blocks = static_cast<int>(kb < sms * 4 ? kb : sms * 4);
    return launch_pdl(bwd_finish_kernel, dim3(gates.n * Hq + key_blocks), dim3(256), 0, st,
                      static_cast<const float*>(colsum), static_cast<const float*>(tileT), gates, cu_kept, B, M_total,
                      Hq, gout, dc);
}

}  // namespace

size_t attention_backward_workspace_bytes(int64_t M_total, int Hq, int Hkv, int d) {
    // a float4 of factors, the key sum of G and a tile sum per row and head, each
    // section padded to 16 bytes
    const size_t mh = static_cast<size_t>(M_total) * static_cast<size_t>(Hq);
    const size_t rows = 4 * mh + 2 * ((mh + 3) & ~static_cast<size_t>(3));
    const int grp = Hkv > 0 ? Hq / Hkv : 1;
    // head_dim 256 always reduces the group's heads through partials
    const bool parts_needed = grp > 1 && (d > 128 || bwd_cluster_size(grp) == 0);
    const size_t parts = parts_needed ? static_cast<size_t>(2) * grp * static_cast<size_t>(M_total) * Hkv * d : 0;
    return (rows + parts) * sizeof(float);
}

cudaError_t launch_gated_attention_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                            const uint16_t* out, const uint16_t* dout, const float* lse,
                                            const int32_t* cu_kept, int B, int64_t M_total, int max_M, int Hq,
                                            int Hkv, int d, const int32_t* pos, const int32_t* rank,
                                            const GateSet& gates, const float* c, float sm_scale, uint16_t* dq,
                                            uint16_t* dk, uint16_t* dv, float* const* dgls, float* const* dscore,
                                            float* const* dg, float* dc, void* ws, cudaStream_t st) {
    if (gates.n < 1 || gates.n > kMaxGates) return cudaErrorInvalidValue;
    BwdGateOut go{};
    for (int i = 0; i < gates.n; ++i) {
        go.dgls[i] = dgls[i];
        go.dscore[i] = dscore ? dscore[i] : nullptr;
        go.dg[i] = dg[i];
    }
    if (d == 64)
        return launch_bwd<64>(q, k, v, out, dout, lse, cu_kept, B, M_total, max_M, Hq, Hkv, pos, rank, gates, c,
                              sm_scale, dq, dk, dv, go, dc, ws, st);
    if (d == 256)
        return launch_bwd<256>(q, k, v, out, dout, lse, cu_kept, B, M_total, max_M, Hq, Hkv, pos, rank, gates, c,
                               sm_scale, dq, dk, dv, go, dc, ws, st);
    return launch_bwd<128>(q, k, v, out, dout, lse, cu_kept, B, M_total, max_M, Hq, Hkv, pos, rank, gates, c,
                           sm_scale, dq, dk, dv, go, dc, ws, st);
}

}  // namespace tg
