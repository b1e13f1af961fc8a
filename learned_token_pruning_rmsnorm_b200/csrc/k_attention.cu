// Stage 4 of the gated prefill: token-gated causal GQA attention over the kept
// tokens (TokenGate AI summary, "Key Contributions" 2 and 3), on the sm_100
// tensor cores.
//
//   logit[q,j] = (q.k_j * sm_scale + softplus(g_h) * gls_j) / tau[q,h]
//   tau[q,h]   = 1 + c_h * ln(pos_q / rank_q)
//   o_q        = sum_j softmax_j(logit[q,:]) v_j     over kept j <= q
//
// One CTA per (query head, 128-query tile, sequence); heaviest causal tiles
// are launched first.  Warp roles (192 threads):
//   warp 4     TMA producer: the Q tile once, then K/V tiles of 128 keys
//              through a two-stage ring (128-byte swizzled boxes of 64 cols)
//   warp 5     MMA issuer (one thread): S_j = Q K_j^T into one of two TMEM
//              S buffers, then O += P_{j-1} V_{j-1} into the TMEM O accumulator
//              with P read from TMEM
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r).  It reads
//              S_j from TMEM, applies scale, gate bias and temperature in the
//              log2 domain with one FFMA per element, masks the causal
//              diagonal, keeps a running max that is only moved (and O only
//              rescaled in TMEM) when it grows by more than 2^8, writes P_j
//              as bf16 pairs over the first 64 columns of its S buffer, and
//              at the end normalises O and stores it.
// This kernel serves odd GQA groups and head_dim 256 (two heads of 256 would
// need 768 TMEM columns); tcgen05 operations of one thread execute in issue
// order, so S_{j+2} overwrites P_j only after PV_j has read it.
// The bias and temperature therefore cost one extra FFMA per score element
// on top of plain attention.

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <vector>

#include "tg_attn_util.cuh"

namespace tg {
namespace {

using namespace sm100;
using namespace attn;

constexpr int NUM_THREADS = 192;

template <int HD>
struct AttnSmem {
    // K and V tiles are double-buffered up to head_dim 128; at 256 one 64 KB tile of
    // each fits beside Q (the K tile of j+1 still loads during the softmax of j, and
    // the V tile of j+1 during S(j+1)).
    static constexpr int KV_STAGES = HD == 256 ? 1 : 2;
    static constexpr int TILE_Q = BM * HD * 2;
    static constexpr int TILE_KV = BN * HD * 2;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + TILE_Q;
    static constexpr int OFF_V = OFF_K + KV_STAGES * TILE_KV;
    static constexpr int OFF_BIAS = OFF_V + KV_STAGES * TILE_KV;
    static constexpr int OFF_BAR = OFF_BIAS + 4 * 2 * BN * 4;  // a private bias copy per softmax warp
    static constexpr int NUM_BARS = 16;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
    static constexpr uint32_t TMEM_COLS = 512;  // S0 | S1 | O (P_j as bf16 over S_(j&1))
    static_assert(ALLOC <= 227 * 1024, "shared memory");
    static_assert(2 * BN + HD <= 512, "TMEM columns");
};

// barrier indices
enum : int {
    B_Q_FULL = 0, B_K_FULL = 1, B_K_EMPTY = 3, B_V_FULL = 5, B_V_EMPTY = 7, B_S_FULL = 9, B_S_FREE = 11,
    B_P_FULL = 13, B_PV_DONE = 14, B_DRAIN = 15
};

// Optional device trace (builds with -DTG_TRACE only): clock64 stamps of the
// pipeline hand-offs of the CTA at blockIdx (0, 0, 0), 64 KV tiles at most.
#ifdef TG_TRACE
__device__ unsigned long long g_attn_trace[24 * 64];  // points 0..23 x 64 tiles
__device__ unsigned long long g_attn_cta[4096 * 12];  // per CTA: phase stamps (ns), SM id | n_kv
#define TG_TRACE_AT(point, j)                                                              \
    do {                                                                                   \
        if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && (j) < 64)             \
            g_attn_trace[(point) * 64 + (j)] = static_cast<unsigned long long>(clock64()); \
    } while (0)
#define TG_CTA_STAMP(slot)                                                                            \
    do {                                                                                              \
        const unsigned idx_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);        \
        if (idx_ < 4096) g_attn_cta[idx_ * 12 + (slot)] = globaltimer();                              \
    } while (0)
#else
#define TG_CTA_STAMP(slot) \
    do {                   \
    } while (0)
#define TG_TRACE_AT(point, j) \
    do {                      \
    } while (0)
#endif

template <int HD>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gated_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ cu_kept,
                     const int32_t* __restrict__ pos, const int32_t* __restrict__ rank, const GateSet gates,
                     const float* __restrict__ c, float sm_scale, int Hq, int Hkv, int n_qt_max,
                     uint16_t* __restrict__ out, float* __restrict__ lse, int* __restrict__ status) {
    using L = AttnSmem<HD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int h = blockIdx.x;
    const int qt = n_qt_max - 1 - static_cast<int>(blockIdx.y);
    const int b = blockIdx.z;
    pdl_wait();  // global memory is read only from here on
    pdl_trigger();
    const int seq0 = cu_kept[b];
    const int Mb = cu_kept[b + 1] - seq0;
    if (qt * BM >= Mb) return;
    const int n_kv = qt + 1;  // BM == BN: the diagonal tile is the last one
    const int hk = h / (Hq / Hkv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + L::OFF_Q, sK0 = sbase + L::OFF_K, sV0 = sbase + L::OFF_V;
    constexpr int NS = L::KV_STAGES;
    auto bar = [&](int i) { return sbase + L::OFF_BAR + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    float* sBias = reinterpret_cast<float*>(smem + L::OFF_BIAS);

    if (threadIdx.x == 0) {
        mbar_init(bar(B_Q_FULL), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_K_FULL + s), 1);
            mbar_init(bar(B_K_EMPTY + s), 1);
            mbar_init(bar(B_V_FULL + s), 1);
            mbar_init(bar(B_V_EMPTY + s), 1);
            mbar_init(bar(B_S_FULL + s), 1);
            mbar_init(bar(B_S_FREE + s), 128);
        }
        mbar_init(bar(B_P_FULL), 128);
        mbar_init(bar(B_PV_DONE), 1);
        mbar_init(bar(B_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 4) {
        tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tmem_O = tmem + 2 * BN;

    if (warp == 4) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            mbar_expect_tx(bar(B_Q_FULL), BM * HD * 2);
#pragma unroll
            for (int hf = 0; hf < HD / 64; ++hf)
                tma_load_2d(sQ + hf * BM * 128, &tmQ, h * HD + hf * 64, seq0 + qt * BM, bar(B_Q_FULL));
            int k_issued[2] = {0, 0}, v_issued[2] = {0, 0};
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % NS;
                if (j >= NS && !mbar_wait(bar(B_K_EMPTY + s), ((j - NS) / NS) & 1, abort_flag, status,
                                          TG_WHERE_PRODUCER))
                    break;
                mbar_expect_tx(bar(B_K_FULL + s), BN * HD * 2);
#pragma unroll
                for (int hf = 0; hf < HD / 64; ++hf)
                    tma_load_2d(sK0 + s * L::TILE_KV + hf * BN * 128, &tmK, hk * HD + hf * 64, seq0 + j * BN,
                                bar(B_K_FULL + s));
                ++k_issued[s];
                if (j >= NS && !mbar_wait(bar(B_V_EMPTY + s), ((j - NS) / NS) & 1, abort_flag, status,
                                          TG_WHERE_PRODUCER))
                    break;
                mbar_expect_tx(bar(B_V_FULL + s), BN * HD * 2);
#pragma unroll
                for (int hf = 0; hf < HD / 64; ++hf)
                    tma_load_2d(sV0 + s * L::TILE_KV + hf * BN * 128, &tmV, hk * HD + hf * 64, seq0 + j * BN,
                                bar(B_V_FULL + s));
                ++v_issued[s];
            }
            if (*abort_flag) {
                // let every copy this thread started land before the CTA exits
                drain_wait(bar(B_Q_FULL), 0, status);
                for (int s = 0; s < NS; ++s) {
                    if (k_issued[s]) drain_wait(bar(B_K_FULL + s), (k_issued[s] - 1) & 1, status);
                    if (v_issued[s]) drain_wait(bar(B_V_FULL + s), (v_issued[s] - 1) & 1, status);
                }
            }
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, HD, true);
            bool ok = mbar_wait(bar(B_Q_FULL), 0, abort_flag, status, TG_WHERE_MMA);
            for (int j = 0; ok && j <= n_kv; ++j) {
                if (j < n_kv) {
                    const int s = j & 1, ks = j % NS;
                    ok = mbar_wait(bar(B_K_FULL + ks), (j / NS) & 1, abort_flag, status, TG_WHERE_MMA);
                    if (ok && j >= 2)
                        ok = mbar_wait(bar(B_S_FREE + s), ((j - 2) >> 1) & 1, abort_flag, status, TG_WHERE_MMA);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t d = tmem + s * BN;
                    const uint32_t kb = sK0 + ks * L::TILE_KV;
#pragma unroll
                    for (int kk = 0; kk < HD / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                        const uint32_t offk = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
                        mma_bf16_ss(d, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(kb + offk, 16, 1024),
                                    idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(B_S_FULL + s));
                    mma_commit(bar(B_K_EMPTY + ks));
                }
                if (j >= 1) {
                    const int jj = j - 1, s = jj & 1, vs = jj % NS;
                    ok = mbar_wait(bar(B_P_FULL), jj & 1, abort_flag, status, TG_WHERE_MMA);
                    if (ok) ok = mbar_wait(bar(B_V_FULL + vs), (jj / NS) & 1, abort_flag, status, TG_WHERE_MMA);
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t vb = sV0 + vs * L::TILE_KV;
                    // A = P_jj from TMEM (16 keys = 8 columns of bf16 pairs per k-step)
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        mma_bf16_ts(tmem_O, tmem + s * BN + kk * 8, smem_desc_sw128(vb + kk * 16 * 128, BN * 128, 1024),
                                    idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(bar(B_PV_DONE));
                    mma_commit(bar(B_V_EMPTY + vs));
                }
            }
            // every MMA (and the barrier arrivals its commits trigger) lands before the CTA exits
            mma_commit(bar(B_DRAIN));
            drain_wait(bar(B_DRAIN), 0, status);
        }
    } else {
        // ---------------------------------------------------------------- softmax warps 0-3
        const int r = threadIdx.x;  // query row within the tile == TMEM lane
        const int q_local = qt * BM + r;
        const bool valid_row = q_local < Mb;
        const int qg = seq0 + q_local;
        float inv_tau = 1.0f;
        if (valid_row)
            inv_tau = 1.0f / (1.0f + c[h] * logf(static_cast<float>(__ldcg(pos + qg)) / static_cast<float>(__ldcg(rank + qg))));
        const float alpha = sm_scale * LOG2E * inv_tau;
        float gscale[kMaxGates];  // per gate: softplus(g_h) in log2 units (0 past the last gate)
#pragma unroll
        for (int gi = 0; gi < kMaxGates; ++gi) gscale[gi] = gi < gates.n ? softplus_f(gates.g[gi][h]) * LOG2E : 0.f;
        const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = true;
        float* wbias = sBias + warp * (2 * BN);  // this warp's copy, double-buffered
        for (int j = 0; j < n_kv; ++j) {
            const int s = j & 1;
            // gate bias of the tile's 128 keys (summed over the gates), log2 domain; each
            // warp keeps its own copy so that only __syncwarp orders it
#pragma unroll
            for (int e = 0; e < BN / 32; ++e) {
                const int key_local = j * BN + e * 32 + lane;
                float bsum = 0.f;
                if (key_local < Mb) {
                    bsum = gscale[0] * __ldcg(gates.gls[0] + seq0 + key_local);
#pragma unroll
                    for (int gi = 1; gi < kMaxGates; ++gi)
                        if (gi < gates.n) bsum += gscale[gi] * __ldcg(gates.gls[gi] + seq0 + key_local);
                }
                wbias[s * BN + e * 32 + lane] = bsum;
            }
            __syncwarp();
            ok = mbar_wait_warp(bar(B_S_FULL + s), (j >> 1) & 1, abort_flag, status, TG_WHERE_SOFTMAX);
            if (!ok) break;
            tc_fence_after();
            float x[BN];
#pragma unroll
            for (int ch = 0; ch < BN / 32; ++ch) tmem_ld32(tmem + lane_addr + s * BN + ch * 32, x + ch * 32);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar(B_S_FREE + s));

            const float* bias = wbias + s * BN;
            float mx = -INFINITY;
            if (j == n_kv - 1) {
                const int lim = q_local - j * BN;  // keys with column > lim lie in the causal future
#pragma unroll
                for (int cc = 0; cc < BN; ++cc) {
                    const float v = fmaf(x[cc], alpha, bias[cc] * inv_tau);
                    x[cc] = cc > lim ? -INFINITY : v;
                    mx = fmaxf(mx, x[cc]);
                }
            } else {
#pragma unroll
                for (int cc = 0; cc < BN; ++cc) {
                    x[cc] = fmaf(x[cc], alpha, bias[cc] * inv_tau);
                    mx = fmaxf(mx, x[cc]);
                }
            }
            float corr = 1.0f;
            bool rescale_o = false;
            if (j == 0 || mx > m_run + RESCALE_THRESHOLD) {
                const float m_new = fmaxf(m_run, mx);
                corr = exp2f(m_run - m_new);
                m_run = m_new;
                rescale_o = j > 0;
            }
            float sum = 0.f;
#pragma unroll
            for (int cc = 0; cc < BN; ++cc) {
                x[cc] = exp2f(x[cc] - m_run);
                sum += x[cc];
            }
            l_run = l_run * corr + sum;
            // the P tile and O may be touched only once PV_{j-1} has completed
            if (j >= 1) {
                ok = mbar_wait_warp(bar(B_PV_DONE), (j - 1) & 1, abort_flag, status, TG_WHERE_SOFTMAX);
                if (!ok) break;
                tc_fence_after();
            }
            if (rescale_o) {
#pragma unroll
                for (int ch = 0; ch < HD / 32; ++ch) {
                    float o[32];
                    tmem_ld32(tmem_O + lane_addr + ch * 32, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= corr;
                    tmem_st32(tmem_O + lane_addr + ch * 32, o);
                }
                tmem_wait_st();
            }
            // P row r as bf16 pairs over the first 64 columns of its S buffer (the A
            // operand of the PV MMA, read from TMEM)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = pack_bf16x2(x[hf * 64 + 2 * e], x[hf * 64 + 2 * e + 1]);
                tmem_st32u(tmem + lane_addr + s * BN + hf * 32, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_P_FULL));
        }
        // ---------------------------------------------------------------- epilogue
        if (ok) ok = mbar_wait_warp(bar(B_PV_DONE), (n_kv - 1) & 1, abort_flag, status, TG_WHERE_SOFTMAX);
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.0f / l_run;
            uint16_t* orow = out + (static_cast<size_t>(qg) * Hq + h) * HD;
#pragma unroll
            for (int ch = 0; ch < HD / 32; ++ch) {
                float o[32];
                tmem_ld32(tmem_O + lane_addr + ch * 32, o);
                tmem_wait_ld();
                if (valid_row) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 v;
                        v.x = pack_bf16x2(o[q4 * 8 + 0] * inv_l, o[q4 * 8 + 1] * inv_l);
                        v.y = pack_bf16x2(o[q4 * 8 + 2] * inv_l, o[q4 * 8 + 3] * inv_l);
                        v.z = pack_bf16x2(o[q4 * 8 + 4] * inv_l, o[q4 * 8 + 5] * inv_l);
                        v.w = pack_bf16x2(o[q4 * 8 + 6] * inv_l, o[q4 * 8 + 7] * inv_l);
                        *reinterpret_cast<uint4*>(orow + ch * 32 + q4 * 8) = v;
                    }
                }
            }
            if (valid_row && lse) lse[static_cast<size_t>(qg) * Hq + h] = (m_run + log2f(l_run)) / LOG2E;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Two query heads of one KV head per CTA (GQA groups of even size).
//
// 320 threads: warps 0-7 = softmax of both heads in turn (thread = one row,
// one half of the columns), warp 8 = TMA producer, warp 9 = MMA issuer.
// Both heads share every K/V tile.  TMEM (512 columns): S0 | S1 | O0 | O1;
// P_h (bf16, two keys per column) is written over the first 64 columns of
// S_h and read from TMEM as the A operand of the PV MMA.  The MMA issuer
// interleaves
//     S0(j) S1(j) | PV0(j) S0(j+1) | PV1(j) S1(j+1) | ...
// and the softmax warps take head 0 of tile j, head 1 of tile j, head 0 of
// tile j+1, ..., so that one head's softmax overlaps the other head's
// tensor-core work;
// tcgen05 operations of one thread execute in issue order, which is what
// lets S_h(j+1) overwrite P_h(j) right after PV_h(j), and what makes the
// commit after S_h(j) also cover PV_h(j-1) (so the softmax may rescale O_h
// as soon as S_h(j) is complete).
constexpr int G2_THREADS = 320;

template <int HD>
struct G2Smem {
    static constexpr int TILE_Q = BM * HD * 2;
    static constexpr int TILE_KV = BN * HD * 2;
    static constexpr int OFF_Q = 0;  // two heads
    static constexpr int OFF_K = OFF_Q + 2 * TILE_Q;
    static constexpr int OFF_V = OFF_K + 2 * TILE_KV;
    // operands of the extra k-step that adds the gate bias to S: 128 rows x 16 bf16,
    // no swizzle (8-row x 16-byte core matrices, K cores 128 B apart, row groups 256 B)
    static constexpr int EXT = BM * 16 * 2;
    static constexpr int OFF_QX = OFF_V + 2 * TILE_KV;  // [head]
    static constexpr int OFF_KX = OFF_QX + 2 * EXT;      // [stage]
    // partial row maxima [parity][half][row] (2 KB) and partial row sums [head][half][row] (2 KB)
    static constexpr int OFF_RED = OFF_KX + 2 * EXT;
    static constexpr int OFF_BAR = OFF_RED + 2 * 2 * BM * 4 + 2 * 2 * BM * 4;
    static constexpr int NUM_BARS = 18;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + 16;
    static constexpr int ALLOC = BYTES + 1024;
    static constexpr uint32_t TMEM_COLS = 512;
};

enum : int {
    G_Q_FULL = 0, G_K_FULL = 1, G_K_EMPTY = 3, G_V_FULL = 5, G_V_EMPTY = 7, G_S_FULL = 9, G_P_FULL = 11,
    G_O_FULL = 13, G_DRAIN = 14
};

// Q_ext columns 4..15 (gates 2..n) of both heads' rows, out of line so that the
// one-gate kernel body stays as it is without them.  Called by every thread of the
// CTA: the barrier orders these writes after the zeroing of cores 8..15.
template <typename L>
__device__ __noinline__ void g2_extra_gates_q(uint8_t* smem, int n, const float* g1, const float* g2,
                                              const float* g3, int pair, float sm_scale) {
    __syncthreads();
    if (threadIdx.x < 2 * BM) {
        const int hh = threadIdx.x / BM, r = threadIdx.x % BM;
        uint8_t* row = smem + L::OFF_QX + hh * L::EXT + (r >> 3) * 256 + (r & 7) * 16;
        for (int gi = 1; gi < n; ++gi) {
            const float* gg = gi == 1 ? g1 : (gi == 2 ? g2 : g3);
            const uint32_t hl = bf16_hi_lo(softplus_f(gg[2 * pair + hh]) / sm_scale);
            *reinterpret_cast<uint2*>(row + (gi >> 1) * 128 + (gi & 1) * 8) = make_uint2(hl, hl);
        }
    }
}

template <int HD>
__global__ void __launch_bounds__(G2_THREADS, 1)
gated_attn_gqa2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ cu_kept,
                       const int32_t* __restrict__ pos, const int32_t* __restrict__ rank, const GateSet gates,
                       const float* __restrict__ c, float sm_scale, int Hq, int Hkv, int n_qt_max, int kv_chunk,
                       SplitWs ws,
                       uint16_t* __restrict__ out, float* __restrict__ lse, int* __restrict__ status, int early) {
    using L = G2Smem<HD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int pair = blockIdx.x;            // query heads 2*pair and 2*pair+1
    const int b = blockIdx.z;
#ifdef TG_TRACE
    const unsigned long long trace_t0 = globaltimer();
#endif
    // `early`: q, k, v, g, c and cu_kept were complete before the preceding kernel started
    // (the caller's guarantee), so the set-up, Q and the first K/V tiles go ahead while that
    // kernel runs; only the compaction map (pos, rank, gls) and the split scratch wait for it,
    // each role executing the wait before its first such access.  Otherwise every global
    // access waits here.
    if (!early) {
        pdl_wait();
        pdl_trigger();
    }
    const int seq0 = cu_kept[b];
    const int Mb = cu_kept[b + 1] - seq0;
    const int n_qt = (Mb + BM - 1) / BM;
    const int C = min(kv_chunk, max(n_qt, 1));
    // unit -> (query tile, chunk) in order of decreasing cost (KV tiles), so that
    // the block scheduler hands out the longest units first
    int64_t u = blockIdx.y;
    const int64_t n_units = units_below(n_qt, C);
    if (u >= n_units) return;
    int qt = 0, chunk = 0;
    if (C >= n_qt) {
        qt = n_qt - 1 - static_cast<int>(u);  // unsplit: query tile qt costs qt + 1
    } else {
        // C >= ceil(n_qt / 2): query tiles C..n_qt-1 split into [0, C) and [C, qt+1).
        // Cost C first: every first chunk; then for v = C, C-1, ..., 1 the unsplit
        // query tile v-1 and the second chunk of query tile v-1+C (if it exists).
        const int a = n_qt - C;
        if (u < a) {
            qt = n_qt - 1 - static_cast<int>(u);
        } else {
            u -= a;
            for (int v = C; v >= 1; --v) {
                if (u == 0) { qt = v - 1; break; }
                --u;
                if (v - 1 + C <= n_qt - 1) {
                    if (u == 0) { qt = v - 1 + C; chunk = 1; break; }
                    --u;
                }
            }
        }
    }
    const int nch = (qt + C) / C;  // ceil((qt + 1) / C), 1 or 2
    const int kv0 = chunk * C;
    const int kv1 = min(qt + 1, kv0 + C);
    const int n_kv = kv1 - kv0;  // the chunk holding the diagonal tile is the last one
    const bool split = nch > 1;
    const int hk = (2 * pair) / (Hq / Hkv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + L::OFF_Q, sK0 = sbase + L::OFF_K, sV0 = sbase + L::OFF_V;
    auto bar = [&](int i) { return sbase + L::OFF_BAR + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    const uint32_t sQX = sbase + L::OFF_QX, sKX = sbase + L::OFF_KX;

    // Gate bias as one more k-step of the S = Q K^T product.  Gate i owns columns
    // 4i .. 4i+3 of the step: row q of Q_ext holds (bh, bl, bh, bl) and row j of K_ext
    // holds (gh, gh, gl, gl), the bf16 high and low parts of bscale_h = softplus(g_h) /
    // sm_scale and of gls_j, so that the four products add bscale_h * gls_j to S with
    // about 2^-16 relative error.  Columns of absent gates are zero: K cores 8..15 of all
    // four tiles are zeroed here and columns 4..7 are written as zeros with the first
    // gate's; further gates (rare) are filled in by out-of-line code, which keeps the
    // one-gate kernel body unchanged.
    for (int i = threadIdx.x; i < 4 * (BM / 8) * 8; i += blockDim.x) {
        const int tile = i / ((BM / 8) * 8), rem = i % ((BM / 8) * 8);
        *reinterpret_cast<uint4*>(smem + L::OFF_QX + tile * L::EXT + (rem >> 3) * 256 + 128 + (rem & 7) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
    if (threadIdx.x < 2 * BM) {
        const int hh = threadIdx.x / BM, r = threadIdx.x % BM;
        const float bscale = softplus_f(gates.g[0][2 * pair + hh]) / sm_scale;
        const uint32_t hl = bf16_hi_lo(bscale);
        *reinterpret_cast<uint4*>(smem + L::OFF_QX + hh * L::EXT + (r >> 3) * 256 + (r & 7) * 16) =
            make_uint4(hl, hl, 0u, 0u);
    }
    if (gates.n > 1)  // uniform: all threads
        g2_extra_gates_q<L>(smem, gates.n, gates.g[1], gates.g[2], gates.g[3], pair, sm_scale);
    fence_proxy_async_smem();

    if (threadIdx.x == 0) {
        mbar_init(bar(G_Q_FULL), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(G_K_FULL + s), 2);  // the K tile's bytes and the producer's K_ext rows
            mbar_init(bar(G_K_EMPTY + s), 1);
            mbar_init(bar(G_V_FULL + s), 1);
            mbar_init(bar(G_V_EMPTY + s), 1);
            mbar_init(bar(G_S_FULL + s), 1);
            mbar_init(bar(G_P_FULL + s), 8);  // one arrival per softmax warp
        }
        mbar_init(bar(G_O_FULL), 1);
        mbar_init(bar(G_DRAIN), 1);
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
    if (threadIdx.x == 0) TG_CTA_STAMP(1);

    if (warp == 8) {
        // ---------------------------------------------------------------- TMA producer
        // The whole warp writes the K_ext rows of each KV tile (lane l: keys 4l .. 4l+3);
        // lane 0 issues the copies.  K_ext(stage) is released with K(stage).
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            mbar_expect_tx(bar(G_Q_FULL), 2 * BM * HD * 2);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int hf = 0; hf < HD / 64; ++hf)
                    tma_load_2d(sQ + hh * L::TILE_Q + hf * BM * 128, &tmQ, (2 * pair + hh) * HD + hf * 64,
                                seq0 + qt * BM, bar(G_Q_FULL));
        }
        int k_issued[2] = {0, 0}, v_issued[2] = {0, 0};
        auto issue_k = [&](int j) {
            const int s = j & 1;
            mbar_expect_tx(bar(G_K_FULL + s), BN * HD * 2);
#pragma unroll
            for (int hf = 0; hf < HD / 64; ++hf)
                tma_load_2d(sK0 + s * L::TILE_KV + hf * BN * 128, &tmK, hk * HD + hf * 64, seq0 + (kv0 + j) * BN,
                            bar(G_K_FULL + s));
            ++k_issued[s];
        };
        auto issue_v = [&](int j) {
            const int s = j & 1;
            mbar_expect_tx(bar(G_V_FULL + s), BN * HD * 2);
#pragma unroll
            for (int hf = 0; hf < HD / 64; ++hf)
                tma_load_2d(sV0 + s * L::TILE_KV + hf * BN * 128, &tmV, hk * HD + hf * 64, seq0 + (kv0 + j) * BN,
                            bar(G_V_FULL + s));
            ++v_issued[s];
        };
        // The first two tiles' K and V copies leave at once (their stages are free): before the
        // compaction map is available in an early launch, and before the first gls loads (which
        // the K_ext rows wait for) in every launch.
        const int pre = min(n_kv, 2);
        if (lane == 0)
            for (int j = 0; j < pre; ++j) {
                issue_k(j);
                issue_v(j);
            }
        if (early) {
            pdl_wait();  // gls (the compaction map) is read from here on
            // dependents are released only now, once the preceding kernel has completed, so
            // a following row gather may read the compaction map straight away
            if (lane == 0) pdl_trigger();
        }
        float gk[4];  // first gate's gls of this lane's keys of the next tile (0 past the end)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int key_local = kv0 * BN + lane * 4 + i;
            gk[i] = key_local < Mb ? ldg_early(gates.gls[0] + seq0 + key_local) : 0.f;
        }
        for (int j = 0; j < n_kv; ++j) {
            const int s = j & 1;
            float gcur[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) gcur[i] = gk[i];
            if (j + 1 < n_kv) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int key_local = (kv0 + j + 1) * BN + lane * 4 + i;
                    gk[i] = key_local < Mb ? ldg_early(gates.gls[0] + seq0 + key_local) : 0.f;
                }
            }
            if (j >= 2 && !mbar_wait_warp(bar(G_K_EMPTY + s), ((j - 2) >> 1) & 1, abort_flag, status,
                                          TG_WHERE_PRODUCER))
                break;
            if (lane == 0 && j >= pre) issue_k(j);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = lane * 4 + i;
                const uint32_t hl = bf16_hi_lo(gcur[i]);
                *reinterpret_cast<uint4*>(smem + L::OFF_KX + s * L::EXT + (r >> 3) * 256 + (r & 7) * 16) =
                    make_uint4(__byte_perm(hl, 0u, 0x1010), __byte_perm(hl, 0u, 0x3232), 0u, 0u);
            }
            // further gates (rare): the same lane rewrites its rows' slots of those gates
#pragma unroll 1
            for (int gi = 1; gi < gates.n; ++gi) {
                // (a select chain, not gates.gls[gi]: a run-time index into the parameter
                // block would copy it to local memory)
                const float* gsrc = (gi == 1 ? gates.gls[1] : (gi == 2 ? gates.gls[2] : gates.gls[3])) + seq0 +
                                    (kv0 + j) * BN;
                const int valid = Mb - (kv0 + j) * BN;
                uint8_t* kx = smem + L::OFF_KX + s * L::EXT;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = lane * 4 + i;
                    const uint32_t hl = bf16_hi_lo(r < valid ? __ldcg(gsrc + r) : 0.f);
                    *reinterpret_cast<uint2*>(kx + (r >> 3) * 256 + (gi >> 1) * 128 + (r & 7) * 16 + (gi & 1) * 8) =
                        make_uint2(__byte_perm(hl, 0u, 0x1010), __byte_perm(hl, 0u, 0x3232));
                }
            }
            fence_proxy_async_smem();  // K_ext is read by the tensor core (async proxy)
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(G_K_FULL + s));  // the K_ext half of the stage
            if (j >= 2 && !mbar_wait_warp(bar(G_V_EMPTY + s), ((j - 2) >> 1) & 1, abort_flag, status,
                                          TG_WHERE_PRODUCER))
                break;
            if (lane == 0 && j >= pre) issue_v(j);
        }
        if (lane == 0 && *abort_flag) {
            drain_wait(bar(G_Q_FULL), 0, status);
            for (int s = 0; s < 2; ++s) {
                if (k_issued[s]) drain_wait(bar(G_K_FULL + s), (k_issued[s] - 1) & 1, status);
                if (v_issued[s]) drain_wait(bar(G_V_FULL + s), (v_issued[s] - 1) & 1, status);
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, HD, true);
            auto issue_s = [&](int hh, int j) {
                const uint32_t kb = sK0 + (j & 1) * L::TILE_KV;
                const uint32_t qb = sQ + hh * L::TILE_Q;
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off_q = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                    const uint32_t off_k = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
                    mma_bf16_ss(tmem + hh * BN, smem_desc_sw128(qb + off_q, 16, 1024),
                                smem_desc_sw128(kb + off_k, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                }
                // + bscale_h * gls_j: the bias k-step (no-swizzle tiles, K cores 128 B apart)
                mma_bf16_ss(tmem + hh * BN, smem_desc_noswz(sQX + hh * L::EXT, 128, 256),
                            smem_desc_noswz(sKX + (j & 1) * L::EXT, 128, 256), idesc_qk, 1u);
            };
            auto issue_pv = [&](int hh, int j) {
                const uint32_t vb = sV0 + (j & 1) * L::TILE_KV;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    mma_bf16_ts(tmem + 2 * BN + hh * HD, tmem + hh * BN + kk * 8,
                                smem_desc_sw128(vb + kk * 16 * 128, BN * 128, 1024), idesc_pv,
                                (j > 0 || kk > 0) ? 1u : 0u);
            };
            bool ok = mbar_wait(bar(G_Q_FULL), 0, abort_flag, status, TG_WHERE_MMA) &&
                      mbar_wait(bar(G_K_FULL), 0, abort_flag, status, TG_WHERE_MMA);
            TG_CTA_STAMP(2);
            if (ok) {
                tc_fence_after();
                issue_s(0, 0);
                mma_commit(bar(G_S_FULL + 0));
                issue_s(1, 0);
                mma_commit(bar(G_S_FULL + 1));
                mma_commit(bar(G_K_EMPTY + 0));
            }
            for (int j = 0; ok && j < n_kv; ++j) {
                const int s = j & 1;
                const bool more = j + 1 < n_kv;
                ok = mbar_wait(bar(G_V_FULL + s), (j >> 1) & 1, abort_flag, status, TG_WHERE_MMA) &&
                     mbar_wait(bar(G_P_FULL + 0), j & 1, abort_flag, status, TG_WHERE_MMA);
                if (!ok) break;
                tc_fence_after();
                TG_TRACE_AT(0, j);  // P0(j) ready, issuing PV0(j)
                issue_pv(0, j);
                if (more) {
                    ok = mbar_wait(bar(G_K_FULL + (s ^ 1)), ((j + 1) >> 1) & 1, abort_flag, status, TG_WHERE_MMA);
                    if (!ok) break;
                    tc_fence_after();
                    issue_s(0, j + 1);
                    mma_commit(bar(G_S_FULL + 0));
                    TG_TRACE_AT(10, j);  // S0(j+1) issued
#ifdef TG_TRACE
                    // trace builds only: stamp the completion of S0(j+1) as the tensor core sees it
                    if (mbar_wait(bar(G_S_FULL + 0), (j + 1) & 1, abort_flag, status, TG_WHERE_MMA)) TG_TRACE_AT(13, j);
#endif
                }
                ok = mbar_wait(bar(G_P_FULL + 1), j & 1, abort_flag, status, TG_WHERE_MMA);
                if (!ok) break;
                tc_fence_after();
                TG_TRACE_AT(1, j);  // P1(j) ready, issuing PV1(j)
                issue_pv(1, j);
                mma_commit(bar(G_V_EMPTY + s));
                if (more) {
                    issue_s(1, j + 1);
                    mma_commit(bar(G_S_FULL + 1));
                    mma_commit(bar(G_K_EMPTY + (s ^ 1)));
                }
            }
            if (ok) mma_commit(bar(G_O_FULL));
            mma_commit(bar(G_DRAIN));
            drain_wait(bar(G_DRAIN), 0, status);
        }
    } else {
        // ---------------------------------------------------------------- softmax, warps 0-7
        // Thread (warp w, lane l) owns query row r = 32 (w & 3) + l (TMEM lane r) and the
        // key / output columns [64 half, 64 half + 64), half = w >> 2, of BOTH heads.  The
        // eight warps take the heads in turn (head 0 of tile j, head 1 of tile j, head 0 of
        // tile j + 1, ...): each head's exponentials run on two warps of every SM
        // sub-partition, which keeps the special-function unit busy, while the tensor core
        // works on the other head.  The two halves of a row combine their partial maxima
        // through shared memory at a barrier that also makes any abort decision uniform.
        // S already holds s + bscale_h * gls_j (the bias k-step), so in log2 units the
        // logit is  x = alpha_q * S  with  alpha_q = sm_scale * log2(e) / tau_q: one FMA per
        // score with the running max folded in, issued as f32x2 pairs, and no shared-memory
        // reads in the loop (those would queue behind the tensor core's operand traffic).
        const int q4 = warp & 3;
        const int half = warp >> 2;
        const int r = q4 * 32 + lane;        // query row == TMEM lane
        const int q_local = qt * BM + r;
        const bool valid_row = q_local < Mb;
        const int qg = seq0 + q_local;
        if (early) pdl_wait();  // pos and rank (the compaction map) and the split scratch from here on
        // (through L2, as ldg_early, since their writer may have run during this kernel's lifetime)
        const float ratio_log =
            valid_row ? logf(static_cast<float>(__ldcg(pos + qg)) / static_cast<float>(__ldcg(rank + qg))) : 0.f;
        // per-head values are scalars selected by the head index (no local-memory arrays)
        const float inv_tau0 = valid_row ? 1.0f / (1.0f + c[2 * pair] * ratio_log) : 1.0f;
        const float inv_tau1 = valid_row ? 1.0f / (1.0f + c[2 * pair + 1] * ratio_log) : 1.0f;
        const float alpha0 = sm_scale * LOG2E * inv_tau0, alpha1 = sm_scale * LOG2E * inv_tau1;
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        float* red = reinterpret_cast<float*>(smem + L::OFF_RED);  // [parity][half][row] partial maxima
        float* lred = red + 2 * 2 * BM;                             // [head][half][row] partial sums
        float m_run0 = -INFINITY, m_run1 = -INFINITY, l_run0 = 0.f, l_run1 = 0.f;
        bool ok = true;
        int arrival = 0;  // thread 0: the split unit's arrival at its counter (taken a tile early)
        for (int j = 0; ok && j < n_kv; ++j) {
            const int jt = kv0 + j;  // KV tile index within the sequence
            if (split && j + 1 == n_kv && threadIdx.x == 0) {
                // its round trip overlaps the last tile; the value is first used in the epilogue
                arrival = atomicAdd(ws.cnt + (static_cast<int64_t>(b) * (Hq / 2) + pair) * ws.slots_per_pair + (qt - C), 1);
            }
            const bool diag = (jt == qt);
            const int lim = q_local - jt * BN - half * 64;  // on the diagonal tile, own columns > lim are future keys
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                const int step = 2 * j + hh;
                const float alpha = hh ? alpha1 : alpha0;
                float m_h = hh ? m_run1 : m_run0;
                const uint32_t tS = tmem + lane_addr + hh * BN;
                const bool okw = mbar_wait_warp(bar(G_S_FULL + hh), j & 1, abort_flag, status, TG_WHERE_SOFTMAX);
                if (r == 0 && half == 0) TG_TRACE_AT(2 + 4 * hh, j);  // S_h(j) ready
                if (threadIdx.x == 0 && step == 0) TG_CTA_STAMP(3);
                float x[64];
                float my = -INFINITY;
                if (okw) {
                    tc_fence_after();
                    tmem_ld32(tS + half * 64, x);
                    tmem_ld32(tS + half * 64 + 32, x + 32);
                    tmem_wait_ld();
                    if (r == 0 && half == 0) TG_TRACE_AT(3 + 4 * hh, j);  // S_h(j) in registers
                    if (diag) {
#pragma unroll
                        for (int cc = 0; cc < 64; ++cc) x[cc] = cc > lim ? -INFINITY : x[cc];
                    }
                    // stabiliser: the row max of the biased scores
                    float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int cc = 0; cc < 64; cc += 2) mp[(cc >> 1) & 3] = max3f(mp[(cc >> 1) & 3], x[cc], x[cc + 1]);
                    my = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
                }
                red[(step & 1) * (2 * BM) + half * BM + r] = my;
                // every S load of both halves is complete past this barrier, so P may overwrite S
                if (bar_red_or(1, 256, !okw)) {
                    ok = false;
                    break;
                }
                my = fmaxf(my, red[(step & 1) * (2 * BM) + (half ^ 1) * BM + r]);
                // floored so that a tile whose keys all carry an infinite negative bias gives
                // p = 0 instead of 2^(-inf + inf)
                const float mx = fmaxf(alpha * my, -1.0e30f);
                float corr = 1.0f;
                bool rescale_o = false;
                if (j == 0 || mx > m_h + RESCALE_THRESHOLD) {
                    const float m_new = fmaxf(m_h, mx);
                    corr = ex2_approx(m_h - m_new);
                    m_h = m_new;
                    rescale_o = j > 0;
                }
                if (hh) m_run1 = m_h; else m_run0 = m_h;
                if (r == 0 && half == 0) TG_TRACE_AT(4 + 4 * hh, j);  // max done
                const uint64_t al2 = f32x2_pack(alpha, alpha);
                const uint64_t nm2 = f32x2_pack(-m_h, -m_h);
                uint64_t sp[4] = {0ull, 0ull, 0ull, 0ull};
                uint32_t pk[32];
#pragma unroll
                for (int c4 = 0; c4 < 16; ++c4) {
                    const int cc = c4 * 4;
                    const uint64_t a0 = f32x2_fma(al2, f32x2_pack(x[cc], x[cc + 1]), nm2);
                    const uint64_t a1 = f32x2_fma(al2, f32x2_pack(x[cc + 2], x[cc + 3]), nm2);
                    const float p0 = ex2_approx(f32x2_lo(a0)), p1 = ex2_approx(f32x2_hi(a0));
                    const float p2 = ex2_approx(f32x2_lo(a1)), p3 = ex2_approx(f32x2_hi(a1));
                    sp[(2 * c4) & 3] = f32x2_add(sp[(2 * c4) & 3], f32x2_pack(p0, p1));
                    sp[(2 * c4 + 1) & 3] = f32x2_add(sp[(2 * c4 + 1) & 3], f32x2_pack(p2, p3));
                    pk[cc / 2] = pack_bf16x2(p0, p1);
                    pk[cc / 2 + 1] = pack_bf16x2(p2, p3);
                }
                // P_h: keys 64 half .. 64 half + 63 -> columns 32 half .. 32 half + 31 of S_h
                tmem_st32u(tS + half * 32, pk);
                if (r == 0 && half == 0) TG_TRACE_AT(11 + 3 * hh, j);  // exponentials done
                const uint64_t s01 = f32x2_add(sp[0], sp[1]), s23 = f32x2_add(sp[2], sp[3]);
                const uint64_t s4 = f32x2_add(s01, s23);
                const float tile_sum = f32x2_lo(s4) + f32x2_hi(s4);
                if (hh) l_run1 = l_run1 * corr + tile_sum; else l_run0 = l_run0 * corr + tile_sum;
                if (rescale_o) {
                    // O_h is stable: PV_h(j-1) completed before S_h(j), PV_h(j) waits for P_h(j)
                    const uint32_t tO = tmem + lane_addr + 2 * BN + hh * HD + half * (HD / 2);
#pragma unroll
                    for (int ch = 0; ch < HD / 64; ++ch) {
                        float o[32];
                        tmem_ld32(tO + ch * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= corr;
                        tmem_st32(tO + ch * 32, o);
                    }
                }
                tmem_wait_st();
                if (r == 0 && half == 0) TG_TRACE_AT(12 + 3 * hh, j);  // P and O stores complete
                tc_fence_before();
                __syncwarp();  // every lane's P and O stores are complete and fenced
                if (lane == 0) mbar_arrive(bar(G_P_FULL + hh));  // one arrival per warp
                if (r == 0 && half == 0) TG_TRACE_AT(5 + 4 * hh, j);  // P_h(j) stored and signalled
            }
        }
        // ---------------------------------------------------------------- epilogue
        if (threadIdx.x == 0) TG_CTA_STAMP(4);
        const bool oko = ok && mbar_wait_warp(bar(G_O_FULL), 0, abort_flag, status, TG_WHERE_SOFTMAX);
        lred[0 * (2 * BM) + half * BM + r] = l_run0;
        lred[1 * (2 * BM) + half * BM + r] = l_run1;
        ok = !bar_red_or(1, 256, !oko);  // uniform over the 256 softmax threads
        if (ok) tc_fence_after();
        if (threadIdx.x == 0) TG_CTA_STAMP(5);
        // per-head values as scalars: the epilogue loops over the heads without unrolling
        const float l_tot0 = l_run0 + lred[0 * (2 * BM) + (half ^ 1) * BM + r];
        const float l_tot1 = l_run1 + lred[1 * (2 * BM) + (half ^ 1) * BM + r];
        const float m_fin0 = m_run0, m_fin1 = m_run1;
        // Output rows leave through shared memory: each thread stages its half row of both
        // heads in the K buffers (free once every MMA has completed), 16-byte chunks XOR-
        // swizzled by the row so that the staging is conflict-free; then each warp writes 32
        // whole rows of one head with coalesced stores (rows past the sequence end are skipped).
        constexpr int CH = HD * 2 / 16;  // 16-byte chunks per bf16 row
        auto stage_row = [&](int hh, const float* o32, int ch32, float w) {  // 32 columns from ch32 * 32
            uint8_t* stage = smem + L::OFF_K + hh * (BM * HD * 2);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int cidx = ch32 * 4 + k4;
                uint4 v;
                v.x = pack_bf16x2(o32[k4 * 8 + 0] * w, o32[k4 * 8 + 1] * w);
                v.y = pack_bf16x2(o32[k4 * 8 + 2] * w, o32[k4 * 8 + 3] * w);
                v.z = pack_bf16x2(o32[k4 * 8 + 4] * w, o32[k4 * 8 + 5] * w);
                v.w = pack_bf16x2(o32[k4 * 8 + 6] * w, o32[k4 * 8 + 7] * w);
                *reinterpret_cast<uint4*>(stage + r * (HD * 2) + ((cidx ^ (r & (CH - 1))) << 4)) = v;
            }
        };
        auto write_rows = [&]() {  // warp w writes rows 32 (w & 3) .. + 31 of head w >> 2
            asm volatile("bar.sync 1, 256;" ::: "memory");
            const int wh = warp >> 2;
            const uint8_t* stg = smem + L::OFF_K + wh * (BM * HD * 2);
            const int hw = 2 * pair + wh;
#pragma unroll 4
            for (int i = 0; i < 32; ++i) {
                const int rr = q4 * 32 + i;
                if (qt * BM + rr >= Mb) break;
                const uint8_t* src = stg + rr * (HD * 2);
                uint16_t* dst = out + (static_cast<size_t>(seq0 + qt * BM + rr) * Hq + hw) * HD;
                if (HD == 128) {
                    const uint2 v = *reinterpret_cast<const uint2*>(src + (((lane >> 1) ^ (rr & (CH - 1))) << 4) +
                                                                    (lane & 1) * 8);
                    *reinterpret_cast<uint2*>(dst + lane * 4) = v;
                } else {
                    const uint32_t v = *reinterpret_cast<const uint32_t*>(
                        src + (((lane >> 2) ^ (rr & (CH - 1))) << 4) + (lane & 3) * 4);
                    *reinterpret_cast<uint32_t*>(dst + lane * 2) = v;
                }
            }
        };
        if (!split) {
            if (ok) {
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t tO = tmem + lane_addr + 2 * BN + hh * HD + half * (HD / 2);
                    const float lt = hh ? l_tot1 : l_tot0, mf = hh ? m_fin1 : m_fin0;
                    const float inv_l = 1.0f / lt;
#pragma unroll
                    for (int ch = 0; ch < HD / 64; ++ch) {
                        float o[32];
                        tmem_ld32(tO + ch * 32, o);
                        tmem_wait_ld();
                        stage_row(hh, o, half * (HD / 64) + ch, inv_l);
                    }
                    if (valid_row && lse && half == 0)
                        lse[static_cast<size_t>(qg) * Hq + 2 * pair + hh] = (mf + log2f(lt)) / LOG2E;
                }
            }
            write_rows();
        } else {
            // The two KV chunks of a split query tile meet through one counter (taken by
            // thread 0 at the start of its last tile): the first to arrive (0 -> 1) writes its
            // normalised partial (bf16 column pairs, [pair][row] so that a warp's 32 rows are one
            // 128-byte write) and log-sum-exp, then publishes them (+1, release); the second
            // (arrival value 1 or 2) waits, if needed, for that publication (the first is
            // resident and depends on nothing else, so the bounded wait ends), merges the
            // partial with its own O read straight from TMEM, writes the rows and resets the
            // counter.
            const int64_t slot = (static_cast<int64_t>(b) * (Hq / 2) + pair) * ws.slots_per_pair + (qt - C);
            int* cnt = ws.cnt + slot;
            const float my_lse0 = m_fin0 + log2f(l_tot0), my_lse1 = m_fin1 + log2f(l_tot1);
            int* s_last = reinterpret_cast<int*>(smem + L::OFF_MISC + 8);
            if (threadIdx.x == 0) *s_last = ok ? arrival : -1;
            asm volatile("bar.sync 1, 256;" ::: "memory");  // all 256 softmax threads, abort or not
            const int arr = *s_last;
            asm volatile("bar.sync 1, 256;" ::: "memory");  // s_last is read before it is reused
            if (arr == 0) {
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t* po = reinterpret_cast<uint32_t*>(ws.o) +
                                   ((slot * ws.max_nch + chunk) * 2 + hh) * (BM * HD / 2) + r;
                    const uint32_t tO = tmem + lane_addr + 2 * BN + hh * HD + half * (HD / 2);
                    const float inv_l = 1.0f / (hh ? l_tot1 : l_tot0);
#pragma unroll
                    for (int ch = 0; ch < HD / 64; ++ch) {
                        float o[32];
                        tmem_ld32(tO + ch * 32, o);
                        tmem_wait_ld();
                        const int cp0 = (half * (HD / 2) + ch * 32) / 2;  // first column pair
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            po[(cp0 + e) * BM] = pack_bf16x2(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
                    }
                    if (half == 0) ws.lse2[((slot * ws.max_nch + chunk) * 2 + hh) * BM + r] = hh ? my_lse1 : my_lse0;
                }
                if (threadIdx.x == 0) TG_CTA_STAMP(8);
                asm volatile("bar.sync 1, 256;" ::: "memory");  // every partial store is issued
                if (threadIdx.x == 0) {
                    asm volatile("fence.acq_rel.gpu;" ::: "memory");
                    atomicAdd(cnt, 1);  // publish
                }
            } else if (arr > 0) {
                // The acquire load (thread 0; the others follow through the barrier) makes the
                // other chunk's partial visible; it returns at once when that chunk had published
                // before this one arrived (arrival value 2).
                if (threadIdx.x == 0) {
                    int ready = 1;
                    const uint64_t t0 = globaltimer();
                    while (ld_acquire_gpu(cnt) < 3) {
                        if (globaltimer() - t0 > TG_WAIT_TIMEOUT_NS) {
                            *abort_flag = 1;
                            atomicOr(status, TG_DEVICE_TIMEOUT | TG_WHERE_SOFTMAX);
                            ready = 0;
                            break;
                        }
                    }
                    *s_last = ready;
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (threadIdx.x == 0) TG_CTA_STAMP(10);
                if (*s_last) {
#pragma unroll 1
                    for (int hh = 0; hh < 2; ++hh) {
                        const int64_t oidx = (slot * ws.max_nch + (chunk ^ 1)) * 2 + hh;
                        const uint32_t* pt = reinterpret_cast<const uint32_t*>(ws.o) + oidx * (BM * HD / 2) + r;
                        // the other chunk's half row of this head, all loads in flight at once
                        uint32_t pw[HD / 4];
#pragma unroll
                        for (int e = 0; e < HD / 4; ++e) pw[e] = pt[(half * (HD / 4) + e) * BM];
                        const float other_lse = ws.lse2[oidx * BM + r];
                        const float ml = hh ? my_lse1 : my_lse0;
                        // Order-independent merge: this chunk's row is rounded to bf16 exactly as
                        // the other's partial was, each weight depends only on its own chunk's
                        // log-sum-exp and the (commutative) sum, and the two products are added,
                        // so the result does not depend on which chunk arrived first.
                        const float mx = fmaxf(ml, other_lse);
                        const float e_me = ex2_approx(ml - mx), e_ot = ex2_approx(other_lse - mx);
                        const float inv_w = 1.0f / (e_me + e_ot);
                        const float w_me = e_me * inv_w, w_ot = e_ot * inv_w;
                        const float inv_l = 1.0f / (hh ? l_tot1 : l_tot0);
                        const uint32_t tO = tmem + lane_addr + 2 * BN + hh * HD + half * (HD / 2);
#pragma unroll
                        for (int ch = 0; ch < HD / 64; ++ch) {
                            float o[32];
                            tmem_ld32(tO + ch * 32, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const uint32_t w = pw[ch * 16 + e];
                                const uint32_t mine = pack_bf16x2(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
                                o[2 * e] = __fadd_rn(__fmul_rn(w_me, __uint_as_float(mine << 16)),
                                                     __fmul_rn(w_ot, __uint_as_float(w << 16)));
                                o[2 * e + 1] = __fadd_rn(__fmul_rn(w_me, __uint_as_float(mine & 0xFFFF0000u)),
                                                         __fmul_rn(w_ot, __uint_as_float(w & 0xFFFF0000u)));
                            }
                            stage_row(hh, o, half * (HD / 64) + ch, 1.0f);
                        }
                        if (valid_row && lse && half == 0)
                            lse[static_cast<size_t>(qg) * Hq + 2 * pair + hh] = (mx + log2f(e_me + e_ot)) / LOG2E;
                    }
                }
                write_rows();
                if (threadIdx.x == 0) *cnt = 0;  // ready for the next call
            }
            if (threadIdx.x == 0) TG_CTA_STAMP(11);
        }
        if (!split && threadIdx.x == 0) TG_CTA_STAMP(8);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
#ifdef TG_TRACE
    if (threadIdx.x == 0) {
        const unsigned idx = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
        if (idx < 4096) {
            unsigned smid;
            asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
            g_attn_cta[idx * 12 + 0] = trace_t0;
            g_attn_cta[idx * 12 + 6] = globaltimer();
            g_attn_cta[idx * 12 + 7] = smid | (static_cast<unsigned long long>(n_kv) << 32) |
                                      (static_cast<unsigned long long>(split) << 40);
        }
    }
#endif
}

template <int HD>
cudaError_t launch_gqa2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const int32_t* cu_kept,
                        int B, int max_M, int Hq, int Hkv, const int32_t* pos, const int32_t* rank,
                        const GateSet& gates, const float* c, float sm_scale, uint16_t* out, float* lse, void* ws,
                        size_t ws_bytes, bool early, cudaStream_t st) {
    using L = G2Smem<HD>;
    static std::atomic<uint64_t> attr_set{0};
    if (cudaError_t e = ensure_smem_limit(gated_attn_gqa2_kernel<HD>, L::ALLOC, attr_set); e != cudaSuccess)
        return e;
    const int n_qt_max = (max_M + BM - 1) / BM;
    int C = n_qt_max > 0 ? n_qt_max : 1;
    SplitWs sw{};
    if (ws != nullptr) {
        const AttnWsLayout lay = attention_ws_layout(B, max_M, Hq, Hkv, HD, true);
        if (ws_bytes < lay.total) return cudaErrorInvalidValue;
        C = lay.C;
        uint8_t* p = static_cast<uint8_t*>(ws);
        sw.cnt = reinterpret_cast<int*>(p + lay.cnt_off);
        sw.o = reinterpret_cast<float*>(p + lay.o_off);
        sw.lse2 = reinterpret_cast<float*>(p + lay.lse_off);
        sw.max_nch = lay.max_nch;
        sw.slots_per_pair = lay.slots_per_pair;
    }
    const int64_t units = units_below_host(n_qt_max, C);
    dim3 grid(Hq / 2, static_cast<unsigned>(units), B);
    return launch_pdl(gated_attn_gqa2_kernel<HD>, grid, dim3(G2_THREADS), static_cast<size_t>(L::ALLOC), st, tq, tk,
                      tv, cu_kept, pos, rank, gates, c, sm_scale, Hq, Hkv, n_qt_max, C, sw, out, lse,
                      device_status_ptr(), early ? 1 : 0);
}

template <int HD>
cudaError_t launch_tc(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept, int B,
                      int64_t M_total, int max_M, int Hq, int Hkv, const int32_t* pos, const int32_t* rank,
                      const GateSet& gates, const float* c, float sm_scale, uint16_t* out, float* lse, void* ws,
                      size_t ws_bytes, bool early, cudaStream_t st) {
    using L = AttnSmem<HD>;
    static std::atomic<uint64_t> attr_set{0};
    if (cudaError_t e = ensure_smem_limit(gated_attn_tc_kernel<HD>, L::ALLOC, attr_set); e != cudaSuccess)
        return e;
    CUtensorMap tq, tk, tv;
    if (!encode_tmap_2d_bf16(&tq, q, static_cast<uint64_t>(Hq) * HD, static_cast<uint64_t>(M_total),
                             static_cast<uint64_t>(Hq) * HD * 2, 64, BM) ||
        !encode_tmap_2d_bf16(&tk, k, static_cast<uint64_t>(Hkv) * HD, static_cast<uint64_t>(M_total),
                             static_cast<uint64_t>(Hkv) * HD * 2, 64, BN) ||
        !encode_tmap_2d_bf16(&tv, v, static_cast<uint64_t>(Hkv) * HD, static_cast<uint64_t>(M_total),
                             static_cast<uint64_t>(Hkv) * HD * 2, 64, BN))
        return cudaErrorInvalidValue;
    if constexpr (HD <= 128) {  // two heads of 256 would need 768 TMEM columns
        if ((Hq / Hkv) % 2 == 0) {
            // the persistent kernel needs the workspace for its unit counter
            if (ws != nullptr && !attention_per_unit_kernel(B, gates.n)) {
                const cudaError_t e = launch_attention_persistent(tq, tk, tv, cu_kept, B, M_total, max_M, Hq, Hkv,
                                                                  HD, pos, rank, gates, c, sm_scale, out, lse, ws,
                                                                  ws_bytes, early, st);
                if (e != cudaErrorNotSupported || gates.n == 0) return e;
            }
            if (gates.n == 0) return cudaErrorNotSupported;
            return launch_gqa2<HD>(tq, tk, tv, cu_kept, B, max_M, Hq, Hkv, pos, rank, gates, c, sm_scale, out, lse,
                                   ws, ws_bytes, early, st);
        }
    }
    if (gates.n == 0) return cudaErrorNotSupported;
    int* status = device_status_ptr();
    const int n_qt_max = (max_M + BM - 1) / BM;
    dim3 grid(Hq, n_qt_max, B);
    return launch_pdl(gated_attn_tc_kernel<HD>, grid, dim3(NUM_THREADS), static_cast<size_t>(L::ALLOC), st, tq, tk, tv,
                      cu_kept, pos, rank, gates, c, sm_scale, Hq, Hkv, n_qt_max, out, lse, status);
}

}  // namespace

#ifdef TG_TRACE
extern "C" __attribute__((visibility("default"))) int tg_trace_read_attention(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, g_attn_trace, sizeof(g_attn_trace)) == cudaSuccess ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int tg_trace_read_attention_ctas(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, g_attn_cta, sizeof(g_attn_cta)) == cudaSuccess ? 0 : 1;
}
#endif

cudaError_t launch_gated_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept,
                                   int B, int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                                   const int32_t* rank, const GateSet& gates, const float* c, float sm_scale,
                                   uint16_t* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t st,
                                   bool inputs_ready) {
    if (M_total == 0 || B == 0) return cudaSuccess;
    if (gates.n < 0 || gates.n > kMaxGates) return cudaErrorInvalidValue;  // 0: no gate (plain attention)
    if (d == 64)
        return launch_tc<64>(q, k, v, cu_kept, B, M_total, max_M, Hq, Hkv, pos, rank, gates, c, sm_scale, out, lse,
                             ws, ws_bytes, inputs_ready, st);
    if (d == 256)
        return launch_tc<256>(q, k, v, cu_kept, B, M_total, max_M, Hq, Hkv, pos, rank, gates, c, sm_scale, out, lse,
                              ws, ws_bytes, inputs_ready, st);
    return launch_tc<128>(q, k, v, cu_kept, B, M_total, max_M, Hq, Hkv, pos, rank, gates, c, sm_scale, out, lse, ws,
                          ws_bytes, inputs_ready, st);
}

namespace {
// 0: by the batch, 1: persistent, 2: one CTA per unit (read on every call, so that a process
// may switch between calls)
int attention_kernel_override() {
    const char* e = std::getenv("TG_ATTENTION_KERNEL");
    if (e == nullptr) return 0;
    if (std::strcmp(e, "persistent") == 0) return 1;
    if (std::strcmp(e, "per_unit") == 0) return 2;
    return 0;
}
}  // namespace

bool attention_per_unit_kernel(int B, int n_gates) {
    const int choice = attention_kernel_override();
    if (n_gates <= 0 || choice == 1) return false;
    return choice == 2 || B == 1;
}

int64_t units_below_host(int x, int C) {
    const int64_t a = x / C, r = x % C;
    return C * a * (a + 1) / 2 + r * (a + 1);
}

// KV chunk length (in 128-key tiles) of the causal work split.  Query tile qt
// of a sequence needs qt + 1 KV tiles; a chunk length C < n_qt cuts the query
// tiles past C into two units ([0, C) and [C, qt + 1)), C >= ceil(n_qt / 2) so
// that two always suffice.  A unit costs about F + n_kv tile pairs on one SM,
// F being the part a unit adds beyond its tiles.  With the persistent kernel
// a CTA loads the next unit while it finishes the current one, so F is about
// one tile pair (the epilogue and the merge); the one-CTA-per-unit kernel pays
// about 9 us of set-up, first loads and epilogue against 2.6-2.9 us per tile
// pair, plus the merge of a split tile: F = 4.0, the value that measured best
// among 2.0, 2.5, 3.1, 4.0 and 5.0 at 32k tokens, K = 2000.  Units are taken
// heaviest first, which is longest-processing-time scheduling, so C is the
// candidate whose LPT makespan over the SMs is smallest (all sequences taken
// at max_M, the bound the host knows); ties go to the larger C (fewer units).
int attention_kv_chunk(int B, int max_M, int Hq, int Hkv, bool have_ws, bool per_unit) {
    const int n_qt = (max_M + BM - 1) / BM;
    if (!have_ws || (Hq / Hkv) % 2 != 0 || n_qt < 4) return n_qt > 0 ? n_qt : 1;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
    const int64_t tiles = static_cast<int64_t>(B) * (Hq / 2);  // (sequence, head pair) instances
    // many waves (each SM's share at least twice the longest unit): splitting only adds fixed costs
    if (static_cast<double>(tiles) * n_qt * (n_qt + 1) / 2.0 >= 2.0 * sms * n_qt) return n_qt;
    // the choice depends on the shape alone: remember it (a few hundred heap operations
    // per candidate would otherwise run on every call)
    static std::mutex mu;
    static std::map<std::tuple<int, int, int, int, int>, int> memo;
    const double F = per_unit ? 4.0 : 1.0;
    const auto key = std::make_tuple(B, n_qt, Hq / 2, sms, F > 2.0 ? 1 : 0);
    {
        std::lock_guard<std::mutex> lk(mu);
        const auto it = memo.find(key);
        if (it != memo.end()) return it->second;
    }
    int best_c = n_qt;
    double best = 1e300;
    std::vector<double> cost;
    std::vector<double> load;
    for (int C = n_qt; C >= (n_qt + 1) / 2; --C) {
        cost.clear();
        for (int qt = 0; qt < n_qt; ++qt) {
            const int n = qt + 1;
            if (n <= C) {
                cost.push_back(F + n);
            } else {
                cost.push_back(F + C);
                cost.push_back(F + (n - C));
            }
        }
        std::sort(cost.begin(), cost.end(), [](double a, double b) { return a > b; });
        // LPT over `sms` machines of the units of all instances (each instance has the same list)
        load.assign(static_cast<size_t>(sms), 0.0);
        std::priority_queue<double, std::vector<double>, std::greater<double>> q(load.begin(), load.end());
        for (double c : cost)
            for (int64_t i = 0; i < tiles; ++i) {
                const double t = q.top();
                q.pop();
                q.push(t + c);
            }
        double mk = 0.0;
        while (!q.empty()) {
            mk = q.top();
            q.pop();
        }
        if (mk < best - 1e-9) {
            best = mk;
            best_c = C;
        }
    }
    std::lock_guard<std::mutex> lk(mu);
    if (memo.size() > 256) memo.clear();
    memo[key] = best_c;
    return best_c;
}

AttnWsLayout attention_ws_layout(int B, int max_M, int Hq, int Hkv, int d, bool per_unit) {
    AttnWsLayout L;
    const int n_qt = (max_M + BM - 1) / BM;
    L.C = n_qt > 0 ? n_qt : 1;
    if (B <= 0 || n_qt <= 0 || Hkv <= 0 || (Hq / Hkv) % 2 != 0 || d > 128) return L;  // one-head kernel: none
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    L.C = attention_kv_chunk(B, max_M, Hq, Hkv, true, per_unit);
    L.total = 256;  // the unit counters of the persistent kernel
    if (L.C < n_qt) {
        L.max_nch = (n_qt + L.C - 1) / L.C;
        L.slots_per_pair = n_qt - L.C;
        L.slots = static_cast<int64_t>(B) * (Hq / 2) * L.slots_per_pair;
        L.cnt_off = 256;
        L.o_off = al(L.cnt_off + static_cast<size_t>(L.slots) * 2 * sizeof(int));
        L.lse_off = L.o_off + static_cast<size_t>(L.slots) * L.max_nch * 2 * BM * d * sizeof(float);
        L.total = L.lse_off + static_cast<size_t>(L.slots) * L.max_nch * 2 * BM * sizeof(float);
        L.zero_bytes = L.o_off;
    }
    return L;
}

// The workspace serves either two-head kernel (their chunk choices differ): the larger need.
size_t attention_workspace_bytes(int B, int max_M, int Hq, int Hkv, int d) {
    return std::max(attention_ws_layout(B, max_M, Hq, Hkv, d, false).total,
                    attention_ws_layout(B, max_M, Hq, Hkv, d, true).total);
}

// ---------------------------------------------------------------------------
// Allocation-free variant of tg_gated_attention.
//
// Some callers cannot allocate device memory at the point where they run the
// attention: a serving engine that reserves every byte of HBM at start-up and
// hands out only fixed buffers, or code running inside a host runtime that
// owns the allocator and offers no way to ask it for scratch.  For them the
// causal-split scratch lives in this fixed array, part of the library's
// device image: every GPU that loads the library holds it until the process
// exits.  All calls on a device share it, and it keeps the last call's
// contents, so calls whose executions overlap on the GPU race on it.
static __device__ __align__(256) unsigned char g_noalloc_attn_scratch[TG_NOALLOC_ATTENTION_SCRATCH_BYTES];

namespace {
constexpr int kNoAllocMaxDevices = 64;
void* g_noalloc_scratch_ptr[kNoAllocMaxDevices] = {};
std::mutex g_noalloc_mu;
}  // namespace

// Device address of the array on the current device; the first call on each
// device resolves it (in host code the array's name is only a stand-in).
cudaError_t noalloc_attention_scratch(void** ptr) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_scratch_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_attn_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_scratch_ptr[dev] = p;
    }
    *ptr = g_noalloc_scratch_ptr[dev];
    return cudaSuccess;
}

cudaError_t launch_gated_attention_noalloc(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                           const int32_t* cu_kept, int B, int64_t M_total, int max_M, int Hq, int Hkv,
                                           int d, const int32_t* pos, const int32_t* rank, const GateSet& gates,
                                           const float* c, float sm_scale, uint16_t* out, float* lse,
                                           cudaStream_t st) {
    const size_t need = attention_workspace_bytes(B, max_M, Hq, Hkv, d);
    if (need > TG_NOALLOC_ATTENTION_SCRATCH_BYTES) return cudaErrorInvalidValue;  // the API rejects it first
    void* ws = nullptr;
    cudaError_t e = noalloc_attention_scratch(&ws);
    if (e != cudaSuccess) return e;
    if (need > 0) {
        // the counters must start at zero: the last call may have stopped early
        e = cudaMemsetAsync(ws, 0,
                            std::max(attention_ws_layout(B, max_M, Hq, Hkv, d, false).zero_bytes,
                                     attention_ws_layout(B, max_M, Hq, Hkv, d, true).zero_bytes),
                            st);
        if (e != cudaSuccess) return e;
    }
    return launch_gated_attention(q, k, v, cu_kept, B, M_total, max_M, Hq, Hkv, d, pos, rank, gates, c, sm_scale,
                                  out, lse, need > 0 ? ws : nullptr, need, st);
}

}  // namespace tg
