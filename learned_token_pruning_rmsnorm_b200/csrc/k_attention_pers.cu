// Stage 4 of the gated prefill, persistent form: token-gated causal GQA
// attention over the kept tokens (TokenGate AI summary, "Key Contributions" 2
// and 3) for head_dim 64 and 128, GQA groups of even size and one gate, and
// the same kernel without the gate (bias 0, temperature 1: ordinary causal
// attention, the unpruned baseline the pages compare against).
//
//   logit[q,j] = (q.k_j * sm_scale + softplus(g_h) * gls_j) / tau[q,h]
//   tau[q,h]   = 1 + c_h * ln(pos_q / rank_q)
//
// One CTA per SM.  A unit is two query heads of one KV head (sharing every K/V
// tile) times one 128-row query tile, or one causal chunk of a long tile (the
// split of k_attention.cu, merged through the caller's workspace).  The first
// unit of a CTA is its block index; later ones come from a global counter, so
// units are taken in order of decreasing cost by whichever SM frees up first,
// and a CTA that starts late (its SM still busy with the previous kernel) simply
// takes fewer.  While a CTA finishes one unit it already loads the next one's
// Q and first K/V tiles, so set-up and first loads are paid once per SM.
//
// 384 threads, three warpgroups:
//   warps 0-3   softmax of head 0 of the pair: thread r owns query row r (TMEM
//               lane r) and all 128 keys of a tile, so the row maximum needs no
//               exchange between threads
//   warps 4-7   softmax of head 1, concurrently: one head's exponentials,
//               loads and stores overlap the other's
//   warp 8      TMA producer: Q of both heads once per unit, K/V tiles of 128
//               keys through a two-stage ring, the gate-bias operand rows, the
//               next unit's number
//   warp 9      MMA issuer (one thread):  S0(j) S1(j) | PV0(j) S0(j+1) |
//               PV1(j) S1(j+1) | ...   (P_h is read from TMEM, written by the
//               softmax as bf16 over the first 64 columns of S_h)
//   warps 10-11 idle (they complete the producer/MMA warpgroup, whose
//               registers are handed to the softmax warpgroups)
// TMEM (512 columns): S0 | S1 | O0 | O1.  Each head's epilogue reads its O
// from TMEM and writes its rows while the other head still computes and the
// tensor core already runs the next unit's first S.

#include "tg_attn_util.cuh"

namespace tg {
namespace {

using namespace sm100;
using namespace attn;

constexpr int PT_THREADS = 384;
constexpr int PT_LAUNCH_REGS = 168;   // registers per thread at launch (65536 / 384, rounded down to 8)
constexpr int PT_SOFTMAX_REGS = 200;  // after the hand-over: 256 x 200 + 128 x 104 = 384 x 168
constexpr int PT_OTHER_REGS = 104;
constexpr int PT_RING = 8;            // unit numbers in flight between the producer and the consumers
// Of every 32 columns of a tile, the first 4 * PT_POLY_QUADS take their exponentials on the
// FMA pipe (exp2_poly_x2) instead of the special-function unit, except in the diagonal tile,
// whose masked elements must come out exactly 0.
#ifndef TG_EXP2_POLY_QUADS
#define TG_EXP2_POLY_QUADS 0
#endif
constexpr int PT_POLY_QUADS = TG_EXP2_POLY_QUADS;
static_assert(PT_POLY_QUADS >= 0 && PT_POLY_QUADS <= 8, "quads of 4 columns per 32");
static_assert(256 * PT_SOFTMAX_REGS + 128 * PT_OTHER_REGS <= PT_THREADS * PT_LAUNCH_REGS, "register hand-over");

template <int HD>
struct PtSmem {
    static constexpr int TILE_Q = BM * HD * 2;
    static constexpr int TILE_KV = BN * HD * 2;
    static constexpr int EXT = BM * 16 * 2;  // one bias k-step operand: 128 rows x 16 bf16
    static constexpr int OFF_Q = 0;                      // [head]
    static constexpr int OFF_K = OFF_Q + 2 * TILE_Q;     // [stage]
    static constexpr int OFF_V = OFF_K + 2 * TILE_KV;    // [stage]
    static constexpr int OFF_QX = OFF_V + 2 * TILE_KV;   // [head]
    static constexpr int OFF_KX = OFF_QX + 2 * EXT;      // [stage]
    static constexpr int OFF_BAR = OFF_KX + 2 * EXT;
    static constexpr int NUM_BARS = 32;
    // tmem slot, abort flag, one arrival slot per head, the unit ring
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int BYTES = OFF_MISC + 16 + 4 * PT_RING;
    static constexpr int ALLOC = BYTES + 1024;
    static_assert(ALLOC <= 227 * 1024, "shared memory");
};

enum : int {
    T_Q_FULL = 0, T_Q_EMPTY = 1, T_K_FULL = 2, T_K_EMPTY = 4, T_V_FULL = 6, T_V_EMPTY = 8, T_S_FULL = 10,
    T_P_FULL = 12, T_O_FULL = 14, T_UNIT = 16, T_DRAIN = 16 + PT_RING
};
static_assert(T_DRAIN < PtSmem<128>::NUM_BARS, "barrier slots");

// One unit of work: (sequence b, head pair, query tile, KV chunk).
struct Unit {
    int b, pair, qt, chunk, kv0, n_kv, seq0, Mb;
    bool split;
};

// Global unit number -> unit, or false for a number that names no work (a sequence
// with fewer units than the longest).  Numbering: u = (v * B + b) * pairs + pair, v the
// unit's place in its sequence's decreasing-cost order, so all sequences' heaviest
// units come first.
// In TG_DEBUG builds a sequence whose rows [cu_kept[b], cu_kept[b+1]) do not lie inside
// [0, M_total) is recorded in the status word and skipped (every role decodes the same way).
__device__ __forceinline__ bool decode_unit(int64_t u, int pairs, int B, const int32_t* cu_kept, int C_all,
                                            Unit* U, int64_t M_total, int* status) {
    const int pair = static_cast<int>(u % pairs);
    const int64_t t = u / pairs;
    const int b = static_cast<int>(t % B);
    const int64_t v = t / B;
    const int seq0 = cu_kept[b];
    const int Mb = cu_kept[b + 1] - seq0;
    const int n_qt = (Mb + BM - 1) / BM;
    if (n_qt <= 0) return false;
    if (!TG_DEBUG_CHECK(seq0 >= 0 && static_cast<int64_t>(seq0) + Mb <= M_total, status, TG_WHERE_ATTENTION))
        return false;
    const int C = min(C_all, n_qt);
    if (v >= units_below(n_qt, C)) return false;
    int qt, chunk;
    unit_tile(v, n_qt, C, &qt, &chunk);
    U->b = b;
    U->pair = pair;
    U->qt = qt;
    U->chunk = chunk;
    U->kv0 = chunk * C;
    U->n_kv = min(qt + 1, U->kv0 + C) - U->kv0;
    U->seq0 = seq0;
    U->Mb = Mb;
    U->split = (qt + C) / C > 1;
    return true;
}

__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Optional device trace (builds with -DTG_TRACE only): per-CTA globaltimer stamps of the
// hand-offs of the first unit and of the whole CTA, with the SM id and the unit count.
#ifdef TG_TRACE
__device__ unsigned long long g_pers_pipe[16 * 64];  // clock64 of pipeline points of CTA 0, first 64 tiles
#define PT_PIPE(point, j)                                                                      \
    do {                                                                                       \
        if (blockIdx.x == 0 && (j) < 64) g_pers_pipe[(point) * 64 + (j)] = clock64();         \
    } while (0)
__device__ unsigned long long g_pers_trace[1024 * 16];
// per CTA, first 4 units: ring read, loop end, O full, epilogue end, info, arrival, S0 seen
__device__ unsigned long long g_pers_units[1024 * 4 * 8];
#define PT_UNIT(uc, slot, val)                                                                  \
    do {                                                                                        \
        if (threadIdx.x == 0 && blockIdx.x < 1024 && (uc) < 4)                                  \
            g_pers_units[(blockIdx.x * 4 + (uc)) * 8 + (slot)] = (val);                         \
    } while (0)
#define PT_STAMP(slot, cond)                                                             \
    do {                                                                                 \
        if ((cond) && blockIdx.x < 1024) g_pers_trace[blockIdx.x * 16 + (slot)] = globaltimer(); \
    } while (0)
#else
#define PT_STAMP(slot, cond) \
    do {                     \
    } while (0)
#define PT_PIPE(point, j) \
    do {                  \
    } while (0)
#define PT_UNIT(uc, slot, val) \
    do {                       \
    } while (0)
#endif

template <int HD, bool GATED>
__global__ void __launch_bounds__(PT_THREADS, 1)
gated_attn_pers_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const int32_t* __restrict__ cu_kept,
                       const int32_t* __restrict__ pos, const int32_t* __restrict__ rank, const GateSet gates,
                       const float* __restrict__ c, float sm_scale, int Hq, int Hkv, int B, int64_t M_total,
                       int kv_chunk, int64_t total_units, SplitWs ws,
                       int* __restrict__ sched, uint16_t* __restrict__ out, float* __restrict__ lse,
                       int* __restrict__ status, int early, int wide_out) {
    using L = PtSmem<HD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pairs = Hq / 2;
    const int group = Hq / Hkv;
    PT_STAMP(0, threadIdx.x == 0);
    // `early`: q, k, v, g, c and cu_kept were complete before the preceding kernel started
    // (the caller's guarantee), so set-up, Q and the first K/V tiles go ahead while that
    // kernel runs; gls, pos, rank, the scratch and the unit counter are touched only after
    // the wait, which each role executes before its first such access.
    if (!early) {
        pdl_wait();
        pdl_trigger();
    }

    const uint32_t sbase = smem_u32(smem);
    const uint32_t sQ = sbase + L::OFF_Q, sK0 = sbase + L::OFF_K, sV0 = sbase + L::OFF_V;
    const uint32_t sQX = sbase + L::OFF_QX, sKX = sbase + L::OFF_KX;
    auto bar = [&](int i) { return sbase + L::OFF_BAR + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
    volatile int* s_arr = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 8);  // [head]
    volatile int* ring = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 16);  // [PT_RING]

    if (GATED) {
        // Gate i owns columns 4i..4i+3 of the bias k-step; the producer writes columns 0..7
        // (gates 0 and 1, zeros for an absent gate 1) and, with three or four gates, columns
        // 8..15, which otherwise stay the zeros written here
        for (int i = threadIdx.x; i < 4 * (BM / 8) * 8; i += blockDim.x) {
            const int tile = i / ((BM / 8) * 8), rem = i % ((BM / 8) * 8);
            *reinterpret_cast<uint4*>(smem + L::OFF_QX + tile * L::EXT + (rem >> 3) * 256 + 128 + (rem & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }
    if (threadIdx.x == 0) {
        mbar_init(bar(T_Q_FULL), GATED ? 2 : 1);  // the Q bytes (+ the producer's bias operand rows)
        mbar_init(bar(T_Q_EMPTY), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(T_K_FULL + s), GATED ? 2 : 1);  // the K bytes (+ the K_ext rows)
            mbar_init(bar(T_K_EMPTY + s), 1);
            mbar_init(bar(T_V_FULL + s), 1);
            mbar_init(bar(T_V_EMPTY + s), 1);
            mbar_init(bar(T_S_FULL + s), 1);
            mbar_init(bar(T_P_FULL + s), 4);  // one arrival per softmax warp of the head
            mbar_init(bar(T_O_FULL + s), 1);
        }
        for (int i = 0; i < PT_RING; ++i) mbar_init(bar(T_UNIT + i), 1);
        mbar_init(bar(T_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    PT_STAMP(1, threadIdx.x == 0);

    // The producer / MMA warpgroup hands most of its registers to the softmax warpgroups;
    // each role's code sits inside the branch that set its register budget.
    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(PT_OTHER_REGS));
    if (warp == 8) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
        }
        bool waited = !early;
        auto wait_inputs = [&]() {
            if (!waited) {
                pdl_wait();
                waited = true;
                // dependents are released only now, once the preceding kernel has completed,
                // so a following row gather may read the compaction map straight away
                if (lane == 0) pdl_trigger();
            }
        };
        int q_issued = 0, k_issued[2] = {0, 0}, v_issued[2] = {0, 0};
        int t = 0, uc = 0;
        int64_t unit = blockIdx.x;
        bool ok = true;
        while (ok) {
            Unit U{};
            bool have = false;
            while (unit < total_units) {
                if (decode_unit(unit, pairs, B, cu_kept, kv_chunk, &U, M_total, status)) {
                    have = true;
                    break;
                }
                wait_inputs();  // the counter is reset by the previous launch's last CTA
                int64_t n = 0;
                if (lane == 0) n = static_cast<int64_t>(gridDim.x) + atomicAdd(sched, 1);
                unit = __shfl_sync(0xffffffffu, n, 0);
            }
            if (lane == 0) {
                ring[uc % PT_RING] = have ? static_cast<int>(unit) : -1;
                mbar_arrive(bar(T_UNIT + uc % PT_RING));
            }
            if (!have) break;
            const int hk = (2 * U.pair) / group;
            // Q of both heads and their bias operand rows: the previous unit's S products
            // must have read both
            if (uc > 0 && !mbar_wait_warp(bar(T_Q_EMPTY), (uc - 1) & 1, abort_flag, status, TG_WHERE_PRODUCER)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                mbar_expect_tx(bar(T_Q_FULL), 2 * BM * HD * 2);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int hf = 0; hf < HD / 64; ++hf)
                        tma_load_2d(sQ + hh * L::TILE_Q + hf * BM * 128, &tmQ, (2 * U.pair + hh) * HD + hf * 64,
                                    U.seq0 + U.qt * BM, bar(T_Q_FULL));
                ++q_issued;
                PT_STAMP(2, uc == 0);
            }
            if (GATED) {
                // Q_ext row of head h: gate i's columns hold (bh, bl, bh, bl), the bf16 high
                // and low parts of softplus(g_i[h]) / sm_scale; lane l writes rows 4l..4l+3
                // of both heads
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int hq = 2 * U.pair + hh;
                    auto hl_of = [&](const float* gp) { return bf16_hi_lo(softplus_f(__ldg(gp + hq)) / sm_scale); };
                    const uint32_t h0 = hl_of(gates.g[0]);
                    const uint32_t h1 = gates.n > 1 ? hl_of(gates.g[1]) : 0u;
                    const uint32_t h2 = gates.n > 2 ? hl_of(gates.g[2]) : 0u;
                    const uint32_t h3 = gates.n > 3 ? hl_of(gates.g[3]) : 0u;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = lane * 4 + i;
                        uint8_t* row = smem + L::OFF_QX + hh * L::EXT + (r >> 3) * 256 + (r & 7) * 16;
                        *reinterpret_cast<uint4*>(row) = make_uint4(h0, h0, h1, h1);
                        if (gates.n > 2) *reinterpret_cast<uint4*>(row + 128) = make_uint4(h2, h2, h3, h3);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(T_Q_FULL));
            }
            auto load_k = [&](int s, int j) {
                mbar_expect_tx(bar(T_K_FULL + s), BN * HD * 2);
#pragma unroll
                for (int hf = 0; hf < HD / 64; ++hf)
                    tma_load_2d(sK0 + s * L::TILE_KV + hf * BN * 128, &tmK, hk * HD + hf * 64,
                                U.seq0 + (U.kv0 + j) * BN, bar(T_K_FULL + s));
                ++k_issued[s];
            };
            auto load_v = [&](int s, int j) {
                mbar_expect_tx(bar(T_V_FULL + s), BN * HD * 2);
#pragma unroll
                for (int hf = 0; hf < HD / 64; ++hf)
                    tma_load_2d(sV0 + s * L::TILE_KV + hf * BN * 128, &tmV, hk * HD + hf * 64,
                                U.seq0 + (U.kv0 + j) * BN, bar(T_V_FULL + s));
                ++v_issued[s];
            };
            // K/V tiles through the two-stage ring (t counts tiles over all units).  The CTA's
            // first two tiles' copies leave at once (t = 0: both stages are free): before the
            // wait in an early launch, and before the first bias loads in every launch.
            const int pre = t == 0 ? min(U.n_kv, 2) : 0;
            if (lane == 0)
                for (int j = 0; j < pre; ++j) {
                    load_k((t + j) & 1, j);
                    load_v((t + j) & 1, j);
                }
            for (int j = 0; j < U.n_kv; ++j, ++t) {
                const int s = t & 1;
                if (j >= pre) {
                    if (t >= 2 &&
                        !mbar_wait_warp(bar(T_K_EMPTY + s), ((t - 2) >> 1) & 1, abort_flag, status, TG_WHERE_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) load_k(s, j);
                }
                if (GATED) {
                    wait_inputs();  // gls (the compaction map) from here on
                    // K_ext row of key k: gate i's columns hold (gh, gh, gl, gl), the bf16 high
                    // and low parts of gls_i[k] (0 past the sequence end); lane l writes keys
                    // 4l..4l+3
                    const int key0 = (U.kv0 + j) * BN + lane * 4;
                    auto kx_of = [&](const float* gp, int i) {
                        const float gv = key0 + i < U.Mb ? ldg_early(gp + U.seq0 + key0 + i) : 0.f;
                        const uint32_t hl = bf16_hi_lo(gv);
                        return make_uint2(__byte_perm(hl, 0u, 0x1010), __byte_perm(hl, 0u, 0x3232));
                    };
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = lane * 4 + i;
                        uint8_t* row = smem + L::OFF_KX + s * L::EXT + (r >> 3) * 256 + (r & 7) * 16;
                        const uint2 k0 = kx_of(gates.gls[0], i);
                        const uint2 k1 = gates.n > 1 ? kx_of(gates.gls[1], i) : make_uint2(0u, 0u);
                        *reinterpret_cast<uint4*>(row) = make_uint4(k0.x, k0.y, k1.x, k1.y);
                        if (gates.n > 2) {
                            const uint2 k2 = kx_of(gates.gls[2], i);
                            const uint2 k3 = gates.n > 3 ? kx_of(gates.gls[3], i) : make_uint2(0u, 0u);
                            *reinterpret_cast<uint4*>(row + 128) = make_uint4(k2.x, k2.y, k3.x, k3.y);
                        }
                    }
                    fence_proxy_async_smem();  // K_ext is read by the tensor core (async proxy)
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar(T_K_FULL + s));
                }
                if (j >= pre) {
                    if (t >= 2 &&
                        !mbar_wait_warp(bar(T_V_EMPTY + s), ((t - 2) >> 1) & 1, abort_flag, status, TG_WHERE_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) load_v(s, j);
                }
            }
            if (!ok) break;
            ++uc;
            wait_inputs();
            int64_t n = 0;
            if (lane == 0) n = static_cast<int64_t>(gridDim.x) + atomicAdd(sched, 1);
            unit = __shfl_sync(0xffffffffu, n, 0);
        }
        if (lane == 0 && *abort_flag) {
            // let every copy this thread started land before the CTA exits
            if (q_issued) drain_wait(bar(T_Q_FULL), (q_issued - 1) & 1, status);
            for (int s = 0; s < 2; ++s) {
                if (k_issued[s]) drain_wait(bar(T_K_FULL + s), (k_issued[s] - 1) & 1, status);
                if (v_issued[s]) drain_wait(bar(T_V_FULL + s), (v_issued[s] - 1) & 1, status);
            }
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, HD, true);
            // Matrix descriptors are built once; a k-step's operand is the same descriptor with
            // its byte offset / 16 added to the start-address field (the offsets stay inside
            // shared memory, so the 14-bit field never carries).  One thread issues every MMA,
            // and building each descriptor from scratch would slow it below the tensor pipe.
            const uint64_t qdesc[2] = {smem_desc_sw128(sQ, 16, 1024), smem_desc_sw128(sQ + L::TILE_Q, 16, 1024)};
            const uint64_t kdesc[2] = {smem_desc_sw128(sK0, 16, 1024), smem_desc_sw128(sK0 + L::TILE_KV, 16, 1024)};
            const uint64_t vdesc[2] = {smem_desc_sw128(sV0, BN * 128, 1024),
                                       smem_desc_sw128(sV0 + L::TILE_KV, BN * 128, 1024)};
            const uint64_t qxdesc = smem_desc_noswz(sQX, 128, 256), kxdesc = smem_desc_noswz(sKX, 128, 256);
            auto issue_s = [&](int hh, int s) {
                const uint64_t qd = qdesc[hh], kd = kdesc[s];
#pragma unroll
                for (int kk = 0; kk < HD / 16; ++kk) {
                    const uint32_t off_q = (kk >> 2) * (BM * 128) + (kk & 3) * 32;
                    const uint32_t off_k = (kk >> 2) * (BN * 128) + (kk & 3) * 32;
                    mma_bf16_ss(tmem + hh * BN, qd + (off_q >> 4), kd + (off_k >> 4), idesc_qk, kk > 0 ? 1u : 0u);
                }
                if (GATED)  // + bscale_h * gls_j: the bias k-step (no-swizzle tiles, K cores 128 B apart)
                    mma_bf16_ss(tmem + hh * BN, qxdesc + ((hh * L::EXT) >> 4), kxdesc + ((s * L::EXT) >> 4), idesc_qk,
                                1u);
            };
            auto issue_pv = [&](int hh, int s, bool acc) {
                const uint64_t vd = vdesc[s];
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    mma_bf16_ts(tmem + 2 * BN + hh * HD, tmem + hh * BN + kk * 8, vd + ((kk * 16 * 128) >> 4),
                                idesc_pv, (acc || kk > 0) ? 1u : 0u);
            };
            int uc = 0, t = 0, it = 0;
            bool ok = true;
            while (ok) {
                ok = mbar_wait(bar(T_UNIT + uc % PT_RING), (uc / PT_RING) & 1, abort_flag, status, TG_WHERE_MMA);
                if (!ok) break;
                const int unit = ring[uc % PT_RING];
                if (unit < 0) break;
                Unit U{};
                decode_unit(unit, pairs, B, cu_kept, kv_chunk, &U, M_total, status);
                ok = mbar_wait(bar(T_Q_FULL), uc & 1, abort_flag, status, TG_WHERE_MMA);
                PT_STAMP(3, uc == 0);
                ok = ok && mbar_wait(bar(T_K_FULL + (t & 1)), (t >> 1) & 1, abort_flag, status, TG_WHERE_MMA);
                PT_STAMP(4, uc == 0);
                if (!ok) break;
                tc_fence_after();
                // S_h(0) of this unit: S_h's last reader (PV_h of the previous unit's last tile)
                // was issued before by this thread, and tcgen05 operations execute in order
                issue_s(0, t & 1);
                mma_commit(bar(T_S_FULL + 0));
                issue_s(1, t & 1);
                mma_commit(bar(T_S_FULL + 1));
                mma_commit(bar(T_K_EMPTY + (t & 1)));
                if (U.n_kv == 1) mma_commit(bar(T_Q_EMPTY));
                for (int j = 0; j < U.n_kv; ++j) {
                    const int s = t & 1;
                    const bool more = j + 1 < U.n_kv;
                    ok = mbar_wait(bar(T_V_FULL + s), (t >> 1) & 1, abort_flag, status, TG_WHERE_MMA) &&
                         mbar_wait(bar(T_P_FULL + 0), it & 1, abort_flag, status, TG_WHERE_MMA);
                    if (!ok) break;
                    tc_fence_after();
                    PT_PIPE(0, it);
                    issue_pv(0, s, j > 0);
                    if (more) {
                        ok = mbar_wait(bar(T_K_FULL + (s ^ 1)), ((t + 1) >> 1) & 1, abort_flag, status, TG_WHERE_MMA);
                        if (!ok) break;
                        tc_fence_after();
                        PT_PIPE(2, it);
                        issue_s(0, s ^ 1);
                        mma_commit(bar(T_S_FULL + 0));
                    } else {
                        mma_commit(bar(T_O_FULL + 0));
                    }
                    ok = mbar_wait(bar(T_P_FULL + 1), it & 1, abort_flag, status, TG_WHERE_MMA);
                    if (!ok) break;
                    tc_fence_after();
                    PT_PIPE(1, it);
                    issue_pv(1, s, j > 0);
                    mma_commit(bar(T_V_EMPTY + s));
                    if (more) {
                        issue_s(1, s ^ 1);
                        mma_commit(bar(T_S_FULL + 1));
                        mma_commit(bar(T_K_EMPTY + (s ^ 1)));
                        if (j + 2 == U.n_kv) mma_commit(bar(T_Q_EMPTY));  // the unit's last S products
                    } else {
                        mma_commit(bar(T_O_FULL + 1));
                    }
                    ++t;
                    ++it;
                }
                ++uc;
            }
            // every MMA (and the barrier arrivals its commits trigger) lands before the CTA exits
            mma_commit(bar(T_DRAIN));
            drain_wait(bar(T_DRAIN), 0, status);
        }
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(PT_SOFTMAX_REGS));
        // ---------------------------------------------------------------- softmax, warps 0-7
        // Warpgroup h = warp / 4 takes head h of the pair; thread r = 32 (warp % 4) + lane
        // owns query row r (TMEM lane r) and every key of a tile.  S already holds
        // s + bscale_h * gls_j (the bias k-step), so in log2 units the logit is
        // x = alpha_q * S with alpha_q = sm_scale * log2(e) / tau_q: one FMA per score with
        // the running max folded in, issued as f32x2 pairs.
        const int h = warp >> 2, q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
        const uint32_t tS = tmem + lane_addr + h * BN;
        const uint32_t tO = tmem + lane_addr + 2 * BN + h * HD;
        // Every decision to leave is taken by the whole warpgroup at a reducing barrier (its
        // own, id 1 + h), so that its four warps always meet at the split epilogue's barriers.
        const int bid = 1 + h;
        bool waited = !early;
        int uc = 0, it = 0;
        for (;;) {
            const bool okr =
                mbar_wait_warp(bar(T_UNIT + uc % PT_RING), (uc / PT_RING) & 1, abort_flag, status, TG_WHERE_SOFTMAX);
            if (bar_red_or(bid, 128, !okr)) break;
            const int unit = ring[uc % PT_RING];
            if (unit < 0) break;
            bool ok = true;
            Unit U{};
            decode_unit(unit, pairs, B, cu_kept, kv_chunk, &U, M_total, status);
            PT_UNIT(uc, 0, globaltimer());
            PT_UNIT(uc, 4, static_cast<unsigned long long>(U.n_kv) | (static_cast<unsigned long long>(U.split) << 8) |
                               (static_cast<unsigned long long>(U.qt) << 24) |
                               (static_cast<unsigned long long>(U.chunk) << 40) |
                               (static_cast<unsigned long long>(U.pair) << 48));
            const int q_local = U.qt * BM + r;
            const bool valid_row = q_local < U.Mb;
            const int64_t qg = static_cast<int64_t>(U.seq0) + q_local;
            const int hw = 2 * U.pair + h;  // this warpgroup's query head
            if (!waited) {
                pdl_wait();  // pos, rank (the compaction map) and the split scratch from here on
                waited = true;
            }
            float inv_tau = 1.0f;
            if (GATED && valid_row)
                inv_tau = 1.0f / (1.0f + __ldg(c + hw) * logf(static_cast<float>(__ldcg(pos + qg)) /
                                                             static_cast<float>(__ldcg(rank + qg))));
            const float alpha = sm_scale * LOG2E * inv_tau;
            const uint64_t al2 = f32x2_pack(alpha, alpha);
            float m_run = -INFINITY, l_run = 0.f;
            int arrival = 0;  // thread r = 0: the split unit's arrival at its counter (taken a tile early)
            int* cnt = nullptr;
            int64_t slot = 0;
            if (U.split) {
                slot = (static_cast<int64_t>(U.b) * pairs + U.pair) * ws.slots_per_pair + (U.qt - kv_chunk);
                cnt = ws.cnt + slot * 2 + h;
            }
            for (int j = 0; j < U.n_kv; ++j, ++it) {
                const int jt = U.kv0 + j;  // KV tile index within the sequence
                if (U.split && j + 1 == U.n_kv && r == 0) arrival = atomicAdd(cnt, 1);
                if (!mbar_wait_warp(bar(T_S_FULL + h), it & 1, abort_flag, status, TG_WHERE_SOFTMAX)) {
                    ok = false;
                    break;
                }
                PT_STAMP(5, uc == 0 && j == 0 && threadIdx.x == 0);
                if (j == 0) PT_UNIT(uc, 6, globaltimer());
#ifdef TG_TRACE
                if (uc == 0 && j == 0 && threadIdx.x == 0 && blockIdx.x < 1024)
                    g_pers_trace[blockIdx.x * 16 + 13] = U.n_kv | (U.split ? 1000 : 0) | (U.qt << 16);
#endif
                if (r == 0) PT_PIPE(4 + h, it);
                tc_fence_after();
                float x[BN];
#pragma unroll
                for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(tS + cc * 32, x + cc * 32);
                tmem_wait_ld();
                if (r == 0) PT_PIPE(6 + h, it);
                if (jt == U.qt) {
                    const int lim = q_local - jt * BN;  // keys with column > lim lie in the causal future
#pragma unroll
                    for (int cc = 0; cc < BN; ++cc) x[cc] = cc > lim ? -INFINITY : x[cc];
                }
                float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int cc = 0; cc < BN; cc += 2) mp[(cc >> 1) & 3] = max3f(mp[(cc >> 1) & 3], x[cc], x[cc + 1]);
                // floored so that a tile whose keys all carry an infinite negative bias gives
                // p = 0 instead of 2^(-inf + inf)
                const float mx = fmaxf(alpha * fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])), -1.0e30f);
                float corr = 1.0f;
                bool rescale_o = false;
                if (j == 0 || mx > m_run + RESCALE_THRESHOLD) {
                    const float m_new = fmaxf(m_run, mx);
                    corr = ex2_approx(m_run - m_new);
                    m_run = m_new;
                    rescale_o = j > 0;
                }
                const uint64_t nm2 = f32x2_pack(-m_run, -m_run);
                if (r == 0) PT_PIPE(8 + h, it);
                const bool poly_ok = jt != U.qt;  // no masked element in this tile
                uint64_t sp[4] = {0ull, 0ull, 0ull, 0ull};
                // P row r as bf16 pairs over the first 64 columns of S_h (the A operand of the
                // PV product, read from TMEM); every S value is in registers already
#pragma unroll
                for (int c32 = 0; c32 < BN / 32; ++c32) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int cc = c32 * 32 + 4 * e;
                        const uint64_t a0 = f32x2_fma(al2, f32x2_pack(x[cc], x[cc + 1]), nm2);
                        const uint64_t a1 = f32x2_fma(al2, f32x2_pack(x[cc + 2], x[cc + 3]), nm2);
                        uint64_t e0, e1;
                        if (e < PT_POLY_QUADS && poly_ok) {
                            e0 = exp2_poly_x2(a0);
                            e1 = exp2_poly_x2(a1);
                        } else {
                            e0 = f32x2_pack(ex2_approx(f32x2_lo(a0)), ex2_approx(f32x2_hi(a0)));
                            e1 = f32x2_pack(ex2_approx(f32x2_lo(a1)), ex2_approx(f32x2_hi(a1)));
                        }
                        sp[(2 * e) & 3] = f32x2_add(sp[(2 * e) & 3], e0);
                        sp[(2 * e + 1) & 3] = f32x2_add(sp[(2 * e + 1) & 3], e1);
                        pk[2 * e] = pack_bf16x2(f32x2_lo(e0), f32x2_hi(e0));
                        pk[2 * e + 1] = pack_bf16x2(f32x2_lo(e1), f32x2_hi(e1));
                    }
                    tmem_st16u(tS + c32 * 16, pk);
                }
                const uint64_t s01 = f32x2_add(sp[0], sp[1]), s23 = f32x2_add(sp[2], sp[3]);
                const uint64_t s4 = f32x2_add(s01, s23);
                l_run = l_run * corr + (f32x2_lo(s4) + f32x2_hi(s4));
                if (rescale_o) {
                    // O_h is stable: the commit after S_h(j) also covers PV_h(j-1), and PV_h(j)
                    // waits for this P
#pragma unroll
                    for (int ch = 0; ch < HD / 32; ++ch) {
                        float o[32];
                        tmem_ld32(tO + ch * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= corr;
                        tmem_st32(tO + ch * 32, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();  // every lane's P and O stores are complete and fenced
                if (r == 0) PT_PIPE(10 + h, it);
                if (lane == 0) mbar_arrive(bar(T_P_FULL + h));
            }
            // ---------------------------------------------------------------- epilogue
            PT_STAMP(6, uc == 0 && threadIdx.x == 0);
            PT_UNIT(uc, 1, globaltimer());
            if (ok) ok = mbar_wait_warp(bar(T_O_FULL + h), uc & 1, abort_flag, status, TG_WHERE_SOFTMAX);
            PT_STAMP(7, uc == 0 && threadIdx.x == 0);
            PT_UNIT(uc, 2, globaltimer());
            if (bar_red_or(bid, 128, !ok)) break;
            tc_fence_after();
            const float inv_l = 1.0f / l_run;
            uint16_t* orow = out + (qg * Hq + hw) * HD;
            // A thread writes its own row; a warp's stores go to 32 different rows, so wider
            // stores mean fewer of them: 32 bytes (one whole sector) when `out` is 32-byte
            // aligned, else 16.
            auto store_chunk = [&](int ch, const float* o32, float w) {  // 32 columns from 32 ch
                if (!valid_row) return;
                if (wide_out) {
#pragma unroll
                    for (int k8 = 0; k8 < 2; ++k8) {
                        const float* p = o32 + k8 * 16;
                        asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(orow + ch * 32 + k8 * 16),
                                     "r"(pack_bf16x2(p[0] * w, p[1] * w)), "r"(pack_bf16x2(p[2] * w, p[3] * w)),
                                     "r"(pack_bf16x2(p[4] * w, p[5] * w)), "r"(pack_bf16x2(p[6] * w, p[7] * w)),
                                     "r"(pack_bf16x2(p[8] * w, p[9] * w)), "r"(pack_bf16x2(p[10] * w, p[11] * w)),
                                     "r"(pack_bf16x2(p[12] * w, p[13] * w)), "r"(pack_bf16x2(p[14] * w, p[15] * w))
                                     : "memory");
                    }
                } else {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        uint4 v;
                        v.x = pack_bf16x2(o32[k4 * 8 + 0] * w, o32[k4 * 8 + 1] * w);
                        v.y = pack_bf16x2(o32[k4 * 8 + 2] * w, o32[k4 * 8 + 3] * w);
                        v.z = pack_bf16x2(o32[k4 * 8 + 4] * w, o32[k4 * 8 + 5] * w);
                        v.w = pack_bf16x2(o32[k4 * 8 + 6] * w, o32[k4 * 8 + 7] * w);
                        *reinterpret_cast<uint4*>(orow + ch * 32 + k4 * 8) = v;
                    }
                }
            };
            if (!U.split) {
#pragma unroll
                for (int ch = 0; ch < HD / 32; ++ch) {
                    float o[32];
                    tmem_ld32(tO + ch * 32, o);
                    tmem_wait_ld();
                    store_chunk(ch, o, inv_l);
                }
                if (valid_row && lse) lse[qg * Hq + hw] = (m_run + log2f(l_run)) / LOG2E;
            } else {
                // The two KV chunks of a split query tile meet through one counter per head
                // (taken by thread 0 at the start of its last tile): the first to arrive
                // (0 -> 1) writes its normalised partial (bf16 column pairs, [pair][row] so that
                // a warp's 32 rows are one 128-byte write) and log-sum-exp, then publishes them
                // (+1, release); the second (arrival value 1 or 2) waits, if needed, for that
                // publication (the first is resident and depends on nothing else, so the
                // bounded wait ends), merges the partial with its own O read from TMEM, writes
                // the rows and resets the counter.
                const float my_lse = m_run + log2f(l_run);
                if (r == 0) s_arr[h] = arrival;
                named_bar_sync(bid, 128);
                const int arr = s_arr[h];
                named_bar_sync(bid, 128);  // s_arr is read before it is reused
                if (arr == 0) {
                    uint32_t* po = reinterpret_cast<uint32_t*>(ws.o) +
                                   ((slot * ws.max_nch + U.chunk) * 2 + h) * (BM * HD / 2) + r;
#pragma unroll
                    for (int ch = 0; ch < HD / 32; ++ch) {
                        float o[32];
                        tmem_ld32(tO + ch * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            po[(ch * 16 + e) * BM] = pack_bf16x2(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
                    }
                    ws.lse2[((slot * ws.max_nch + U.chunk) * 2 + h) * BM + r] = my_lse;
                    named_bar_sync(bid, 128);  // every partial store is issued
                    if (r == 0) {
                        asm volatile("fence.acq_rel.gpu;" ::: "memory");
                        atomicAdd(cnt, 1);  // publish
                    }
                } else {
                    // The acquire load (thread 0; the others follow through the barrier) makes
                    // the other chunk's partial visible; it returns at once when that chunk had
                    // published before this one arrived (arrival value 2).
                    if (r == 0) {
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
                        s_arr[h] = ready;
                    }
                    named_bar_sync(bid, 128);
                    const int ready = s_arr[h];
                    const int64_t oidx = (slot * ws.max_nch + (U.chunk ^ 1)) * 2 + h;
                    const uint32_t* pt = reinterpret_cast<const uint32_t*>(ws.o) + oidx * (BM * HD / 2) + r;
                    // Order-independent merge: this chunk's row is rounded to bf16 exactly as the
                    // other's partial was, each weight depends only on its own chunk's
                    // log-sum-exp and the (commutative) sum, and the two products are added, so
                    // the result does not depend on which chunk arrived first.
                    const float other_lse = ready ? __ldcg(ws.lse2 + oidx * BM + r) : my_lse;
                    const float mx = fmaxf(my_lse, other_lse);
                    const float e_me = ex2_approx(my_lse - mx), e_ot = ex2_approx(other_lse - mx);
                    const float inv_w = 1.0f / (e_me + e_ot);
                    const float w_me = e_me * inv_w, w_ot = e_ot * inv_w;
                    // The other partial's next 32 columns are loaded while this 32 are merged, so
                    // the loads' round trips to L2 overlap (head_dim 128; at 64 each chunk loads
                    // its own, which keeps that instance free of spills).
                    constexpr bool kAhead = HD > 64;
                    uint32_t pw[16], pn[16];
                    if (kAhead && ready) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pn[e] = __ldcg(pt + e * BM);
                    }
#pragma unroll
                    for (int ch = 0; ch < HD / 32; ++ch) {
                        if (kAhead) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) pw[e] = pn[e];
                            if (ready && ch + 1 < HD / 32) {
#pragma unroll
                                for (int e = 0; e < 16; ++e) pn[e] = __ldcg(pt + ((ch + 1) * 16 + e) * BM);
                            }
                        }
                        float o[32];
                        tmem_ld32(tO + ch * 32, o);
                        tmem_wait_ld();
                        if (ready) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const uint32_t w = kAhead ? pw[e] : __ldcg(pt + (ch * 16 + e) * BM);
                                const uint32_t mine = pack_bf16x2(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
                                o[2 * e] = __fadd_rn(__fmul_rn(w_me, __uint_as_float(mine << 16)),
                                                     __fmul_rn(w_ot, __uint_as_float(w << 16)));
                                o[2 * e + 1] = __fadd_rn(__fmul_rn(w_me, __uint_as_float(mine & 0xFFFF0000u)),
                                                         __fmul_rn(w_ot, __uint_as_float(w & 0xFFFF0000u)));
                            }
                            store_chunk(ch, o, 1.0f);
                        }
                    }
                    if (ready && valid_row && lse) lse[qg * Hq + hw] = (mx + log2f(e_me + e_ot)) / LOG2E;
                    named_bar_sync(bid, 128);  // every read of the partial is done
                    if (r == 0) *cnt = 0;      // ready for the next call
                }
            }
            // the O reads are complete before the next unit's first PV_h overwrites O_h
            // (that product waits for this warpgroup's next P arrival)
            tc_fence_before();
            PT_STAMP(8, uc == 0 && threadIdx.x == 0);
            PT_UNIT(uc, 3, globaltimer());
            PT_UNIT(uc, 5, static_cast<unsigned long long>(U.split ? s_arr[h] + 1 : 0));
            ++uc;
        }
#ifdef TG_TRACE
        if (threadIdx.x == 0 && blockIdx.x < 1024) {
            unsigned smid;
            asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
            g_pers_trace[blockIdx.x * 16 + 9] = globaltimer();
            g_pers_trace[blockIdx.x * 16 + 11] = smid | (static_cast<unsigned long long>(uc) << 32);
            g_pers_trace[blockIdx.x * 16 + 12] = it;  // tiles this CTA processed
        }
#endif
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    PT_STAMP(10, threadIdx.x == 0);
    if (threadIdx.x == 0) {
        // the last CTA to finish resets the unit counter for the next launch
        __threadfence();
        if (atomicAdd(sched + 1, 1) == static_cast<int>(gridDim.x) - 1) {
            sched[0] = 0;
            sched[1] = 0;
            __threadfence();
        }
    }
}

__global__ void exp2_poly_selftest_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
    for (int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x); i < n;
         i += 2 * static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
        const uint64_t r = exp2_poly_x2(f32x2_pack(a, b));
        y[i] = f32x2_lo(r);
        if (i + 1 < n) y[i + 1] = f32x2_hi(r);
    }
}

}  // namespace

cudaError_t launch_exp2_poly_selftest(const float* x, float* y, int64_t n, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const int64_t blocks = (n + 511) / 512;
    exp2_poly_selftest_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 256, 0, st>>>(x, y, n);
    return cudaGetLastError();
}

#ifdef TG_TRACE
extern "C" __attribute__((visibility("default"))) int tg_trace_read_attention_pers(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, g_pers_trace, sizeof(g_pers_trace)) == cudaSuccess ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int tg_trace_read_attention_pers_units(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, g_pers_units, sizeof(g_pers_units)) == cudaSuccess ? 0 : 1;
}
extern "C" __attribute__((visibility("default"))) int tg_trace_read_attention_pers_pipe(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, g_pers_pipe, sizeof(g_pers_pipe)) == cudaSuccess ? 0 : 1;
}
#endif

// Registers per thread the persistent kernel was built with, or 0 if it cannot run (its
// register hand-over needs exactly the launch budget).
template <int HD, bool GATED>
static int pers_launch_regs() {
    cudaFuncAttributes a{};
    if (cudaFuncGetAttributes(&a, gated_attn_pers_kernel<HD, GATED>) != cudaSuccess) return 0;
    return a.numRegs;
}

template <int HD, bool GATED>
static cudaError_t launch_pers_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                    const int32_t* cu_kept, int B, int64_t M_total, int max_M, int Hq, int Hkv,
                                    const int32_t* pos,
                                    const int32_t* rank, const GateSet& gates, const float* c, float sm_scale,
                                    uint16_t* out, float* lse, void* ws, size_t ws_bytes, bool early,
                                    cudaStream_t st) {
    using L = PtSmem<HD>;
    static std::atomic<uint64_t> attr_set{0};
    static std::atomic<int> regs{-1};
    if (regs.load() < 0) regs.store(pers_launch_regs<HD, GATED>());
    // the register hand-over (setmaxnreg) is sized for exactly PT_LAUNCH_REGS at launch
    if (regs.load() != PT_LAUNCH_REGS) return cudaErrorNotSupported;
    if (cudaError_t e = ensure_smem_limit(gated_attn_pers_kernel<HD, GATED>, L::ALLOC, attr_set); e != cudaSuccess)
        return e;
    const AttnWsLayout lay = attention_ws_layout(B, max_M, Hq, Hkv, HD, false);
    if (ws == nullptr || ws_bytes < lay.total) return cudaErrorInvalidValue;
    uint8_t* base = static_cast<uint8_t*>(ws);
    SplitWs sw{};
    sw.cnt = reinterpret_cast<int*>(base + lay.cnt_off);
    sw.o = reinterpret_cast<float*>(base + lay.o_off);
    sw.lse2 = reinterpret_cast<float*>(base + lay.lse_off);
    sw.max_nch = lay.max_nch;
    sw.slots_per_pair = lay.slots_per_pair;
    const int n_qt_max = (max_M + BM - 1) / BM;
    const int64_t total = units_below_host(n_qt_max, lay.C) * B * (Hq / 2);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned grid = static_cast<unsigned>(total < sms ? total : sms);
    return launch_pdl(gated_attn_pers_kernel<HD, GATED>, dim3(grid), dim3(PT_THREADS), static_cast<size_t>(L::ALLOC),
                      st, tq, tk, tv, cu_kept, pos, rank, gates, c, sm_scale, Hq, Hkv, B, M_total, lay.C, total, sw,
                      reinterpret_cast<int*>(base), out, lse, device_status_ptr(), early ? 1 : 0,
                      (reinterpret_cast<uintptr_t>(out) & 31u) == 0 ? 1 : 0);
}

cudaError_t launch_attention_persistent(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                        const int32_t* cu_kept, int B, int64_t M_total, int max_M, int Hq,
                                        int Hkv, int d, const int32_t* pos, const int32_t* rank,
                                        const GateSet& gates, const float* c, float sm_scale, uint16_t* out,
                                        float* lse, void* ws, size_t ws_bytes, bool early, cudaStream_t st) {
    const bool gated = gates.n > 0;
    if (d == 64)
        return gated ? launch_pers_impl<64, true>(tq, tk, tv, cu_kept, B, M_total, max_M, Hq, Hkv, pos, rank, gates, c,
                                                  sm_scale, out, lse, ws, ws_bytes, early, st)
                     : launch_pers_impl<64, false>(tq, tk, tv, cu_kept, B, M_total, max_M, Hq, Hkv, pos, rank, gates, c,
                                                   sm_scale, out, lse, ws, ws_bytes, early, st);
    if (d == 128)
        return gated ? launch_pers_impl<128, true>(tq, tk, tv, cu_kept, B, M_total, max_M, Hq, Hkv, pos, rank, gates, c,
                                                   sm_scale, out, lse, ws, ws_bytes, early, st)
                     : launch_pers_impl<128, false>(tq, tk, tv, cu_kept, B, M_total, max_M, Hq, Hkv, pos, rank, gates, c,
                                                    sm_scale, out, lse, ws, ws_bytes, early, st);
    return cudaErrorNotSupported;
}

}  // namespace tg
