// Stage 1 of the gated prefill: the gate's weight preparation and the gate
// score of every prunable token (TokenGate AI summary, "Key Contributions" 1:
// an MLP over each token's RMSNorm-normalised post-attention residual).
//
//   r_t = 1 / sqrt(mean_i x_ti^2 + eps)
//   s_t = b2 + sum_j w2[j] * SiLU(r_t * (Wg[j,:] . x_t) + b1[j])
// with Wg = bf16(gamma (.) W1^T) prepared once by tg_gate_prepare.
//
// Scoring is one pass over the prunable rows of `hidden` on the tensor cores:
//   - persistent CTAs, each owning tiles of NACC x 128 rows; the NACC
//     accumulators (128 x I fp32 each, in TMEM) share every Wg tile, so the
//     gate weight is streamed from L2 once per 128*NACC rows;
//   - warp 0 streams 64-channel slices of the rows and of Wg with TMA
//     (128-byte swizzle) through a STAGES-deep ring; warp 1 issues
//     tcgen05.mma (M=128, N=I, K=16) per accumulator;
//   - 4*NACC warps read each row's slice from the same shared-memory tiles to
//     accumulate sum(x^2) while the MMAs run, then apply rsqrt, b1, SiLU and
//     the w2 dot product to the accumulator rows read from TMEM.
// HBM traffic is the hidden rows of the span (read once) plus one fp32 score
// per row; the normalised activations are never rounded before the product.

#include "tg_sm100.cuh"

namespace tg {
namespace {

using namespace sm100;

__global__ void gate_prepare_kernel(const uint16_t* __restrict__ gamma, const uint16_t* __restrict__ W1, int D, int I,
                                    uint16_t* __restrict__ Wg) {
    const int64_t n = static_cast<int64_t>(I) * D;
    for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int j = static_cast<int>(e / D), i = static_cast<int>(e - static_cast<int64_t>(j) * D);
        const float p = bf16_bits_to_float(gamma[i]) * bf16_bits_to_float(W1[static_cast<int64_t>(i) * I + j]);
        const __nv_bfloat16 r = __float2bfloat16_rn(p);
        Wg[e] = *reinterpret_cast<const uint16_t*>(&r);
    }
}

// Optional device trace (builds with -DTG_TRACE only): clock64 stamps of the
// first CTA's pipeline per k-block (producer issue, MMA start, MMA issued,
// sum of squares done) and globaltimer start/end stamps of every CTA.
#ifdef TG_TRACE
__device__ unsigned long long g_score_trace[4 * 128];
__device__ unsigned long long g_score_cta[512 * 2];
#define SC_TRACE(point, k)                                                                  \
    do {                                                                                    \
        if (blockIdx.x == 0 && (k) < 128)                                                   \
            g_score_trace[(point) * 128 + (k)] = static_cast<unsigned long long>(clock64()); \
    } while (0)
#define SC_CTA(slot)                                                                          \
    do {                                                                                      \
        if (blockIdx.x < 512) g_score_cta[blockIdx.x * 2 + (slot)] = globaltimer();            \
    } while (0)
#else
#define SC_TRACE(point, k) \
    do {                   \
    } while (0)
#define SC_CTA(slot) \
    do {             \
    } while (0)
#endif

constexpr int KB = 64;                // channels per pipeline stage (one 128-byte swizzle row)
constexpr int TILE_A = 128 * KB * 2;  // one 128-row slice: 16 KB

// Two epilogue warps per (accumulator, TMEM lane group): each sums the squares of half of a
// row's channels in every slice and runs the gate MLP's epilogue over half of its columns;
// the pair adds its halves through shared memory in a fixed order.
template <int NACC>
struct ScoreCfg {
    static constexpr int STAGES = NACC == 2 ? 3 : 4;
    static constexpr int EPI_COMBOS = 4 * NACC;  // (accumulator, lane group)
    static constexpr int EPI_WARPS = 2 * EPI_COMBOS;
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;
    static constexpr uint32_t TMEM_COLS = NACC == 2 ? 512 : 256;
    static constexpr int ROWS = 128 * NACC;
};

// bar.red.or over the epilogue warps (named barrier 1): every one learns whether any gave up
__device__ __forceinline__ bool epi_red_or(int nthreads, bool pred) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"(static_cast<uint32_t>(pred)), "r"(nthreads)
        : "memory");
    return res != 0;
}

template <int NACC>
__host__ __device__ constexpr int score_stage_bytes(int I) { return NACC * TILE_A + I * 128; }

// stages x (NACC row slices + one Wg slice of I rows), b1, w2, 16 barriers, tmem slot + abort
// flag, the epilogue pairs' exchange ([2][NACC * 128] sums of squares, the same for the dots)
template <int NACC>
__host__ __device__ constexpr int score_smem_bytes(int I) {
    return ScoreCfg<NACC>::STAGES * score_stage_bytes<NACC>(I) + 2 * 256 * 4 + 16 * 8 + 16 +
           4 * NACC * 128 * 4 + 1024;
}

// SiLU(z) = z / (1 + e^-z).  e^-z takes one special-function-unit operation; the
// reciprocal runs on the FMA pipe instead of a second one (the epilogue, 2 x 65536 of
// them per 256-row tile, was bound by that unit): a seed from the float's bits
// (r0 = bits(0x7EF31000 - bits(d)), a constant fitted for this kernel, within 5.1% of 1/d)
// and three Newton steps r <- r (2 - d r), relative error below 1e-7.  d is capped so that
// e^-z = inf still gives a finite seed (z / 1e30 ~ -0, as the exact quotient).
__device__ __forceinline__ float silu_f(float z) {
    const float d = fminf(1.0f + ex2_approx(-1.4426950408889634f * z), 1.0e30f);
    float r = __uint_as_float(0x7EF31000u - __float_as_uint(d));
    r = fmaf(r, fmaf(-d, r, 1.0f), r);
    r = fmaf(r, fmaf(-d, r, 1.0f), r);
    r = fmaf(r, fmaf(-d, r, 1.0f), r);
    return z * r;
}

// Tile t of the concatenated per-sequence tile lists -> (first row, end of span, sequence).
__device__ __forceinline__ bool map_tile(int64_t t, int rows, const int32_t* cu_seqlens, const int32_t* span, int B,
                                         int64_t* row0, int64_t* row_end, int* seq = nullptr) {
    for (int b = 0; b < B; ++b) {
        const int64_t s0 = cu_seqlens[b], n = cu_seqlens[b + 1] - s0;
        const int64_t p0 = s0 + min(max(static_cast<int64_t>(span[2 * b]), int64_t(0)), n);
        const int64_t p1 = max(p0, s0 + min(static_cast<int64_t>(span[2 * b + 1]), n));
        const int64_t nt = (p1 - p0 + rows - 1) / rows;
        if (t < nt) {
            *row0 = p0 + t * rows;
            *row_end = p1;
            if (seq) *seq = b;
            return true;
        }
        t -= nt;
    }
    return false;
}

template <int NACC>
__global__ void __launch_bounds__(ScoreCfg<NACC>::THREADS, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ span, int B, int D, int I,
                const float* __restrict__ b1, const float* __restrict__ w2, float b2, float eps,
                float* __restrict__ scores, int64_t T, int* __restrict__ status, int* __restrict__ key_hist) {
    using C = ScoreCfg<NACC>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int stage_bytes = score_stage_bytes<NACC>(I);
    float* s_b1 = reinterpret_cast<float*>(smem + STAGES * stage_bytes);
    float* s_w2 = s_b1 + 256;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + STAGES * stage_bytes + 2 * 256 * 4;
    // barriers: full[STAGES], empty[STAGES], acc_full, acc_empty, drain
    auto full = [&](int s) { return bar0 + 8u * s; };
    auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
    const uint32_t acc_full = bar0 + 8u * (2 * STAGES), acc_empty = bar0 + 8u * (2 * STAGES + 1);
    const uint32_t drain = bar0 + 8u * (2 * STAGES + 2);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + STAGES * stage_bytes + 2 * 256 * 4 + 16 * 8);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* xss = reinterpret_cast<float*>(smem + STAGES * stage_bytes + 2 * 256 * 4 + 16 * 8 + 16);  // [2][NACC*128]
    float* xac = xss + 2 * NACC * 128;                                                                 // [2][NACC*128]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = D / KB;
    if (threadIdx.x == 0) SC_CTA(0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full(s), 1);
            mbar_init(empty(s), 1 + C::EPI_WARPS);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, C::EPI_WARPS);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // global memory is read only from here on (see pdl_wait)
    pdl_wait();
    pdl_trigger();
    for (int j = threadIdx.x; j < I; j += blockDim.x) {
        s_b1[j] = b1[j];
        s_w2[j] = w2[j];
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmX);
            prefetch_tmap(&tmW);
            int64_t it = 0;
            int issued[STAGES] = {};
            bool ok = true;
            for (int64_t t = blockIdx.x; ok; t += gridDim.x) {
                int64_t row0, row_end;
                if (!map_tile(t, C::ROWS, cu_seqlens, span, B, &row0, &row_end)) break;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = static_cast<int>(it % STAGES);
                    const int use = static_cast<int>(it / STAGES);
                    if (use > 0 && !mbar_wait(empty(s), (use - 1) & 1, abort_flag, status, TG_WHERE_PRODUCER)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = sbase + s * stage_bytes;
                    SC_TRACE(0, it);
                    mbar_expect_tx(full(s), stage_bytes);
#pragma unroll
                    for (int a = 0; a < NACC; ++a)
                        tma_load_2d(st + a * TILE_A, &tmX, kb * KB, static_cast<int32_t>(row0 + a * 128), full(s));
                    tma_load_2d(st + NACC * TILE_A, &tmW, kb * KB, 0, full(s));
                    ++issued[s];
                }
            }
            if (*abort_flag) {
                // let every copy this thread started land before the CTA exits
                volatile int never = 0;
                for (int s = 0; s < STAGES; ++s)
                    if (issued[s]) mbar_wait(full(s), (issued[s] - 1) & 1, &never, status, TG_WHERE_DRAIN);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, I, false);
            int64_t it = 0;
            int tcount = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; ok; t += gridDim.x, ++tcount) {
                int64_t row0, row_end;
                if (!map_tile(t, C::ROWS, cu_seqlens, span, B, &row0, &row_end)) break;
                if (tcount > 0 && !mbar_wait(acc_empty, (tcount - 1) & 1, abort_flag, status, TG_WHERE_MMA)) break;
                tc_fence_after();
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = static_cast<int>(it % STAGES);
                    const int use = static_cast<int>(it / STAGES);
                    if (!mbar_wait(full(s), use & 1, abort_flag, status, TG_WHERE_MMA)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    SC_TRACE(1, it);
                    // one descriptor per operand of the stage; a k-step adds its byte offset / 16
                    // to the start-address field (no carry: offsets stay inside shared memory)
                    const uint32_t st = sbase + s * stage_bytes;
                    const uint64_t bdesc0 = smem_desc_sw128(st + NACC * TILE_A, 16, 1024);
                    const uint64_t adesc0 = smem_desc_sw128(st, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < KB / 16; ++kk) {
#pragma unroll
                        for (int a = 0; a < NACC; ++a)
                            mma_bf16_ss(tmem + a * 256, adesc0 + ((a * TILE_A + kk * 32) >> 4), bdesc0 + ((kk * 32) >> 4),
                                        idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(empty(s));
                    SC_TRACE(2, it);
                }
                if (ok) mma_commit(acc_full);
            }
            // every MMA, and the barrier arrivals its commits trigger, lands before the CTA exits
            mma_commit(drain);
            volatile int never = 0;
            mbar_wait(drain, 0, &never, status, TG_WHERE_DRAIN);
        }
    } else {
        // ---------------------------------------------------------------- sum of squares + epilogue
        const int e = warp - 2;                 // 0 .. EPI_WARPS-1
        const int hs = e / C::EPI_COMBOS;       // which half of the channels and columns
        const int a = (e % C::EPI_COMBOS) >> 2; // accumulator of this warp
        const int lg = warp & 3;                // TMEM lane group this warp may access
        const int r = lg * 32 + lane;           // row within the 128-row slice == TMEM lane
        const uint32_t lane_addr = static_cast<uint32_t>(lg * 32) << 16;
        const int xi = a * 128 + r;             // this row's slot in the pair exchange
        constexpr int EPI_T = 32 * C::EPI_WARPS;
        // columns of this warp: the first or second half of the 32-column chunks (the 16-column
        // tail, when I is 16 mod 32, goes with the second half)
        const int I32 = I & ~31;
        const int nfull = I32 / 32;
        const int c_begin = hs ? (nfull / 2) * 32 : 0, c_end = hs ? I32 : (nfull / 2) * 32;
        const bool tail = hs == 1 && I32 < I;
        int64_t it = 0;
        int tcount = 0;
        bool ok = true;
        for (int64_t t = blockIdx.x; ok; t += gridDim.x, ++tcount) {
            int64_t row0, row_end;
            int seq = 0;
            if (!map_tile(t, C::ROWS, cu_seqlens, span, B, &row0, &row_end, &seq)) break;
            float ss = 0.f;
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int s = static_cast<int>(it % STAGES);
                const int use = static_cast<int>(it / STAGES);
                if (!mbar_wait_warp(full(s), use & 1, abort_flag, status, TG_WHERE_SOFTMAX)) {
                    ok = false;
                    break;
                }
                // half of the row's 64 channels of this slice (logical 16-byte chunks 4 hs ..
                // 4 hs + 3).  Lane r reads physical chunk (c ^ (r & 7)): the 128-byte swizzle then
                // spreads a warp's 32 rows over all banks; chunk order is irrelevant for a sum of
                // squares.
                const uint8_t* rowp = smem + s * stage_bytes + a * TILE_A + r * 128;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const uint4 v = *reinterpret_cast<const uint4*>(rowp + (((4 * hs + ch) ^ (r & 7)) << 4));
                    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float lo = __uint_as_float(wv[q] << 16), hi = __uint_as_float(wv[q] & 0xFFFF0000u);
                        ss = fmaf(lo, lo, ss);
                        ss = fmaf(hi, hi, ss);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty(s));
                if (warp == 2 && lane == 0) SC_TRACE(3, it);
            }
            xss[hs * (NACC * 128) + xi] = ss;
            const bool okw = ok && mbar_wait_warp(acc_full, tcount & 1, abort_flag, status, TG_WHERE_SOFTMAX);
            // every epilogue warp leaves together (the pairs meet at the barriers below)
            if (epi_red_or(EPI_T, !okw)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const float sst = xss[xi] + xss[NACC * 128 + xi];  // the same order in both warps of the pair
            const float rr = rsqrtf(sst / static_cast<float>(D) + eps);
            float acc_s = 0.f;
            for (int c0 = c_begin; c0 < c_end; c0 += 32) {
                float z[32];
                tmem_ld32(tmem + a * 256 + lane_addr + c0, z);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 32; ++q) acc_s = fmaf(s_w2[c0 + q], silu_f(fmaf(rr, z[q], s_b1[c0 + q])), acc_s);
            }
            if (tail) {  // the last 16 columns when I is 16 mod 32
                float z[32];
                tmem_ld32(tmem + a * 256 + lane_addr + I32, z);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 16; ++q) acc_s = fmaf(s_w2[I32 + q], silu_f(fmaf(rr, z[q], s_b1[I32 + q])), acc_s);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty);
            xac[hs * (NACC * 128) + xi] = acc_s;
            asm volatile("bar.sync 1, %0;" ::"r"(EPI_T) : "memory");  // both halves of every row are in
            if (hs == 0) {
                const float score = xac[xi] + xac[NACC * 128 + xi] + b2;
                const int64_t row = row0 + a * 128 + r;
                const bool valid = row < row_end && TG_DEBUG_CHECK(row >= 0 && row < T, status, TG_WHERE_SCORE);
                if (valid) scores[row] = score;
                if (key_hist != nullptr) {
                    // the selection's first pass: this sequence's scores counted by the top 11 bits
                    // of their order-preserving key, one atomic per distinct bucket of the warp
                    const int bin = valid ? seq * 2048 + static_cast<int>(score_key(score) >> 21) : -1;
                    const unsigned same = __match_any_sync(0xffffffffu, bin);
                    if (valid && lane == __ffs(same) - 1) atomicAdd(key_hist + bin, __popc(same));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) SC_CTA(1);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int NACC>
cudaError_t launch_score_tc(const uint16_t* hidden, const int32_t* cu_seqlens, const int32_t* span, int B, int64_t T,
                            int D, const uint16_t* Wg, const float* b1, const float* w2, float b2, int I, float eps,
                            float* scores, int* key_hist, int sms, cudaStream_t st) {
    using C = ScoreCfg<NACC>;
    static std::atomic<uint64_t> attr_set{0};
    if (cudaError_t e = ensure_smem_limit(score_tc_kernel<NACC>, score_smem_bytes<NACC>(256), attr_set); e != cudaSuccess)
        return e;
    CUtensorMap tx, tw;
    if (!encode_tmap_2d_bf16(&tx, hidden, static_cast<uint64_t>(D), static_cast<uint64_t>(T),
                             static_cast<uint64_t>(D) * 2, KB, 128) ||
        !encode_tmap_2d_bf16(&tw, Wg, static_cast<uint64_t>(D), static_cast<uint64_t>(I), static_cast<uint64_t>(D) * 2,
                             KB, static_cast<uint32_t>(I)))
        return cudaErrorInvalidValue;
    const int64_t tiles_bound = (T + C::ROWS - 1) / C::ROWS + B;
    const int grid = static_cast<int>(tiles_bound < sms ? tiles_bound : sms);
    const cudaError_t le = launch_pdl(score_tc_kernel<NACC>, dim3(grid), dim3(C::THREADS),
                                      static_cast<size_t>(score_smem_bytes<NACC>(I)), st, tx, tw, cu_seqlens, span, B,
                                      D, I, b1, w2, b2, eps, scores, T, device_status_ptr(), key_hist);
    if (le != cudaSuccess) return le;
    return cudaGetLastError();
}

}  // namespace

#ifdef TG_TRACE
extern "C" __attribute__((visibility("default"))) int tg_trace_read_score(unsigned long long* pipe, unsigned long long* ctas) {
    if (cudaMemcpyFromSymbol(pipe, g_score_trace, sizeof(g_score_trace)) != cudaSuccess) return 1;
    return cudaMemcpyFromSymbol(ctas, g_score_cta, sizeof(g_score_cta)) == cudaSuccess ? 0 : 1;
}
#endif

cudaError_t launch_gate_prepare(const uint16_t* gamma, const uint16_t* W1, int D, int I, uint16_t* Wg,
                                cudaStream_t st) {
    const int64_t n = static_cast<int64_t>(I) * D;
    const int grid = static_cast<int>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    gate_prepare_kernel<<<grid, 256, 0, st>>>(gamma, W1, D, I, Wg);
    return cudaGetLastError();
}

cudaError_t launch_score(const uint16_t* hidden, const int32_t* cu_seqlens, const int32_t* span, int B,
                         int64_t T, int D, const uint16_t* Wg, const float* b1, const float* w2, float b2, int I,
                         float eps, float* scores, cudaStream_t st, int* key_hist) {
    if (T == 0 || B == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // 256-row tiles halve the gate-weight traffic from L2 once there are more
    // 128-row tiles than SMs; below that, 128-row tiles spread the rows wider.
    if ((T + 127) / 128 > sms)
        return launch_score_tc<2>(hidden, cu_seqlens, span, B, T, D, Wg, b1, w2, b2, I, eps, scores, key_hist, sms,
                                  st);
    return launch_score_tc<1>(hidden, cu_seqlens, span, B, T, D, Wg, b1, w2, b2, I, eps, scores, key_hist, sms, st);
}

}  // namespace tg
