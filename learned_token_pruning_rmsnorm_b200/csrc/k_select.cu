// Stages 2 and 3 of the gated prefill: deterministic top-K selection over each
// sequence's prunable span, the stable compaction scan, and the row gather.
//
// Selection keeps the K best prunable tokens and every non-prunable token
// (TokenGate AI summary, "Key Contributions" 1; README copy, "How it works").
// Order: higher score first, then lower token index.
//
// Design (one CTA of 1024 threads per sequence; the span holds at most a few
// hundred thousand scores, which sit in L2 right after the scoring kernel):
//   1. radix select on order-preserving uint32 keys, 8-bit digits, MSB first,
//      four passes; per-warp shared-memory histograms fed by warp-aggregated
//      atomics (__match_any_sync), so that the few hot exponent bins of the
//      first pass do not serialise.  Keys are cached in shared memory when the
//      span fits (<= SEL_SMEM_KEYS keys), else re-read from global memory.
//      Result: the K-th key u*, and need_eq = how many keys equal to u* are
//      kept (the lowest-indexed ones).
//   2. one ordered pass over the sequence in chunks of 1024 x SEL_ITEMS
//      tokens: a block scan ranks the keys equal to u*, a second block scan
//      numbers the kept tokens, and each kept token writes its compaction
//      outputs (kept_idx, pos, rank, logsigmoid of its score).
// Everything is deterministic: atomics only build counts.

#include "tg_internal.cuh"

namespace tg {
namespace {

constexpr int SEL_THREADS = 1024;
constexpr int SEL_WARPS = SEL_THREADS / 32;
constexpr int SEL_ITEMS = 16;                 // consecutive tokens per thread in the ordered scan
constexpr int SEL_CACHE_KEYS = 40960;         // spans up to this length keep their keys in shared memory
constexpr int SEL_HIST_BINS = 2048;
constexpr int SEL_SMEM_BYTES = SEL_CACHE_KEYS * 4 + SEL_HIST_BINS * 4;

struct SelShared {
    int warp_sums[SEL_WARPS];
    int total;
    uint32_t prefix, mask;
    int remaining, bin_count;
};

// Inclusive scan of one int per thread over the block; returns the
// inclusive prefix and writes the block total to *total.  All threads call it.
__device__ __forceinline__ int block_inclusive_scan(int v, int* total, SelShared& sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) sh.warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int w = sh.warp_sums[lane];
        int s = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += y;
        }
        sh.warp_sums[lane] = s - w;  // exclusive prefix of the warp totals
        if (lane == 31) sh.total = s;
    }
    __syncthreads();
    const int res = sh.warp_sums[warp] + x;
    *total = sh.total;
    __syncthreads();
    return res;
}

__device__ __forceinline__ float logsigmoid_f(float s) { return fminf(s, 0.0f) - log1pf(expf(-fabsf(s))); }

// inverse of score_key (every NaN comes back as a NaN, -0 as +0)
__device__ __forceinline__ float key_to_score(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

__global__ void __launch_bounds__(SEL_THREADS, 1)
select_scan_kernel(int mode, const float* __restrict__ scores, const uint8_t* __restrict__ keep_in,
                   const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ span,
                   const int32_t* __restrict__ kbud, const int32_t* __restrict__ cu_kept,
                   uint8_t* __restrict__ keep_out, int32_t* __restrict__ kept_idx, int32_t* __restrict__ pos,
                   int32_t* __restrict__ rank, float* __restrict__ gls) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint32_t* skeys = reinterpret_cast<uint32_t*>(smem_raw);
    int* hist = reinterpret_cast<int*>(smem_raw + SEL_CACHE_KEYS * 4);
    __shared__ SelShared sh;

    const int b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31;
    const int64_t s0 = cu_seqlens[b], s1 = cu_seqlens[b + 1];
    // spans are clamped into the sequence so that a malformed span cannot index outside it
    const int64_t p0 = s0 + min(max(static_cast<int64_t>(span[2 * b]), int64_t(0)), s1 - s0);
    const int64_t p1 = max(p0, s0 + min(static_cast<int64_t>(span[2 * b + 1]), s1 - s0));
    const int64_t P = p1 - p0;
    const bool emit = kept_idx != nullptr;  // cu_kept is only read when emitting
    const int64_t m0 = emit ? cu_kept[b] : 0, m1 = emit ? cu_kept[b + 1] : 0;

    int64_t kk = P;
    if (mode == 0) {
        const int32_t kb = kbud[b];
        kk = (kb < 0 || static_cast<int64_t>(kb) > P) ? P : static_cast<int64_t>(kb);
    }
    const bool do_radix = (mode == 0) && kk > 0 && kk < P;
    const bool cached = do_radix && P <= SEL_CACHE_KEYS;

    uint32_t thr = 0;        // the K-th largest key
    int64_t need_eq = 0;     // keys equal to thr that are kept (the lowest-indexed ones)
    bool all_eq_kept = true; // every key equal to thr is kept: no tie ranking needed

    if (do_radix) {
        if (cached) {
            for (int64_t i = tid; i < P; i += SEL_THREADS) skeys[i] = score_key(__ldg(scores + p0 + i));
        }
        if (tid == 0) {
            sh.prefix = 0u;
            sh.mask = 0u;
            sh.remaining = static_cast<int>(kk);
        }
        // radix select, most significant digits first: 11 + 11 + 10 bits
        const int shifts[3] = {21, 10, 0};
        const int widths[3] = {11, 11, 10};
        const int64_t P_pad = (P + SEL_THREADS - 1) / SEL_THREADS * SEL_THREADS;
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = shifts[pass];
            const int nbins = 1 << widths[pass];
            const uint32_t dmask = static_cast<uint32_t>(nbins - 1);
            for (int i = tid; i < nbins; i += SEL_THREADS) hist[i] = 0;
            __syncthreads();
            const uint32_t prefix = sh.prefix, mask = sh.mask;
            for (int64_t i = tid; i < P_pad; i += SEL_THREADS) {
                bool valid = i < P;
                uint32_t key = 0;
                if (valid) key = cached ? skeys[i] : score_key(__ldg(scores + p0 + i));
                valid = valid && ((key & mask) == prefix);
                const unsigned act = __ballot_sync(0xffffffffu, valid);
                if (valid) {
                    const uint32_t digit = (key >> shift) & dmask;
                    const unsigned peers = __match_any_sync(act, digit);
                    if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], __popc(peers));
                }
            }
            __syncthreads();
            // locate the digit holding the remaining-th largest key: thread t owns the
            // bins of digits nbins-1-t*bpt ... in descending order
            const int bpt = nbins / SEL_THREADS;  // 2 or 1
            int cnt[2] = {0, 0};
            int local = 0;
            for (int e = 0; e < bpt; ++e) {
                cnt[e] = hist[nbins - 1 - (tid * bpt + e)];
                local += cnt[e];
            }
            int total = 0;
            const int incl = block_inclusive_scan(local, &total, sh);
            const int excl = incl - local;
            const int rem = sh.remaining;
            __syncthreads();  // every thread has read sh.remaining before it is rewritten
            if (excl < rem && incl >= rem) {
                int cum = excl;
                for (int e = 0; e < bpt; ++e) {
                    if (cum + cnt[e] >= rem) {
                        const uint32_t dgt = static_cast<uint32_t>(nbins - 1 - (tid * bpt + e));
                        sh.prefix = prefix | (dgt << shift);
                        sh.mask = mask | (dmask << shift);
                        sh.remaining = rem - cum;
                        sh.bin_count = cnt[e];
                        break;
                    }
                    cum += cnt[e];
                }
            }
            __syncthreads();
        }
        thr = sh.prefix;
        need_eq = sh.remaining;
        all_eq_kept = need_eq == sh.bin_count;  // the last bin holds exactly the keys equal to thr
    }

    // ---------------------------------------------------------------- ordered scan
    const int64_t n = s1 - s0;
    int64_t eq_carry = 0, kept_carry = 0;
    for (int64_t cbase = 0; cbase < n; cbase += static_cast<int64_t>(SEL_THREADS) * SEL_ITEMS) {
        const int64_t t_first = s0 + cbase + static_cast<int64_t>(tid) * SEL_ITEMS;
        uint32_t kept_bits = 0, eq_bits = 0;
        int n_eq = 0;
#pragma unroll
        for (int e = 0; e < SEL_ITEMS; ++e) {
            const int64_t t = t_first + e;
            const bool in = t < s1;
            const bool prun = in && t >= p0 && t < p1;
            bool kept;
            if (mode == 1) {
                kept = in && keep_in[t] != 0;
            } else if (!prun) {
                kept = in;
            } else if (!do_radix) {
                kept = kk > 0;  // kk >= P keeps all, kk == 0 keeps none
            } else {
                const uint32_t key = cached ? skeys[t - p0] : score_key(__ldg(scores + t));
                const bool eq = key == thr;
                kept = key > thr || (eq && all_eq_kept);
                if (eq && !all_eq_kept) {
                    eq_bits |= 1u << e;
                    ++n_eq;
                }
            }
            kept_bits |= kept ? (1u << e) : 0u;
        }
        if (!all_eq_kept) {
            // rank the keys equal to thr in index order; the first need_eq are kept
            int eq_total = 0;
            int64_t eq_rank = eq_carry + block_inclusive_scan(n_eq, &eq_total, sh) - n_eq;
#pragma unroll
            for (int e = 0; e < SEL_ITEMS; ++e) {
                if (eq_bits & (1u << e)) {
                    if (eq_rank < need_eq) kept_bits |= 1u << e;
                    ++eq_rank;
                }
            }
            eq_carry += eq_total;
        }
        const int n_kept = __popc(kept_bits);
        int kept_total = 0;
        int64_t m = m0 + kept_carry + block_inclusive_scan(n_kept, &kept_total, sh) - n_kept;
        kept_carry += kept_total;
        if (mode == 0) {
#pragma unroll
            for (int e = 0; e < SEL_ITEMS; ++e) {
                const int64_t t = t_first + e;
                if (t < s1) keep_out[t] = (kept_bits >> e) & 1u;
            }
        }
        if (emit && kept_bits) {
#pragma unroll
            for (int e = 0; e < SEL_ITEMS; ++e) {
                if (!((kept_bits >> e) & 1u)) continue;
                const int64_t t = t_first + e;
                // a caller-given keep vector that disagrees with cu_kept must
                // not write outside [m0, m1)
                if (m < m1) {
                    const bool prun = t >= p0 && t < p1;
                    float g = 0.0f;
                    if (prun) g = logsigmoid_f(cached ? key_to_score(skeys[t - p0]) : __ldg(scores + t));
                    kept_idx[m] = static_cast<int32_t>(t);
                    pos[m] = static_cast<int32_t>(t - s0 + 1);
                    rank[m] = static_cast<int32_t>(m - m0 + 1);
                    gls[m] = g;
                }
                ++m;
            }
        }
    }
}

// Row gather hidden_kept[m, :] = hidden[kept_idx[m], :], one warp per row,
// 16-byte accesses, every load of a row issued before its stores.
template <int VPL>  // 16-byte vectors per lane per row
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint4* __restrict__ hidden, const int32_t* __restrict__ kept_idx, int64_t M, int64_t T,
                   int vecs_per_row, uint4* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t m = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); m < M;
         m += warps_total) {
        const int64_t src = kept_idx[m];
        if (src < 0 || src >= T) continue;  // an unwritten map entry (inconsistent keep flags) copies nothing
        const uint4* s = hidden + src * vecs_per_row;
        uint4* d = out + m * vecs_per_row;
        for (int c0 = 0; c0 < vecs_per_row; c0 += 32 * VPL) {
            uint4 r[VPL];
#pragma unroll
            for (int e = 0; e < VPL; ++e) {
                const int c = c0 + e * 32 + lane;
                if (c < vecs_per_row) r[e] = __ldg(s + c);
            }
#pragma unroll
            for (int e = 0; e < VPL; ++e) {
                const int c = c0 + e * 32 + lane;
                if (c < vecs_per_row) d[c] = r[e];
            }
        }
    }
}

}  // namespace

cudaError_t launch_select_scan(int mode, const float* scores, const uint8_t* keep_in, const int32_t* cu_seqlens,
                               const int32_t* span, const int32_t* k, const int32_t* cu_kept, int B,
                               uint8_t* keep_out, int32_t* kept_idx, int32_t* pos, int32_t* rank, float* gls,
                               cudaStream_t st) {
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(select_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             SEL_SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    if (B == 0) return cudaSuccess;
    select_scan_kernel<<<B, SEL_THREADS, SEL_SMEM_BYTES, st>>>(mode, scores, keep_in, cu_seqlens, span, k, cu_kept,
                                                               keep_out, kept_idx, pos, rank, gls);
    return cudaGetLastError();
}

cudaError_t launch_gather_rows(const uint16_t* hidden, const int32_t* kept_idx, int64_t M_total, int64_t T, int D,
                               uint16_t* hidden_kept, cudaStream_t st) {
    if (M_total == 0) return cudaSuccess;
    const int vpr = D / 8;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks_needed = (M_total + 7) / 8;
    const int grid = static_cast<int>(blocks_needed < static_cast<int64_t>(sms) * 8 ? blocks_needed : sms * 8);
    const uint4* h = reinterpret_cast<const uint4*>(hidden);
    uint4* o = reinterpret_cast<uint4*>(hidden_kept);
    if (vpr >= 256)
        gather_rows_kernel<8><<<grid, 256, 0, st>>>(h, kept_idx, M_total, T, vpr, o);
    else
        gather_rows_kernel<2><<<grid, 256, 0, st>>>(h, kept_idx, M_total, T, vpr, o);
    return cudaGetLastError();
}

}  // namespace tg
