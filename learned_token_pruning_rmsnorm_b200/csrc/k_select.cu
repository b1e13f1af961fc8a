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
constexpr int SEL_ITEMS = 8;
constexpr int SEL_SMEM_KEYS = 36864;  // 144 KB of cached keys
constexpr int SEL_HIST_BYTES = SEL_WARPS * 256 * 4;
constexpr int SEL_SMEM_BYTES = SEL_SMEM_KEYS * 4 + SEL_HIST_BYTES;

struct SelShared {
    int warp_sums[SEL_WARPS];
    int bcast[4];
};

// Exclusive scan of one int per thread over the block; returns the prefix and
// writes the block total to *total.  All threads must call it.
__device__ __forceinline__ int block_exclusive_scan(int v, int* total, SelShared& sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) sh.warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = sh.warp_sums[lane];
        int s = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += y;
        }
        sh.warp_sums[lane] = s - w;  // exclusive prefix of warp totals
        if (lane == 31) sh.bcast[0] = s;
    }
    __syncthreads();
    const int res = sh.warp_sums[warp] + x - v;
    *total = sh.bcast[0];
    __syncthreads();
    return res;
}

__device__ __forceinline__ float logsigmoid_f(float s) { return fminf(s, 0.0f) - log1pf(expf(-fabsf(s))); }

__global__ void __launch_bounds__(SEL_THREADS, 1)
select_scan_kernel(int mode, const float* __restrict__ scores, const uint8_t* __restrict__ keep_in,
                   const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ span,
                   const int32_t* __restrict__ kbud, const int32_t* __restrict__ cu_kept,
                   uint8_t* __restrict__ keep_out, int32_t* __restrict__ kept_idx, int32_t* __restrict__ pos,
                   int32_t* __restrict__ rank, float* __restrict__ gls) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint32_t* skeys = reinterpret_cast<uint32_t*>(smem_raw);
    int* hist = reinterpret_cast<int*>(smem_raw + SEL_SMEM_KEYS * 4);  // [SEL_WARPS][256]
    __shared__ SelShared sh;
    __shared__ uint32_t s_prefix, s_mask;
    __shared__ int s_remaining;

    const int b = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t s0 = cu_seqlens[b], s1 = cu_seqlens[b + 1];
    // spans are clamped into the sequence so that a malformed span cannot index outside it
    const int64_t p0 = s0 + min(max(static_cast<int64_t>(span[2 * b]), int64_t(0)), s1 - s0);
    const int64_t p1 = max(p0, s0 + min(static_cast<int64_t>(span[2 * b + 1]), s1 - s0));
    const int64_t P = p1 - p0;
    const bool emit = kept_idx != nullptr;  // cu_kept is only read when emitting
    const int64_t m0 = emit ? cu_kept[b] : 0, m1 = emit ? cu_kept[b + 1] : 0;

    int64_t kk = P;
    uint32_t thr = 0;       // the K-th largest key (when 0 < kk < P)
    int64_t need_eq = 0;    // keys equal to thr that are kept
    if (mode == 0) {
        const int32_t kb = kbud[b];
        kk = (kb < 0 || static_cast<int64_t>(kb) > P) ? P : static_cast<int64_t>(kb);
    }
    const bool do_radix = (mode == 0) && kk > 0 && kk < P;

    if (do_radix) {
        const bool cached = P <= SEL_SMEM_KEYS;
        if (cached) {
            for (int64_t i = tid; i < P; i += SEL_THREADS) skeys[i] = score_key(scores[p0 + i]);
        }
        if (tid == 0) {
            s_prefix = 0u;
            s_mask = 0u;
            s_remaining = static_cast<int>(kk);
        }
        __syncthreads();
        for (int pass = 0; pass < 4; ++pass) {
            const int shift = 24 - 8 * pass;
            for (int i = tid; i < SEL_WARPS * 256; i += SEL_THREADS) hist[i] = 0;
            __syncthreads();
            const uint32_t prefix = s_prefix, mask = s_mask;
            int* my_hist = hist + warp * 256;
            // the loop bound is uniform per warp so that __match_any_sync sees full warps
            for (int64_t base = 0; base < P; base += SEL_THREADS) {
                const int64_t i = base + tid;
                bool valid = i < P;
                uint32_t key = 0;
                if (valid) key = cached ? skeys[i] : score_key(scores[p0 + i]);
                valid = valid && ((key & mask) == prefix);
                const uint32_t digit = valid ? ((key >> shift) & 255u) : 256u;
                const unsigned peers = __match_any_sync(0xffffffffu, digit);
                const int leader = __ffs(peers) - 1;
                if (valid && lane == leader) atomicAdd(&my_hist[digit], __popc(peers));
            }
            __syncthreads();
            // fold the per-warp histograms into warp 0's copy
            for (int bin = tid; bin < 256; bin += SEL_THREADS) {
                int sum = 0;
                for (int w = 0; w < SEL_WARPS; ++w) sum += hist[w * 256 + bin];
                hist[bin] = sum;
            }
            __syncthreads();
            if (warp == 0) {
                // digits in descending order: lane l covers digits 255-8l ... 248-8l
                int cnt[8];
                int lsum = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    cnt[e] = hist[255 - (lane * 8 + e)];
                    lsum += cnt[e];
                }
                int incl = lsum;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    int y = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += y;
                }
                const int excl = incl - lsum;
                const int rem = s_remaining;
                __syncwarp();  // every lane has read s_remaining before one lane rewrites it
                if (excl < rem && incl >= rem) {
                    int cum = excl;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (cum + cnt[e] >= rem) {
                            const uint32_t dgt = 255u - static_cast<uint32_t>(lane * 8 + e);
                            s_prefix = prefix | (dgt << shift);
                            s_mask = mask | (255u << shift);
                            s_remaining = rem - cum;
                            break;
                        }
                        cum += cnt[e];
                    }
                }
            }
            __syncthreads();
        }
        thr = s_prefix;
        need_eq = s_remaining;
    }

    // ---------------------------------------------------------------- ordered scan
    const int64_t n = s1 - s0;
    int64_t eq_carry = 0, kept_carry = 0;
    for (int64_t cbase = 0; cbase < n; cbase += static_cast<int64_t>(SEL_THREADS) * SEL_ITEMS) {
        const int64_t t_first = s0 + cbase + static_cast<int64_t>(tid) * SEL_ITEMS;
        bool kept[SEL_ITEMS];
        bool prun[SEL_ITEMS];
        float sc[SEL_ITEMS];
        int n_eq = 0;
        bool is_eq[SEL_ITEMS];
#pragma unroll
        for (int e = 0; e < SEL_ITEMS; ++e) {
            const int64_t t = t_first + e;
            const bool in = t < s1;
            prun[e] = in && t >= p0 && t < p1;
            sc[e] = prun[e] ? scores[t] : 0.0f;
            is_eq[e] = false;
            if (mode == 1) {
                kept[e] = in && keep_in[t] != 0;
            } else if (!prun[e]) {
                kept[e] = in;
            } else if (kk >= P) {
                kept[e] = true;
            } else if (kk == 0) {
                kept[e] = false;
            } else {
                const uint32_t key = score_key(sc[e]);
                kept[e] = key > thr;
                is_eq[e] = key == thr;
                n_eq += is_eq[e] ? 1 : 0;
            }
        }
        if (do_radix) {
            int eq_total = 0;
            int64_t eq_rank = eq_carry + block_exclusive_scan(n_eq, &eq_total, sh);
#pragma unroll
            for (int e = 0; e < SEL_ITEMS; ++e) {
                if (is_eq[e]) {
                    kept[e] = eq_rank < need_eq;
                    ++eq_rank;
                }
            }
            eq_carry += eq_total;
        }
        int n_kept = 0;
#pragma unroll
        for (int e = 0; e < SEL_ITEMS; ++e) n_kept += kept[e] ? 1 : 0;
        int kept_total = 0;
        int64_t m = m0 + kept_carry + block_exclusive_scan(n_kept, &kept_total, sh);
        kept_carry += kept_total;
#pragma unroll
        for (int e = 0; e < SEL_ITEMS; ++e) {
            const int64_t t = t_first + e;
            if (t >= s1) break;
            if (mode == 0) keep_out[t] = kept[e] ? 1 : 0;
            if (kept[e]) {
                // a caller-given keep vector that disagrees with cu_kept must
                // not write outside [m0, m1)
                if (emit && m < m1) {
                    kept_idx[m] = static_cast<int32_t>(t);
                    pos[m] = static_cast<int32_t>(t - s0 + 1);
                    rank[m] = static_cast<int32_t>(m - m0 + 1);
                    gls[m] = prun[e] ? logsigmoid_f(sc[e]) : 0.0f;
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
