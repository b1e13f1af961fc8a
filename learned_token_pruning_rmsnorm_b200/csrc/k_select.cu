// Stages 2 and 3 of the gated prefill: deterministic top-K selection over each
// sequence's prunable span, the stable compaction scan, and the row gather.
//
// Selection keeps the K best prunable tokens and every non-prunable token
// (TokenGate AI summary, "Key Contributions" 1; README copy, "How it works").
// Order: higher score first, then lower token index.
//
// Design: one cluster of SEL_CL CTAs per sequence.  CTA i owns a contiguous
// slice of the sequence's tokens and caches the order-preserving uint32 keys
// of its prunable tokens in shared memory.
//   1. bucket select: each pass histograms the keys of the current range into
//      <= 2048 buckets of width 2^s (the first pass the whole key range by its
//      top 11 bits, the next ones the chosen bucket by the following 11 and 10
//      bits) and sums them into 64 superbins.
//      One warp per CTA then reads the 8 x 64 superbin sums and the 8 x 32
//      buckets of the chosen superbin through distributed shared memory and
//      narrows the range to the bucket holding the K-th key.  The passes stop
//      when that bucket is a single key value thr (need_eq = how many keys
//      equal to thr are kept: the lowest-indexed ones), at most three, or as
//      soon as every key of the bucket is taken (usually after two): then the
//      rule is key >= the bucket's lower edge, with no tie to rank.
//   2. ordered scan: every warp owns a contiguous run of the slice and walks
//      it 32 tokens at a time; ballots count the kept tokens, one block scan
//      over the warp totals and one exchange of slice totals across the
//      cluster number them, and each kept token writes its compaction-map
//      entry (kept_idx, pos, rank, logsigmoid of its score) in coalesced
//      stores with no further barrier.
// Everything is deterministic: atomics only build counts.

#include <cooperative_groups.h>

#include "tg_internal.cuh"

namespace cg = cooperative_groups;

namespace tg {
namespace {

// Optional device trace (builds with -DTG_TRACE only): clock64 stamps of the
// phases of the first CTA of the first sequence.
#ifdef TG_TRACE
__device__ unsigned long long g_sel_trace[32];
#define SEL_TRACE(point)                                                                         \
    do {                                                                                         \
        if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)                              \
            g_sel_trace[(point)] = static_cast<unsigned long long>(clock64());                   \
    } while (0)
#else
#define SEL_TRACE(point) \
    do {                 \
    } while (0)
#endif

constexpr int SEL_CL = 8;                     // CTAs per sequence (one cluster)
constexpr int SEL_THREADS = 1024;
constexpr int SEL_WARPS = SEL_THREADS / 32;
constexpr int SEL_CACHE_KEYS = 32768;         // keys cached per CTA (128 KB)
constexpr int SEL_BINS = 2048;
constexpr int SEL_SUPER = SEL_BINS / 32;      // superbins of 32 buckets
constexpr int SEL_SMEM_BYTES = SEL_CACHE_KEYS * 4 + 2 * SEL_BINS * 4;

struct SelShared {
    int coarse[2][SEL_SUPER];  // per pass parity: bucket counts summed over each superbin
    int xchg[2];               // slice totals published to the cluster: kept, tie-ranked
    int wsum[SEL_WARPS];       // a first-pass histogram summed over each warp's 64 buckets
    int warp_kept[SEL_WARPS];  // exclusive prefix over the warps of this CTA
    int warp_eq[SEL_WARPS];
    uint32_t lo;               // current key range [lo, lo + width)
    uint64_t width;
    int remaining;             // keys still to take from the current range, counted from its top
    int bin_count;
};

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
    for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

__device__ __forceinline__ int warp_inclusive_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += y;
    }
    return v;
}

__device__ __forceinline__ float logsigmoid_f(float s) { return fminf(s, 0.0f) - log1pf(expf(-fabsf(s))); }

// inverse of score_key (every NaN comes back as a NaN, -0 as +0)
__device__ __forceinline__ float key_to_score(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

__device__ __forceinline__ int bit_length(uint64_t v) { return v ? 64 - __clzll(static_cast<long long>(v)) : 0; }

// split cluster barrier: arrive once this CTA reads no more remote shared
// memory, wait before leaving so that no CTA exits while another reads it
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__global__ void __cluster_dims__(SEL_CL, 1, 1) __launch_bounds__(SEL_THREADS, 1)
select_scan_kernel(int mode, const float* __restrict__ scores, const uint8_t* __restrict__ keep_in,
                   const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ span,
                   const int32_t* __restrict__ kbud, const int32_t* __restrict__ cu_kept,
                   uint8_t* __restrict__ keep_out, int32_t* __restrict__ kept_idx, int32_t* __restrict__ pos,
                   int32_t* __restrict__ rank, float* __restrict__ gls, int* __restrict__ key_hist) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint32_t* skeys = reinterpret_cast<uint32_t*>(smem_raw);
    int* hist_buf = reinterpret_cast<int*>(smem_raw + SEL_CACHE_KEYS * 4);  // [2][SEL_BINS]
    __shared__ SelShared sh;
    cg::cluster_group cl = cg::this_cluster();

    const int crank = static_cast<int>(cl.block_rank());
    SEL_TRACE(0);
    pdl_wait();  // global memory is read only from here on
    pdl_trigger();
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t s0 = cu_seqlens[b], s1 = cu_seqlens[b + 1];
    // spans are clamped into the sequence so that a malformed span cannot index outside it
    const int64_t p0 = s0 + min(max(static_cast<int64_t>(span[2 * b]), int64_t(0)), s1 - s0);
    const int64_t p1 = max(p0, s0 + min(static_cast<int64_t>(span[2 * b + 1]), s1 - s0));
    const int64_t P = p1 - p0;
    const bool emit = kept_idx != nullptr;  // cu_kept is only read when emitting
    const int64_t m0 = emit ? cu_kept[b] : 0, m1 = emit ? cu_kept[b + 1] : 0;

    // this CTA's token slice [t0, t1) (a multiple of 1024 tokens long), split
    // into one contiguous run per warp
    const int64_t n = s1 - s0;
    const int64_t per = ((n + SEL_CL - 1) / SEL_CL + SEL_THREADS - 1) / SEL_THREADS * SEL_THREADS;
    const int64_t t0 = min(s1, s0 + per * crank), t1 = min(s1, t0 + per);
    const int64_t per_warp = per / SEL_WARPS;
    const int64_t w0 = min(t1, t0 + per_warp * warp), w1 = min(t1, w0 + per_warp);
    // prunable part of the slice [k0, k1) and whether its keys fit the cache
    const int64_t k0 = max(t0, p0), k1 = max(k0, min(t1, p1));
    const bool cached = (k1 - k0) <= SEL_CACHE_KEYS;

    int64_t kk = P;
    if (mode == 0) {
        const int32_t kb = kbud[b];
        kk = (kb < 0 || static_cast<int64_t>(kb) > P) ? P : static_cast<int64_t>(kb);
    }
    const bool do_select = (mode == 0) && kk > 0 && kk < P;

    uint32_t thr = 0;        // the K-th largest key
    int64_t need_eq = 0;     // keys equal to thr that are kept
    bool all_eq_kept = true; // every key equal to thr is kept: no tie ranking needed

    // ------------------------------------------------ cache keys (for the selection and for gls)
    const bool need_gls = emit && kk > 0;  // some prunable token is kept: its logsigmoid is emitted
    if (cached && (do_select || need_gls)) {
#pragma unroll 8
        for (int64_t t = k0 + tid; t < k1; t += SEL_THREADS) skeys[t - k0] = score_key(__ldcg(scores + t));
    }
    SEL_TRACE(1);

    if (do_select) {  // uniform over the cluster: it depends on the sequence only
        // The first pass buckets the whole key range by the top 11 bits (sign, exponent and two
        // mantissa bits of the score), each later pass the chosen bucket by the next 11 and then
        // 10 bits, so three passes resolve any key and no agreement on the keys' range is
        // needed before the first.
        if (tid == 0) {
            sh.lo = 0u;
            sh.width = static_cast<uint64_t>(1) << 32;
            sh.remaining = static_cast<int>(kk);
            sh.bin_count = 0;
        }
        if (key_hist != nullptr) {
            // The score kernel took the first pass (the top 11 bits of every key of this
            // sequence): every CTA reads the same counts and finds the same bucket itself, the
            // K-th key from the top (its 64-bucket warp segment, then the bucket), with no
            // cluster round trip.
            const int* kh = key_hist + static_cast<int64_t>(b) * SEL_BINS;
            int* hist0 = hist_buf;  // free until the passes below
            const int v0 = __ldcg(kh + 2 * tid), v1 = __ldcg(kh + 2 * tid + 1);
            hist0[2 * tid] = v0;
            hist0[2 * tid + 1] = v1;
            const int wsum = warp_sum(v0 + v1);
            if (lane == 0) sh.wsum[warp] = wsum;
            __syncthreads();
            if (warp == 0) {
                const int rem = static_cast<int>(kk);
                const int v = sh.wsum[SEL_WARPS - 1 - lane];
                const int incl = warp_inclusive_scan(v);
                const unsigned hit = __ballot_sync(0xffffffffu, incl - v < rem && incl >= rem);
                if (hit != 0u) {  // else (counts inconsistent with the span) the full passes run
                    const int L = __ffs(hit) - 1;
                    const int rem1 = rem - __shfl_sync(0xffffffffu, incl - v, L);
                    const int base = 64 * (SEL_WARPS - 1 - L);
                    const int hi = hist0[base + 63 - 2 * lane], lo2 = hist0[base + 62 - 2 * lane];
                    const int incl2 = warp_inclusive_scan(hi + lo2);
                    const int excl2 = incl2 - hi - lo2;
                    if (excl2 < rem1 && incl2 >= rem1) {
                        const bool upper = excl2 + hi >= rem1;
                        const int bin = upper ? base + 63 - 2 * lane : base + 62 - 2 * lane;
                        sh.lo = static_cast<uint32_t>(bin) << 21;
                        sh.width = static_cast<uint64_t>(1) << 21;
                        sh.remaining = upper ? rem1 - excl2 : rem1 - excl2 - hi;
                        sh.bin_count = upper ? hi : lo2;
                    }
                }
            }
        }
        __syncthreads();  // the key cache and the range are in place
        SEL_TRACE(2);
        // ------------------------------------------------ bucket passes
        // (none when the score kernel's first pass already ends the search: every key of the
        // chosen bucket is taken)
        for (int pass = 0; !(key_hist != nullptr && sh.remaining == sh.bin_count && sh.width < (1ull << 32));
             ++pass) {
            const uint32_t lo = sh.lo;
            const uint64_t width = sh.width;
            const int sh_bits = max(0, bit_length(width - 1) - 11);  // bucket width 2^sh_bits, <= 2048 buckets
            // both buffers alternate by pass: another CTA may still read the previous pass's
            int* hist = hist_buf + (pass & 1) * SEL_BINS;
            int* coarse = sh.coarse[pass & 1];
            hist[tid] = 0;
            hist[tid + SEL_THREADS] = 0;
            __syncthreads();
#pragma unroll 4
            for (int64_t t = k0 + tid; t < k1; t += SEL_THREADS) {
                const uint32_t key = cached ? skeys[t - k0] : score_key(__ldcg(scores + t));
                const uint32_t d = key - lo;  // wraps for keys below lo: excluded by the range test
                if (key >= lo && static_cast<uint64_t>(d) < width) atomicAdd(&hist[d >> sh_bits], 1);
            }
            __syncthreads();
            {   // superbin sums: warp w sums buckets [64w, 64w + 64)
                const int a = warp_sum(hist[64 * warp + lane]);
                const int c = warp_sum(hist[64 * warp + 32 + lane]);
                if (lane == 0) {
                    coarse[2 * warp] = a;
                    coarse[2 * warp + 1] = c;
                }
            }
            cl.sync();  // every CTA's histogram and superbin sums of this pass are complete
            if (warp == 0) {
                // the rem-th key from the top: first its superbin (lane l owns superbins
                // 63 - 2l and 62 - 2l of all CTAs), then its bucket (lane l owns bucket
                // 32 S + 31 - l of all CTAs); every CTA finds the same bucket
                const int rem = sh.remaining;
                int hi = 0, lo2 = 0;
                {
                    int vh[SEL_CL], vl[SEL_CL];
#pragma unroll
                    for (int r = 0; r < SEL_CL; ++r) {
                        const int* cr = cl.map_shared_rank(coarse, r);
                        vh[r] = cr[SEL_SUPER - 1 - 2 * lane];
                        vl[r] = cr[SEL_SUPER - 2 - 2 * lane];
                    }
#pragma unroll
                    for (int r = 0; r < SEL_CL; ++r) {
                        hi += vh[r];
                        lo2 += vl[r];
                    }
                }
                const int incl = warp_inclusive_scan(hi + lo2);
                const int excl = incl - hi - lo2;
                const unsigned hit = __ballot_sync(0xffffffffu, excl < rem && incl >= rem);
                if (hit != 0u) {
                    const int L = __ffs(hit) - 1;
                    const int excl_L = __shfl_sync(0xffffffffu, excl, L);
                    const int hi_L = __shfl_sync(0xffffffffu, hi, L);
                    const bool upper = excl_L + hi_L >= rem;
                    const int S = upper ? SEL_SUPER - 1 - 2 * L : SEL_SUPER - 2 - 2 * L;
                    const int rem2 = upper ? rem - excl_L : rem - excl_L - hi_L;
                    const int bin = 32 * S + 31 - lane;
                    int v[SEL_CL];
#pragma unroll
                    for (int r = 0; r < SEL_CL; ++r) v[r] = cl.map_shared_rank(hist, r)[bin];
                    int cnt = 0;
#pragma unroll
                    for (int r = 0; r < SEL_CL; ++r) cnt += v[r];
                    const int incl2 = warp_inclusive_scan(cnt);
                    const int excl2 = incl2 - cnt;
                    if (excl2 < rem2 && incl2 >= rem2) {
                        const uint64_t new_lo = static_cast<uint64_t>(lo) + (static_cast<uint64_t>(bin) << sh_bits);
                        const uint64_t end = static_cast<uint64_t>(lo) + width;
                        sh.lo = static_cast<uint32_t>(new_lo);
                        sh.width = min(static_cast<uint64_t>(1) << sh_bits, end - new_lo);
                        sh.remaining = rem2 - excl2;
                        sh.bin_count = cnt;
                    }
                } else if (lane == 0) {
                    // unreachable while the range holds >= rem keys; end the search on lo
                    sh.width = 1;
                    sh.remaining = 0;
                    sh.bin_count = 0;
                }
            }
            __syncthreads();
            SEL_TRACE(3 + pass);
            // done when the bucket is a single key value, or when every key of the bucket is
            // taken: then "key >= its lower edge" is the whole rule (thr = lo, all kept below)
            if (sh_bits == 0 || pass >= 3 || sh.remaining == sh.bin_count) break;
        }
        thr = sh.lo;
        need_eq = sh.remaining;
        all_eq_kept = need_eq == sh.bin_count;
    }

    // ---------------------------------------------------------------- ordered scan
    // kept flag of token t; eq marks a key equal to thr that is ranked by index
    // when only some of them are kept
    auto flags = [&](int64_t t, bool& kept, bool& eq) {
        kept = false;
        eq = false;
        if (t >= w1) return;
        const bool prun = t >= p0 && t < p1;
        if (mode == 1) {
            kept = __ldcg(keep_in + t) != 0;
        } else if (!prun) {
            kept = true;
        } else if (!do_select) {
            kept = kk > 0;  // kk >= P keeps all, kk == 0 keeps none
        } else {
            const uint32_t key = cached ? skeys[t - k0] : score_key(__ldcg(scores + t));
            kept = key > thr || (key == thr && all_eq_kept);
            eq = key == thr && !all_eq_kept;
        }
    };
    const unsigned lt_mask = (1u << lane) - 1u;

    // warp totals: kept tokens and (for the tie ranking) keys equal to thr
    int my_kept = 0, my_eq = 0;
#pragma unroll 4
    for (int64_t base = w0; base < w1; base += 32) {
        bool kept, eq;
        flags(base + lane, kept, eq);
        my_kept += __popc(__ballot_sync(0xffffffffu, kept));
        my_eq += __popc(__ballot_sync(0xffffffffu, eq));
    }
    if (lane == 0) {
        sh.warp_kept[warp] = my_kept;
        sh.warp_eq[warp] = my_eq;
    }
    __syncthreads();
    if (warp == 0) {
        const int vk = sh.warp_kept[lane], ve = sh.warp_eq[lane];
        const int ik = warp_inclusive_scan(vk), ie = warp_inclusive_scan(ve);
        sh.warp_kept[lane] = ik - vk;
        sh.warp_eq[lane] = ie - ve;
        if (lane == 31) {
            sh.xchg[0] = ik;
            sh.xchg[1] = ie;
        }
    }
    SEL_TRACE(8);
    cl.sync();  // slice totals published; also orders the key cache before the emission
    SEL_TRACE(9);
    // every CTA read the score kernel's counts before the barrier above: zero them for the next
    // call, each CTA its eighth
    if (key_hist != nullptr && tid < SEL_BINS / SEL_CL)
        key_hist[static_cast<int64_t>(b) * SEL_BINS + crank * (SEL_BINS / SEL_CL) + tid] = 0;
    int64_t kept_before = sh.warp_kept[warp], eq_before = sh.warp_eq[warp];
    {
        int vk[SEL_CL], ve[SEL_CL];
#pragma unroll
        for (int r = 0; r < SEL_CL; ++r) {
            const SelShared* o = cl.map_shared_rank(&sh, r);
            vk[r] = o->xchg[0];
            ve[r] = o->xchg[1];
        }
#pragma unroll
        for (int r = 0; r < SEL_CL; ++r) {
            if (r < crank) {
                kept_before += vk[r];
                eq_before += ve[r];
            }
        }
    }
    SEL_TRACE(6);
    cluster_arrive_release();  // no remote reads after this point
    SEL_TRACE(7);
    // kept_before counts the tie-ranked keys as not kept; min(eq_before, need_eq) of
    // those before this warp's run are kept
    int64_t m = m0 + kept_before + (all_eq_kept ? 0 : min(eq_before, need_eq));
    int64_t eq_seen = eq_before;
    for (int64_t base = w0; base < w1; base += 32) {
        const int64_t t = base + lane;
        bool kept, eq;
        flags(t, kept, eq);
        const unsigned eq_ball = __ballot_sync(0xffffffffu, eq);
        if (eq && eq_seen + __popc(eq_ball & lt_mask) < need_eq) kept = true;
        eq_seen += __popc(eq_ball);
        const unsigned kept_ball = __ballot_sync(0xffffffffu, kept);
        if (t < w1) {
            if (mode == 0) keep_out[t] = kept ? 1 : 0;
            const int64_t mi = m + __popc(kept_ball & lt_mask);
            // a caller-given keep vector that disagrees with cu_kept must not
            // write outside [m0, m1)
            if (emit && kept && mi < m1) {
                const bool prun = t >= p0 && t < p1;
                float g = 0.0f;
                if (prun) g = logsigmoid_f(cached ? key_to_score(skeys[t - k0]) : __ldcg(scores + t));
                kept_idx[mi] = static_cast<int32_t>(t);
                pos[mi] = static_cast<int32_t>(t - s0 + 1);
                rank[mi] = static_cast<int32_t>(mi - m0 + 1);
                gls[mi] = g;
            }
        }
        m += __popc(kept_ball);
    }
    SEL_TRACE(10);
    cluster_wait_acquire();
    SEL_TRACE(11);
}

// Row gather hidden_kept[m, :] = hidden[kept_idx[m], :], one warp per row,
// 16-byte accesses, every load of a row issued before its stores.
template <int VPL>  // 16-byte vectors per lane per row
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint4* __restrict__ hidden, const int32_t* __restrict__ kept_idx, int64_t M, int64_t T,
                   int vecs_per_row, uint4* __restrict__ out, int wait_at_end) {
    const int lane = threadIdx.x & 31;
    // wait_at_end: the map and rows were complete before the preceding kernel was released,
    // so only the kernel's completion waits for it (which keeps "this kernel is done" meaning
    // "everything before it is done" for the work that follows)
    if (!wait_at_end) pdl_wait();  // global memory is read only from here on
    pdl_trigger();
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t m = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); m < M;
         m += warps_total) {
        const int64_t src = __ldcg(kept_idx + m);
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
    if (wait_at_end) pdl_wait();
}

// Gather of narrow rows (one 4- or 8-byte word each, e.g. a position or a gate's
// logsigmoid per kept row): dst[m] = src[kept_idx[m]], one thread per row.
template <typename W>
__global__ void __launch_bounds__(256)
gather_words_kernel(const W* __restrict__ src, const int32_t* __restrict__ kept_idx, int64_t M, int64_t T,
                    W* __restrict__ out, int wait_at_end) {
    if (!wait_at_end) pdl_wait();  // as in gather_rows_kernel
    pdl_trigger();
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t m = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; m < M; m += stride) {
        const int64_t i = __ldcg(kept_idx + m);
        if (i >= 0 && i < T) out[m] = __ldcg(src + i);
    }
    if (wait_at_end) pdl_wait();
}

// Row scatter out[idx[m], :] = in[m, :] (the inverse of the gather), one warp per
// row; indices outside [0, T) write nothing.
template <int VPL>
__global__ void __launch_bounds__(256)
scatter_rows_kernel(const uint4* __restrict__ in, const int32_t* __restrict__ idx, int64_t M, int64_t T,
                    int vecs_per_row, uint4* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    pdl_wait();  // global memory is read only from here on
    pdl_trigger();
    const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t m = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); m < M;
         m += warps_total) {
        const int64_t dst = __ldcg(idx + m);
        if (dst < 0 || dst >= T) continue;
        const uint4* s = in + m * vecs_per_row;
        uint4* d = out + dst * vecs_per_row;
        for (int c0 = 0; c0 < vecs_per_row; c0 += 32 * VPL) {
            uint4 r[VPL];
#pragma unroll
            for (int e = 0; e < VPL; ++e) {
                const int c = c0 + e * 32 + lane;
                if (c < vecs_per_row) r[e] = __ldcg(s + c);
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

#ifdef TG_TRACE
extern "C" __attribute__((visibility("default"))) int tg_trace_read_select(unsigned long long* host) {
    return cudaMemcpyFromSymbol(host, g_sel_trace, sizeof(g_sel_trace)) == cudaSuccess ? 0 : 1;
}
#endif

cudaError_t launch_select_scan(int mode, const float* scores, const uint8_t* keep_in, const int32_t* cu_seqlens,
                               const int32_t* span, const int32_t* k, const int32_t* cu_kept, int B, int64_t T,
                               uint8_t* keep_out, int32_t* kept_idx, int32_t* pos, int32_t* rank, float* gls,
                               cudaStream_t st, int* key_hist) {
    static std::atomic<uint64_t> attr_set{0};
    if (cudaError_t e = ensure_smem_limit(select_scan_kernel, SEL_SMEM_BYTES, attr_set); e != cudaSuccess)
        return e;
    if (B == 0) return cudaSuccess;
    return launch_pdl(select_scan_kernel, dim3(SEL_CL, B), dim3(SEL_THREADS), static_cast<size_t>(SEL_SMEM_BYTES), st,
                      mode, scores, keep_in, cu_seqlens, span, k, cu_kept, keep_out, kept_idx, pos, rank, gls,
                      key_hist);
}

cudaError_t launch_gather_bytes(const void* src, const int32_t* kept_idx, int64_t M_total, int64_t T,
                                int64_t row_bytes, void* dst, cudaStream_t st, bool wait_at_end) {
    const int wae = wait_at_end ? 1 : 0;
    if (M_total == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (row_bytes == 4 || row_bytes == 8) {
        const int64_t need = (M_total + 255) / 256;
        const int grid = static_cast<int>(need < static_cast<int64_t>(sms) * 8 ? need : sms * 8);
        if (row_bytes == 4)
            return launch_pdl(gather_words_kernel<uint32_t>, dim3(grid), dim3(256), 0, st,
                              static_cast<const uint32_t*>(src), kept_idx, M_total, T, static_cast<uint32_t*>(dst),
                              wae);
        return launch_pdl(gather_words_kernel<unsigned long long>, dim3(grid), dim3(256), 0, st,
                          static_cast<const unsigned long long*>(src), kept_idx, M_total, T,
                          static_cast<unsigned long long*>(dst), wae);
    }
    const int64_t vpr64 = row_bytes / 16;
    if (vpr64 <= 0 || vpr64 * 16 != row_bytes || vpr64 > (int64_t(1) << 30)) return cudaErrorInvalidValue;
    const int vpr = static_cast<int>(vpr64);
    const int64_t blocks_needed = (M_total + 7) / 8;
    const int grid = static_cast<int>(blocks_needed < static_cast<int64_t>(sms) * 8 ? blocks_needed : sms * 8);
    const uint4* h = static_cast<const uint4*>(src);
    uint4* o = static_cast<uint4*>(dst);
    // one round trip per row where it fits: all of a 4 KB or 2 KB row's loads in flight before its stores
    if (vpr >= 256)
        return launch_pdl(gather_rows_kernel<8>, dim3(grid), dim3(256), 0, st, h, kept_idx, M_total, T, vpr, o, wae);
    if (vpr >= 128)
        return launch_pdl(gather_rows_kernel<4>, dim3(grid), dim3(256), 0, st, h, kept_idx, M_total, T, vpr, o, wae);
    return launch_pdl(gather_rows_kernel<2>, dim3(grid), dim3(256), 0, st, h, kept_idx, M_total, T, vpr, o, wae);
}

cudaError_t launch_scatter_bytes(const void* src, const int32_t* idx, int64_t M, int64_t T, int64_t row_bytes,
                                 void* dst, cudaStream_t st) {
    if (M == 0) return cudaSuccess;
    const int64_t vpr64 = row_bytes / 16;
    if (vpr64 <= 0 || vpr64 * 16 != row_bytes || vpr64 > (int64_t(1) << 30)) return cudaErrorInvalidValue;
    const int vpr = static_cast<int>(vpr64);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t blocks_needed = (M + 7) / 8;
    const int grid = static_cast<int>(blocks_needed < static_cast<int64_t>(sms) * 8 ? blocks_needed : sms * 8);
    const uint4* h = static_cast<const uint4*>(src);
    uint4* o = static_cast<uint4*>(dst);
    if (vpr >= 256) return launch_pdl(scatter_rows_kernel<8>, dim3(grid), dim3(256), 0, st, h, idx, M, T, vpr, o);
    return launch_pdl(scatter_rows_kernel<2>, dim3(grid), dim3(256), 0, st, h, idx, M, T, vpr, o);
}

cudaError_t launch_gather_rows(const uint16_t* hidden, const int32_t* kept_idx, int64_t M_total, int64_t T, int D,
                               uint16_t* hidden_kept, cudaStream_t st, bool wait_at_end) {
    return launch_gather_bytes(hidden, kept_idx, M_total, T, static_cast<int64_t>(D) * 2, hidden_kept, st,
                               wait_at_end);
}

}  // namespace tg
