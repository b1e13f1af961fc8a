// Stages 2 and 3 of the gated prefill: deterministic top-K selection over each
// sequence's prunable span, the stable compaction scan, and the row gather.
//
// Selection keeps the K best prunable tokens and every non-prunable token
// (TokenGate AI summary, "Key Contributions" 1; README copy, "How it works").
// Order: higher score first, then lower token index.
//
// Design: one cluster of SEL_CL CTAs per sequence.  CTA i owns a contiguous
// slice of the sequence's tokens and caches the order-preserving uint32 keys
// of its prunable tokens in shared memory, by their offset in the slice.
//   1. bucket select: each pass histograms the keys of the current range into
//      <= 2048 buckets of width 2^s (the first pass the whole key range by its
//      top 11 bits, the next ones the chosen bucket by the following 11 and 10
//      bits) and sums them into 64 superbins; it also counts the keys above
//      the range.  One warp per CTA then reads the 8 x 64 superbin sums, the
//      counts above and the 8 x 32 buckets of the chosen superbin through
//      distributed shared memory and narrows the range to the bucket holding
//      the K-th key.  The passes stop when that bucket is a single key value
//      thr (need_eq = how many keys equal to thr are kept: the lowest-indexed
//      ones), at most three, or as soon as every key of the bucket is taken
//      (usually after two): then the rule is key >= the bucket's lower edge,
//      with no tie to rank.  The same counts give every slice's number of
//      kept tokens, so the CTAs need no further exchange.
//   2. ordered scan: every warp owns a contiguous run of the slice and walks
//      it 128 tokens at a time, 4 consecutive tokens per lane (one 16-byte
//      load of cached keys); ballots of each of the 4 token positions number
//      the kept tokens after one block scan over the warp totals.  The kept
//      tokens of up to 4096 consecutive entries are listed in shared memory,
//      and the threads then write those compaction-map entries (kept_idx,
//      pos, rank, logsigmoid of the score) densely.  When the counts did not
//      come from the last pass (caller-given keep flags, a search the score
//      kernel's first pass already ended) the slice totals are exchanged once
//      through distributed shared memory.
// Everything is deterministic: atomics only build counts.

#include <cooperative_groups.h>

#include "tg_internal.cuh"

namespace cg = cooperative_groups;

namespace tg {
namespace {

// Optional device trace (builds with -DTG_TRACE only): globaltimer stamps (ns) of the
// phases of every CTA of the first sequence, 16 points per CTA.
#ifdef TG_TRACE
__device__ unsigned long long g_sel_trace[8 * 16];
#define SEL_TRACE(point)                                                                         \
    do {                                                                                         \
        if (blockIdx.y == 0 && blockIdx.x < 8 && threadIdx.x == 0) {                             \
            unsigned long long t_;                                                               \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                               \
            g_sel_trace[blockIdx.x * 16 + (point)] = t_;                                         \
        }                                                                                        \
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
constexpr int SEL_LIST = 4096;                // compaction-map entries emitted per round
constexpr int SEL_SMEM_BYTES = SEL_CACHE_KEYS * 4 + 2 * SEL_BINS * 4 + SEL_LIST * 4;

struct SelShared {
    int coarse[2][SEL_SUPER];  // per pass parity: bucket counts summed over each superbin
    int above[2];              // per pass parity: this CTA's keys above the pass's range
    int xchg[2];               // slice totals published to the cluster: kept, tie-ranked
    int wsum[SEL_WARPS];       // a first-pass histogram summed over each warp's 64 buckets
    int warp_kept[SEL_WARPS];  // exclusive prefix over the warps of this CTA
    int warp_eq[SEL_WARPS];
    int cta_kept;              // kept tokens of the slices before this one (tie-ranked keys excluded)
    int cta_eq;                // tie-ranked keys of the slices before this one
    int counts_known;          // cta_kept / cta_eq came from the last pass (no exchange needed)
    uint32_t lo;               // current key range [lo, lo + width)
    uint64_t width;
    int remaining;             // keys still to take from the current range, counted from its top
    int bin_count;
};

__device__ __forceinline__ int warp_sum(int v) { return __reduce_add_sync(0xffffffffu, v); }

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

// split cluster barrier: arrive once this CTA reads no more remote shared memory, wait
// before leaving so that no CTA exits while another reads it.  The arrive is relaxed: every
// value read remotely has been consumed before it, and no CTA reads what this one writes
// after it, so it needs no memory fence.
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// Token slice [a0, a1) of cluster rank r: SEL_CL slices of `per` tokens (a multiple of
// SEL_THREADS), the last ones shorter or empty.  Token indices fit in 32 bits (cu_seqlens is
// int32); the products are formed in 64 bits so that no intermediate overflows.
__device__ __forceinline__ void slice_of(int r, int s0, int s1, int per, int& a0, int& a1) {
    const int64_t x0 = min(static_cast<int64_t>(s1), static_cast<int64_t>(s0) + static_cast<int64_t>(per) * r);
    a0 = static_cast<int>(x0);
    a1 = static_cast<int>(min(static_cast<int64_t>(s1), x0 + per));
}

__global__ void __cluster_dims__(SEL_CL, 1, 1) __launch_bounds__(SEL_THREADS, 1)
select_scan_kernel(int mode, int early, const float* __restrict__ scores, const uint8_t* __restrict__ keep_in,
                   const int32_t* __restrict__ cu_seqlens, const int32_t* __restrict__ span,
                   const int32_t* __restrict__ kbud, const int32_t* __restrict__ cu_kept,
                   uint8_t* __restrict__ keep_out, int32_t* __restrict__ kept_idx, int32_t* __restrict__ pos,
                   int32_t* __restrict__ rank, float* __restrict__ gls, int* __restrict__ key_hist) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint32_t* skeys = reinterpret_cast<uint32_t*>(smem_raw);
    int* hist_buf = reinterpret_cast<int*>(smem_raw + SEL_CACHE_KEYS * 4);  // [2][SEL_BINS]
    int* list = hist_buf + 2 * SEL_BINS;  // [SEL_LIST]
    __shared__ SelShared sh;
    cg::cluster_group cl = cg::this_cluster();

    const int crank = static_cast<int>(cl.block_rank());
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool emit = kept_idx != nullptr;  // cu_kept is only read when emitting
    // The sequence's bounds, span, budget and output range.  Inside the prefill layer they are
    // the caller's, complete before the call (`early`), and are read before the wait for the
    // score kernel; otherwise after it.
    int s0 = 0, s1 = 0, sp0 = 0, sp1 = 0, kb = -1, m0 = 0, m1 = 0;
    auto load_meta = [&]() {
        s0 = cu_seqlens[b];
        s1 = cu_seqlens[b + 1];
        sp0 = span[2 * b];
        sp1 = span[2 * b + 1];
        if (mode == 0) kb = kbud[b];
        if (emit) {
            m0 = cu_kept[b];
            m1 = cu_kept[b + 1];
        }
    };
    if (early) load_meta();
    SEL_TRACE(0);
    pdl_wait();  // the scores (and the first-pass counts) are read only from here on
    SEL_TRACE(12);
    pdl_trigger();
    if (!early) load_meta();
    // spans are clamped into the sequence so that a malformed span cannot index outside it
    const int n = s1 - s0;
    const int p0 = s0 + min(max(sp0, 0), n);
    const int p1 = max(p0, s0 + min(sp1, n));
    const int P = p1 - p0;

    // this CTA's token slice [t0, t1), split into one contiguous run per warp
    const int per = static_cast<int>(((static_cast<int64_t>(n) + SEL_CL - 1) / SEL_CL + SEL_THREADS - 1) /
                                     SEL_THREADS * SEL_THREADS);
    int t0, t1;
    slice_of(crank, s0, s1, per, t0, t1);
    const int per_warp = per / SEL_WARPS;  // a multiple of 32
    const int w0 = static_cast<int>(min(static_cast<int64_t>(t1), static_cast<int64_t>(t0) + static_cast<int64_t>(per_warp) * warp));
    const int w1 = static_cast<int>(min(static_cast<int64_t>(t1), static_cast<int64_t>(w0) + per_warp));
    // prunable part of the slice [k0, k1); the keys are cached by their offset from t0 when
    // the slice fits the cache (uniform over the cluster), so that a lane's 4 consecutive
    // tokens (offset a multiple of 4) are one 16-byte shared-memory load
    const int k0 = max(t0, p0), k1 = max(k0, min(t1, p1));
    const int nk = k1 - k0;
    const bool cached = per <= SEL_CACHE_KEYS;

    int kk = P;
    if (mode == 0) kk = (kb < 0 || kb > P) ? P : kb;
    const bool do_select = (mode == 0) && kk > 0 && kk < P;
    const bool use_hist = do_select && key_hist != nullptr;

    uint32_t thr = 0;        // the K-th largest key
    int need_eq = 0;         // keys equal to thr that are kept
    bool all_eq_kept = true; // every key equal to thr is kept: no tie ranking needed

    if (tid == 0) sh.counts_known = 0;
    // ------------------------------------------------ cache keys (for the selection and for gls)
    // the score kernel's first-pass counts are loaded together with the keys (one round trip)
    int hv0 = 0, hv1 = 0;
    if (use_hist) {
        const int* kh = key_hist + static_cast<int64_t>(b) * SEL_BINS;
        hv0 = __ldcg(kh + 2 * tid);
        hv1 = __ldcg(kh + 2 * tid + 1);
    }
    const bool need_gls = emit && kk > 0;  // some prunable token is kept: its logsigmoid is emitted
    if (cached && (do_select || need_gls)) {
        for (int c = 0; c < nk; c += 4 * SEL_THREADS) {
            uint32_t v[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int o = c + i * SEL_THREADS + tid;
                v[i] = o < nk ? score_key(__ldcg(scores + k0 + o)) : 0u;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int o = c + i * SEL_THREADS + tid;
                if (o < nk) skeys[k0 - t0 + o] = v[i];
            }
        }
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
            sh.remaining = kk;
            sh.bin_count = 0;
        }
        if (use_hist) {
            // The score kernel took the first pass (the top 11 bits of every key of this
            // sequence): every CTA reads the same counts and finds the same bucket itself, the
            // K-th key from the top (its 64-bucket warp segment, then the bucket), with no
            // cluster round trip.
            int* hist0 = hist_buf;  // free until the passes below
            hist0[2 * tid] = hv0;
            hist0[2 * tid + 1] = hv1;
            const int wsum = warp_sum(hv0 + hv1);
            if (lane == 0) sh.wsum[warp] = wsum;
            __syncthreads();
            if (warp == 0) {
                const int rem = kk;
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
        for (int pass = 0; !(use_hist && sh.remaining == sh.bin_count && sh.width < (1ull << 32)); ++pass) {
            const uint32_t lo = sh.lo;
            const uint64_t width = sh.width;
            const uint64_t range_end = static_cast<uint64_t>(lo) + width;  // keys >= range_end lie above
            const int sh_bits = max(0, bit_length(width - 1) - 11);  // bucket width 2^sh_bits, <= 2048 buckets
            // both buffers alternate by pass: another CTA may still read the previous pass's
            int* hist = hist_buf + (pass & 1) * SEL_BINS;
            int* coarse = sh.coarse[pass & 1];
            hist[tid] = 0;
            hist[tid + SEL_THREADS] = 0;
            if (tid == 0) sh.above[pass & 1] = 0;
            __syncthreads();
            int my_above = 0;
            auto count_key = [&](uint32_t key) {
                const uint32_t d = key - lo;  // wraps for keys below lo: excluded by the range test
                if (key >= lo && static_cast<uint64_t>(d) < width) atomicAdd(&hist[d >> sh_bits], 1);
                my_above += static_cast<uint64_t>(key) >= range_end ? 1 : 0;
            };
            if (cached) {  // 4 keys per load, offsets [k0 - t0, k1 - t0) of the cache
                const int c0 = k0 - t0, c1 = k1 - t0;
                for (int o = (c0 & ~3) + 4 * tid; o < c1; o += 4 * SEL_THREADS) {
                    const uint4 q = *reinterpret_cast<const uint4*>(skeys + o);
                    if (o >= c0 && o + 4 <= c1) {
                        count_key(q.x);
                        count_key(q.y);
                        count_key(q.z);
                        count_key(q.w);
                    } else {
                        const uint32_t kv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            if (o + i >= c0 && o + i < c1) count_key(kv[i]);
                    }
                }
            } else {
#pragma unroll 4
                for (int t = k0 + tid; t < k1; t += SEL_THREADS) count_key(score_key(__ldcg(scores + t)));
            }
            my_above = warp_sum(my_above);
            if (lane == 0 && my_above != 0) atomicAdd(&sh.above[pass & 1], my_above);
            __syncthreads();
            if (pass == 0) SEL_TRACE(13);
            {   // superbin sums: warp w sums buckets [64w, 64w + 64)
                const int a = warp_sum(hist[64 * warp + lane]);
                const int c = warp_sum(hist[64 * warp + 32 + lane]);
                if (lane == 0) {
                    coarse[2 * warp] = a;
                    coarse[2 * warp + 1] = c;
                }
            }
            cl.sync();  // every CTA's histogram, superbin sums and count above of this pass are complete
            if (pass == 0) SEL_TRACE(14);
            if (warp == 0) {
                // the rem-th key from the top: first its superbin (lane l owns superbins
                // 63 - 2l and 62 - 2l of all CTAs), then its bucket (lane l owns bucket
                // 32 S + 31 - l of all CTAs); every CTA finds the same bucket
                const int rem = sh.remaining;
                int vh[SEL_CL], vl[SEL_CL];
                int hi = 0, lo2 = 0;
#pragma unroll
                for (int r = 0; r < SEL_CL; ++r) {
                    const int* cr = cl.map_shared_rank(coarse, r);
                    vh[r] = cr[SEL_SUPER - 1 - 2 * lane];
                    vl[r] = cr[SEL_SUPER - 2 - 2 * lane];
                }
                // lane r < SEL_CL: slice r's keys above the range
                const int ab = lane < SEL_CL ? *cl.map_shared_rank(&sh.above[pass & 1], lane) : 0;
#pragma unroll
                for (int r = 0; r < SEL_CL; ++r) {
                    hi += vh[r];
                    lo2 += vl[r];
                }
                const int incl = warp_inclusive_scan(hi + lo2);
                const int excl = incl - hi - lo2;
                const unsigned hit = __ballot_sync(0xffffffffu, excl < rem && incl >= rem);
                bool decided = false;
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
                    const unsigned hit2 = __ballot_sync(0xffffffffu, excl2 < rem2 && incl2 >= rem2);
                    if (hit2 != 0u) {
                        decided = true;
                        const int Lb = __ffs(hit2) - 1;
                        const int remaining = rem2 - __shfl_sync(0xffffffffu, excl2, Lb);
                        const int bin_count = __shfl_sync(0xffffffffu, cnt, Lb);
                        if (lane == Lb) {
                            const uint64_t new_lo = static_cast<uint64_t>(lo) + (static_cast<uint64_t>(bin) << sh_bits);
                            sh.lo = static_cast<uint32_t>(new_lo);
                            sh.width = min(static_cast<uint64_t>(1) << sh_bits, range_end - new_lo);
                            sh.remaining = remaining;
                            sh.bin_count = bin_count;
                        }
                        if (sh_bits == 0 || pass >= 3 || remaining == bin_count) {
                            // The search ends here, so every slice's count of kept keys follows
                            // from this pass's counts: the keys above the range, the superbins
                            // above S, the buckets of S above the chosen one and, when all of it
                            // is taken, the chosen bucket (else its keys are ranked by index).
                            const bool all_kept = remaining == bin_count;
                            int kept_r = 0, eq_r = 0;  // lane r < SEL_CL: slice r's
#pragma unroll
                            for (int r = 0; r < SEL_CL; ++r) {
                                const int sup = lane < L ? vh[r] + vl[r] : (lane == L && !upper ? vh[r] : 0);
                                const int above_bin = warp_sum(sup + (lane < Lb ? v[r] : 0));
                                const int in_bin = __shfl_sync(0xffffffffu, v[r], Lb);
                                if (lane == r) {
                                    kept_r = ab + above_bin + (all_kept ? in_bin : 0);
                                    eq_r = all_kept ? 0 : in_bin;
                                }
                            }
                            if (lane < SEL_CL) {
                                int a0, a1;
                                slice_of(lane, s0, s1, per, a0, a1);
                                const int b0 = max(a0, p0), b1 = max(b0, min(a1, p1));
                                kept_r += (a1 - a0) - (b1 - b0);  // tokens outside the span are kept
                            }
                            const int ik = warp_inclusive_scan(lane < SEL_CL ? kept_r : 0);
                            const int ie = warp_inclusive_scan(lane < SEL_CL ? eq_r : 0);
                            if (lane == crank) {
                                sh.cta_kept = ik - kept_r;
                                sh.cta_eq = ie - eq_r;
                                sh.counts_known = 1;
                            }
                        }
                    }
                }
                if (!decided && lane == 0) {
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
    } else if (mode == 0 && warp == 0) {
        // no selection: every token outside the span is kept, and every prunable one if kk > 0
        __syncwarp();  // after tid 0 cleared counts_known
        int kept_r = 0;
        if (lane < SEL_CL) {
            int a0, a1;
            slice_of(lane, s0, s1, per, a0, a1);
            const int b0 = max(a0, p0), b1 = max(b0, min(a1, p1));
            kept_r = kk > 0 ? a1 - a0 : (a1 - a0) - (b1 - b0);
        }
        const int ik = warp_inclusive_scan(kept_r);
        if (lane == crank) {
            sh.cta_kept = ik - kept_r;
            sh.cta_eq = 0;
            sh.counts_known = 1;
        }
    }

    // ---------------------------------------------------------------- ordered scan
    // Each lane takes 4 consecutive tokens of its warp's run (128 per warp and step).  flags4
    // sets bit i of kmask when token t + i is kept and of emask when it is a key equal to thr
    // ranked by index (only some of those are kept); t - t0 is a multiple of 4.
    auto flags4 = [&](int t, unsigned& kmask, unsigned& emask) {
        kmask = 0u;
        emask = 0u;
        uint32_t key[4] = {0u, 0u, 0u, 0u};
        if (do_select) {
            if (cached) {
                // In bounds: a warp's last step overruns its run by less than 128 tokens, so
                // t - t0 + 3 < SEL_CACHE_KEYS for every t a lane reaches (per <= SEL_CACHE_KEYS,
                // a multiple of 1024).  Slots of tokens outside [k0, k1) hold stale values, read
                // only for tokens that ignore their key (outside the span or past the run).
                const uint4 q = *reinterpret_cast<const uint4*>(skeys + (t - t0));
                key[0] = q.x;
                key[1] = q.y;
                key[2] = q.z;
                key[3] = q.w;
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (t + i < w1 && t + i >= p0 && t + i < p1) key[i] = score_key(__ldcg(scores + t + i));
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int ti = t + i;
            if (ti >= w1) break;
            const bool prun = ti >= p0 && ti < p1;
            bool kept, eq = false;
            if (mode == 1) {
                kept = __ldcg(keep_in + ti) != 0;
            } else if (!prun) {
                kept = true;
            } else if (!do_select) {
                kept = kk > 0;  // kk >= P keeps all, kk == 0 keeps none
            } else {
                kept = key[i] > thr || (key[i] == thr && all_eq_kept);
                eq = key[i] == thr && !all_eq_kept;
            }
            kmask |= (kept ? 1u : 0u) << i;
            emask |= (eq ? 1u : 0u) << i;
        }
    };
    const unsigned lt_mask = (1u << lane) - 1u;

    // warp totals: kept tokens and (for the tie ranking) keys equal to thr
    int my_kept = 0, my_eq = 0;
    for (int base = w0; base < w1; base += 128) {
        unsigned km, em;
        flags4(base + 4 * lane, km, em);
        my_kept += __popc(km);
        my_eq += __popc(em);
    }
    my_kept = warp_sum(my_kept);
    my_eq = warp_sum(my_eq);
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
    const bool counts_known = sh.counts_known != 0;  // uniform over the cluster
    int cta_kept, cta_eq;
    if (counts_known) {
        __syncthreads();  // the warp prefixes and this CTA's totals are in place
        cta_kept = sh.cta_kept;
        cta_eq = sh.cta_eq;
    } else {
        cl.sync();  // slice totals published
        cta_kept = 0;
        cta_eq = 0;
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
                cta_kept += vk[r];
                cta_eq += ve[r];
            }
        }
    }
    SEL_TRACE(9);
    cluster_arrive_relaxed();  // no remote reads after this point
    // every CTA read the score kernel's counts before a cluster barrier above (the first pass's,
    // or the exchange's): zero them for the next call, each CTA its eighth
    if (key_hist != nullptr && tid < SEL_BINS / SEL_CL)
        key_hist[static_cast<int64_t>(b) * SEL_BINS + crank * (SEL_BINS / SEL_CL) + tid] = 0;
    SEL_TRACE(7);

    // kept_before counts the tie-ranked keys as not kept; min(eq_before, need_eq) of
    // those before this warp's run are kept
    const int kept_before = cta_kept + sh.warp_kept[warp], eq_before = cta_eq + sh.warp_eq[warp];
    const int m_cta = m0 + cta_kept + (all_eq_kept ? 0 : min(cta_eq, need_eq));  // this slice's first entry
    const int n_cta = sh.xchg[0] + (all_eq_kept ? 0 : min(cta_eq + sh.xchg[1], need_eq) - min(cta_eq, need_eq));
    const int m_warp = m0 + kept_before + (all_eq_kept ? 0 : min(eq_before, need_eq));

    // Emission: a walk over each warp's run numbers the kept tokens (and writes the keep flags in
    // its first round); each round lists the tokens of up to SEL_LIST consecutive entries in
    // shared memory, and the threads then write those entries of the map densely.
    const int rounds = max(emit ? (n_cta + SEL_LIST - 1) / SEL_LIST : 0, mode == 0 ? 1 : 0);
    // a lane's 4 tokens start at an offset from s0 that is a multiple of 4
    const bool keep_words = ((reinterpret_cast<uintptr_t>(keep_out) + static_cast<uintptr_t>(s0)) & 3u) == 0;
    for (int round = 0; round < rounds; ++round) {
        const int j_lo = round * SEL_LIST;
        int m = m_warp - m_cta;  // this slice's entry index of the warp's next kept token
        int eq_seen = eq_before;
        for (int base = w0; base < w1; base += 128) {
            const int t = base + 4 * lane;
            unsigned km, em;
            flags4(t, km, em);
            if (!all_eq_kept) {  // the first need_eq keys equal to thr, by index, are kept
                unsigned eb[4];
                int before = eq_seen;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    eb[i] = __ballot_sync(0xffffffffu, (em >> i) & 1u);
                    before += __popc(eb[i] & lt_mask);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (((em >> i) & 1u) && before + __popc(em & ((1u << i) - 1u)) < need_eq) km |= 1u << i;
                eq_seen += __popc(eb[0]) + __popc(eb[1]) + __popc(eb[2]) + __popc(eb[3]);
            }
            int j = m - j_lo, step = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const unsigned kb_ = __ballot_sync(0xffffffffu, (km >> i) & 1u);
                j += __popc(kb_ & lt_mask);
                step += __popc(kb_);
            }
            if (mode == 0 && round == 0) {
                if (keep_words && t + 3 < w1) {  // the 4 flags as one 4-byte store
                    *reinterpret_cast<uint32_t*>(keep_out + t) =
                        (km & 1u) | ((km & 2u) << 7) | ((km & 4u) << 14) | ((km & 8u) << 21);
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        if (t + i < w1) keep_out[t + i] = (km >> i) & 1u;
                }
            }
            if (emit) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if ((km >> i) & 1u) {  // kept tokens lie below w1
                        if (j >= 0 && j < SEL_LIST) list[j] = t + i;
                        ++j;
                    }
                }
            }
            m += step;
        }
        if (round == 0) SEL_TRACE(6);
        if (!emit) break;
        __syncthreads();  // the round's list is complete
        if (round == 0) SEL_TRACE(15);
        const int n_round = min(SEL_LIST, n_cta - j_lo);
        for (int j = tid; j < n_round; j += SEL_THREADS) {
            const int t = list[j];
            const int mi = m_cta + j_lo + j;
            // a caller-given keep vector that disagrees with cu_kept must not write
            // outside [m0, m1)
            if (mi < m1) {
                const bool prun = t >= p0 && t < p1;
                float g = 0.0f;
                if (prun) g = logsigmoid_f(cached ? key_to_score(skeys[t - t0]) : __ldcg(scores + t));
                kept_idx[mi] = t;
                pos[mi] = t - s0 + 1;
                rank[mi] = mi - m0 + 1;
                gls[mi] = g;
            }
        }
        __syncthreads();  // the list is read before the next round writes it
    }
    SEL_TRACE(10);
    cluster_wait();
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
                               cudaStream_t st, int* key_hist, bool early) {
    static std::atomic<uint64_t> attr_set{0};
    if (cudaError_t e = ensure_smem_limit(select_scan_kernel, SEL_SMEM_BYTES, attr_set); e != cudaSuccess)
        return e;
    if (B == 0) return cudaSuccess;
    return launch_pdl(select_scan_kernel, dim3(SEL_CL, B), dim3(SEL_THREADS), static_cast<size_t>(SEL_SMEM_BYTES), st,
                      mode, early ? 1 : 0, scores, keep_in, cu_seqlens, span, k, cu_kept, keep_out, kept_idx, pos, rank, gls,
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
