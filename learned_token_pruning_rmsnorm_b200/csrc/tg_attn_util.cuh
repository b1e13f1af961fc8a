// Device helpers shared by the forward attention kernels: packed fp32 pairs,
// bf16 packing and the (high, low) split of the gate-bias operands, bounded
// drains, loads that read data written during the kernel's lifetime, the
// causal work split's unit numbering and its scratch layout.
#pragma once

#include "tg_sm100.cuh"

namespace tg {
namespace attn {

using namespace sm100;

constexpr int BM = 128;  // query rows per tile (TMEM lanes)
constexpr int BN = 128;  // keys per tile
constexpr float LOG2E = 1.4426950408889634f;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 units: rescale only when the max grows by > 2^8

__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, int* status) {
    volatile int never = 0;
    return mbar_wait(bar, parity, &never, status, TG_WHERE_DRAIN);
}

// Global load that stays where it is written (volatile asm is not moved across the
// other volatile asm statements), so that a prefetch issued a tile ahead is not sunk by the
// compiler to its first use.  It reads through L2 (.cg), not the read-only path: with
// programmatic dependent launch the kernel that writes the compaction map may still be
// running during this kernel's lifetime, and the non-coherent path then returned stale
// values now and then.
__device__ __forceinline__ float ldg_early(const float* p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// max of three floats (one instruction on sm_100)
// Load with acquire semantics at GPU scope: reads that follow it (in this thread, and in
// threads that pass a CTA barrier after it) see every write released before the value read.
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Packed fp32 pairs (lo in bits 0-31): two FMAs or adds per instruction on sm_100.
__device__ __forceinline__ uint64_t f32x2_pack(float lo, float hi) {
    return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float f32x2_lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float f32x2_hi(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// 2^x of a pair of fp32 values on the FMA pipe, to share the exponentials of the softmax
// with the special-function unit.  Cody-Waite style range reduction: adding and removing
// 1.5 * 2^23 rounds x to an integer n (exactly, for |x| < 2^22), f = x - n lies in
// [-0.5, 0.5]; 2^f comes from a degree-3 polynomial whose coefficients were fitted for this
// library (Lawson's iteratively reweighted least squares towards the minimax relative
// error over [-0.5, 0.5]: 7.5e-5 at most, evaluated in fp32), and 2^n is added into the
// exponent field.  Inputs are clamped to >= -125 first, so that the result stays a normal
// number (below that it is a tiny number of at most 2^-124 instead of 0; the softmax only
// passes x <= 0 and sends its masked elements to the special-function unit).
constexpr float EXP2_C0 = 0.9999280571937561f;
constexpr float EXP2_C1 = 0.6932609677314758f;
constexpr float EXP2_C2 = 0.24261116981506348f;
constexpr float EXP2_C3 = 0.05517167970538139f;
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x2) {
    const uint64_t xc = f32x2_pack(fmaxf(f32x2_lo(x2), -125.0f), fmaxf(f32x2_hi(x2), -125.0f));
    const uint64_t j = f32x2_add(xc, f32x2_pack(12582912.0f, 12582912.0f));  // 1.5 * 2^23 + round(x)
    const uint64_t n = f32x2_add(j, f32x2_pack(-12582912.0f, -12582912.0f));
    const uint64_t f = f32x2_fma(n, f32x2_pack(-1.0f, -1.0f), xc);
    uint64_t p = f32x2_fma(f, f32x2_pack(EXP2_C3, EXP2_C3), f32x2_pack(EXP2_C2, EXP2_C2));
    p = f32x2_fma(p, f, f32x2_pack(EXP2_C1, EXP2_C1));
    p = f32x2_fma(p, f, f32x2_pack(EXP2_C0, EXP2_C0));
    // the low bits of j hold n (two's complement): n << 23 moves it into the exponent field
    const uint32_t r0 = static_cast<uint32_t>(p) + (static_cast<uint32_t>(j) << 23);
    const uint32_t r1 = static_cast<uint32_t>(p >> 32) + (static_cast<uint32_t>(j >> 32) << 23);
    return static_cast<uint64_t>(r0) | (static_cast<uint64_t>(r1) << 32);
}

// Named barrier `id` over `n` threads that also returns the OR of `pred` over them.
__device__ __forceinline__ bool bar_red_or(int id, int n, bool pred) {
    uint32_t res;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(res)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(n)
        : "memory");
    return res != 0;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// (high, low) bf16 split of v packed as a pair: high = bf16(v), low = bf16(v - high).
// Infinities are clamped to the largest finite magnitude so that products with a zero
// low part of the other operand stay finite (the sum still overflows to infinity).
__device__ __forceinline__ uint32_t bf16_hi_lo(float v) {
    const float c = fminf(fmaxf(v, -3.0e38f), 3.0e38f);  // NaN stays NaN
    const __nv_bfloat16 hi = __float2bfloat16_rn(isnan(v) ? v : c);
    const float lo = (isnan(v) ? v : c) - __bfloat162float(hi);
    return pack_bf16x2(__bfloat162float(hi), lo);
}

// Causal work split.  Query tile qt of a sequence needs KV tiles 0..qt.  With
// a chunk length C, it is cut into ceil((qt+1)/C) units of at most C KV
// tiles; units are numbered heaviest query tile first, so the block
// scheduler hands out long units first.  units_below(x) counts the units of
// query tiles 0..x-1:  sum_{L=1..x} ceil(L/C) = C*a*(a+1)/2 + r*(a+1), x = a*C + r.
__device__ __forceinline__ int64_t units_below(int x, int C) {
    const int64_t a = x / C, r = x % C;
    return C * a * (a + 1) / 2 + r * (a + 1);
}

// Scratch of the KV split, per split query tile (qt >= C) of each (sequence,
// head pair): nch partial results (O / l in fp32 and m + log2 l per row and
// head) and one arrival counter that the merging CTA resets to zero.
struct SplitWs {
    float* o;       // [slots][max_nch][2][HD/2][BM] bf16 column pairs (sized for fp32; half is used)
    float* lse2;    // [slots][max_nch][2][BM]
    int* cnt;       // [slots][2] (one counter per head of the pair)
    int max_nch;
    int slots_per_pair;  // n_qt_max - C (query tiles that may be split)
};

// Unit number v of one (sequence, head pair) -> (query tile, chunk), in order of
// decreasing cost.  C >= ceil(n_qt / 2): query tiles C..n_qt-1 split into [0, C) and
// [C, qt+1).  Cost C first: every first chunk; then for w = C, C-1, ..., 1 the
// unsplit query tile w-1 and the second chunk of query tile w-1+C (if it exists).
__device__ __forceinline__ void unit_tile(int64_t v, int n_qt, int C, int* qt, int* chunk) {
    *qt = 0;
    *chunk = 0;
    if (C >= n_qt) {
        *qt = n_qt - 1 - static_cast<int>(v);
        return;
    }
    const int a = n_qt - C;
    if (v < a) {
        *qt = n_qt - 1 - static_cast<int>(v);
        return;
    }
    v -= a;
    for (int w = C; w >= 1; --w) {
        if (v == 0) {
            *qt = w - 1;
            return;
        }
        --v;
        if (w - 1 + C <= n_qt - 1) {
            if (v == 0) {
                *qt = w - 1 + C;
                *chunk = 1;
                return;
            }
            --v;
        }
    }
}

// Byte layout of the attention's caller workspace (host and device agree on it):
//   [0, 256)            the persistent kernel's unit counter and finished-CTA counter
//   [cnt_off, o_off)    the causal split's arrival counters, two per split slot
//   [o_off, lse_off)    partial outputs, [lse_off, total) partial log-sum-exps
// The counters, [0, zero_bytes), must be zero before a call and are zero after it.
struct AttnWsLayout {
    size_t cnt_off = 256, o_off = 256, lse_off = 256, total = 0, zero_bytes = 256;
    int C = 1, max_nch = 1, slots_per_pair = 0;
    int64_t slots = 0;
};


}  // namespace attn

// Workspace layout of the forward attention for these sizes (host side; the kernels get
// the pointers it describes).
// per_unit: the layout for the one-CTA-per-unit kernel's chunk choice, else the persistent kernel's
attn::AttnWsLayout attention_ws_layout(int B, int max_M, int Hq, int Hkv, int d, bool per_unit);

// The persistent attention (k_attention_pers.cu): head_dim 64 or 128, GQA groups of
// even size, 1 to kMaxGates gates, or none (gates.n == 0: bias 0, tau 1, c unused).
// Needs the workspace (its unit counter); returns cudaErrorNotSupported when it cannot
// run on this build or device, so that the caller can fall back.
cudaError_t launch_attention_persistent(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                        const int32_t* cu_kept, int B, int64_t M_total, int max_M, int Hq,
                                        int Hkv, int d, const int32_t* pos, const int32_t* rank,
                                        const GateSet& gates, const float* c, float sm_scale, uint16_t* out,
                                        float* lse, void* ws, size_t ws_bytes, bool early, cudaStream_t st);
}  // namespace tg
