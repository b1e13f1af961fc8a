// Stage 4 of the gated prefill: token-gated causal GQA attention over the kept
// tokens (TokenGate AI summary, "Key Contributions" 2 and 3).
//
//   logit[q,j] = (q.k_j * sm_scale + softplus(g_h) * gls_j) / tau[q,h]
//   tau[q,h]   = 1 + c_h * ln(pos_q / rank_q)
//   o_q        = sum_j softmax_j(logit[q,:]) v_j     over kept j <= q
//
// Simple warp-per-(query, head) kernel with an online softmax in fp32.

#include "tg_internal.cuh"

namespace tg {
namespace {

__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))); }

template <int HD>
__global__ void __launch_bounds__(128)
attn_simple_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                   const int32_t* __restrict__ cu_kept, int B, int64_t M, int Hq, int Hkv,
                   const int32_t* __restrict__ pos, const int32_t* __restrict__ rank, const float* __restrict__ gls,
                   const float* __restrict__ g, const float* __restrict__ c, float sm_scale,
                   uint16_t* __restrict__ out, float* __restrict__ lse) {
    constexpr int E = HD / 32;
    const int lane = threadIdx.x & 31;
    const int64_t wid = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (wid >= M * Hq) return;
    const int64_t i = wid / Hq;
    const int h = static_cast<int>(wid - i * Hq);
    int b = 0;
    while (b + 1 < B && cu_kept[b + 1] <= i) ++b;
    const int64_t j0 = cu_kept[b];
    const int hk = h / (Hq / Hkv);

    float qv[E];
#pragma unroll
    for (int e = 0; e < E; ++e) qv[e] = bf16_bits_to_float(q[(i * Hq + h) * HD + lane * E + e]);
    const float gain = softplus_f(g[h]);
    const float tau = 1.0f + c[h] * logf(static_cast<float>(pos[i]) / static_cast<float>(rank[i]));
    const float inv_tau = 1.0f / tau;
    float m = -INFINITY, l = 0.f, acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int64_t j = j0; j <= i; ++j) {
        const uint16_t* kr = k + (j * Hkv + hk) * HD + lane * E;
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) dot = fmaf(qv[e], bf16_bits_to_float(kr[e]), dot);
#pragma unroll
        for (int off = 16; off; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        const float logit = (dot * sm_scale + gain * gls[j]) * inv_tau;
        const float m_new = fmaxf(m, logit);
        const float corr = expf(m - m_new);
        const float p = expf(logit - m_new);
        l = l * corr + p;
        const uint16_t* vr = v + (j * Hkv + hk) * HD + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(p, bf16_bits_to_float(vr[e]), acc[e] * corr);
        m = m_new;
    }
    const float inv_l = 1.0f / l;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const __nv_bfloat16 r = __float2bfloat16_rn(acc[e] * inv_l);
        out[(i * Hq + h) * HD + lane * E + e] = *reinterpret_cast<const uint16_t*>(&r);
    }
    if (lse && lane == 0) lse[i * Hq + h] = m + logf(l);
}

}  // namespace

cudaError_t launch_gated_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept,
                                   int B, int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                                   const int32_t* rank, const float* gls, const float* g, const float* c,
                                   float sm_scale, uint16_t* out, float* lse, cudaStream_t st) {
    (void)max_M;
    const int64_t warps = M_total * Hq;
    if (warps == 0) return cudaSuccess;
    const unsigned grid = static_cast<unsigned>((warps + 3) / 4);
    if (d == 64)
        attn_simple_kernel<64><<<grid, 128, 0, st>>>(q, k, v, cu_kept, B, M_total, Hq, Hkv, pos, rank, gls, g, c,
                                                     sm_scale, out, lse);
    else
        attn_simple_kernel<128><<<grid, 128, 0, st>>>(q, k, v, cu_kept, B, M_total, Hq, Hkv, pos, rank, gls, g, c,
                                                      sm_scale, out, lse);
    return cudaGetLastError();
}

}  // namespace tg
