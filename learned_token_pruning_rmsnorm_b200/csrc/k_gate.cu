// Stage 1 of the gated prefill: the gate's weight preparation and the gate
// score of every prunable token (TokenGate AI summary, "Key Contributions" 1:
// an MLP over each token's RMSNorm-normalised post-attention residual).
//
//   r_t = 1 / sqrt(mean_i x_ti^2 + eps)
//   s_t = b2 + sum_j w2[j] * SiLU(r_t * (Wg[j,:] . x_t) + b1[j])
// with Wg = bf16(gamma (.) W1^T) prepared once by tg_gate_prepare.

#include "tg_internal.cuh"

namespace tg {
namespace {

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

// Simple CUDA-core scoring kernel: ROWS tokens per CTA, one thread per gate
// unit j (blockDim.x == I), the contraction staged through shared memory in
// chunks of 64 channels.
constexpr int SC_ROWS = 16;
constexpr int SC_KC = 32;

__global__ void __launch_bounds__(256)
score_simple_kernel(const uint16_t* __restrict__ hidden, const int32_t* __restrict__ cu_seqlens,
                    const int32_t* __restrict__ span, int B, int D, const uint16_t* __restrict__ Wg,
                    const float* __restrict__ b1, const float* __restrict__ w2, float b2, int I, float eps,
                    float* __restrict__ scores) {
    __shared__ float xs[SC_ROWS][SC_KC + 1];
    __shared__ float ws[256][SC_KC + 1];
    __shared__ float rs[SC_ROWS];
    __shared__ float red[SC_ROWS][8];
    __shared__ int64_t rows[SC_ROWS];

    // map this CTA's tile to (sequence, first prunable row)
    int64_t tile = blockIdx.x;
    int b = 0;
    int64_t r0 = -1, r1 = -1;
    for (; b < B; ++b) {
        const int64_t s0 = cu_seqlens[b], n = cu_seqlens[b + 1] - s0;
        const int64_t p0 = s0 + min(max(static_cast<int64_t>(span[2 * b]), int64_t(0)), n);
        const int64_t p1 = max(p0, s0 + min(static_cast<int64_t>(span[2 * b + 1]), n));
        const int64_t nt = (p1 - p0 + SC_ROWS - 1) / SC_ROWS;
        if (tile < nt) {
            r0 = p0 + tile * SC_ROWS;
            r1 = p1;
            break;
        }
        tile -= nt;
    }
    if (r0 < 0) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    if (tid < SC_ROWS) rows[tid] = (r0 + tid < r1) ? r0 + tid : -1;
    __syncthreads();
    // sum of squares, one warp per row
    for (int r = warp; r < SC_ROWS; r += nwarps) {
        float ss = 0.f;
        if (rows[r] >= 0)
            for (int i = lane; i < D; i += 32) {
                const float x = bf16_bits_to_float(hidden[rows[r] * D + i]);
                ss = fmaf(x, x, ss);
            }
        for (int off = 16; off; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if (lane == 0) rs[r] = rsqrtf(ss / static_cast<float>(D) + eps);
    }
    float acc[SC_ROWS];
#pragma unroll
    for (int r = 0; r < SC_ROWS; ++r) acc[r] = 0.f;
    const int j = tid;
    for (int k0 = 0; k0 < D; k0 += SC_KC) {
        __syncthreads();
        for (int e = tid; e < SC_ROWS * SC_KC; e += blockDim.x) {
            const int r = e / SC_KC, kk = e % SC_KC;
            xs[r][kk] = rows[r] >= 0 ? bf16_bits_to_float(hidden[rows[r] * D + k0 + kk]) : 0.f;
        }
        for (int e = tid; e < I * SC_KC; e += blockDim.x) {
            const int jj = e / SC_KC, kk = e % SC_KC;
            ws[jj][kk] = bf16_bits_to_float(Wg[static_cast<int64_t>(jj) * D + k0 + kk]);
        }
        __syncthreads();
        if (j < I) {
            for (int kk = 0; kk < SC_KC; ++kk) {
                const float w = ws[j][kk];
#pragma unroll
                for (int r = 0; r < SC_ROWS; ++r) acc[r] = fmaf(w, xs[r][kk], acc[r]);
            }
        }
    }
    // epilogue: SiLU, output layer, reduction over j
    for (int r = 0; r < SC_ROWS; ++r) {
        float v = 0.f;
        if (j < I) {
            const float z = fmaf(rs[r], acc[r], b1[j]);
            v = w2[j] * (z / (1.0f + expf(-z)));
        }
        for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) red[r][warp] = v;
    }
    __syncthreads();
    if (tid < SC_ROWS && rows[tid] >= 0) {
        float s = b2;
        for (int w = 0; w < nwarps; ++w) s += red[tid][w];
        scores[rows[tid]] = s;
    }
}

}  // namespace

cudaError_t launch_gate_prepare(const uint16_t* gamma, const uint16_t* W1, int D, int I, uint16_t* Wg,
                                cudaStream_t st) {
    const int64_t n = static_cast<int64_t>(I) * D;
    const int grid = static_cast<int>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    gate_prepare_kernel<<<grid, 256, 0, st>>>(gamma, W1, D, I, Wg);
    return cudaGetLastError();
}

cudaError_t launch_score(const uint16_t* hidden, const int32_t* cu_seqlens, const int32_t* span, int B,
                         int64_t T, int D, const uint16_t* Wg, const float* b1, const float* w2, float b2, int I,
                         float eps, float* scores, cudaStream_t st) {
    const int64_t tiles = (T + SC_ROWS - 1) / SC_ROWS + B;  // upper bound over all spans
    if (tiles <= 0) return cudaSuccess;
    score_simple_kernel<<<static_cast<unsigned>(tiles), 256, 0, st>>>(hidden, cu_seqlens, span, B, D, Wg, b1, w2, b2,
                                                                     I, eps, scores);
    return cudaGetLastError();
}

}  // namespace tg
