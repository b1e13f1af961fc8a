// Internal declarations shared by the CUDA translation units of libtokengate.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>

#include "tokengate.h"

namespace tg {

// Programmatic dependent launch.  Kernels of the path are launched with
// programmatic stream serialisation, so that a kernel can be resident, and
// through the part of its prologue that reads no global memory (barrier init,
// TMEM allocation, descriptor prefetch), while the kernel before it in the
// stream finishes.  Each such kernel executes pdl_wait() before its first read
// of global memory (the wait returns once the preceding grid has completed and
// its writes are visible; without the launch attribute it returns at once) and
// pdl_trigger() after it, which lets the next kernel be scheduled early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// launch_pdl with a 1-D thread-block cluster of `cluster_x` CTAs (grid.x a multiple of it).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                      unsigned cluster_x, Args... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Raises a kernel's dynamic shared-memory limit once per device (the
// attribute is per device; `done` holds one bit per device ordinal).
template <typename Kernel>
inline cudaError_t ensure_smem_limit(Kernel* kernel, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// Device status word bits (see tg_device_status in tokengate.h).
constexpr int TG_DEVICE_TIMEOUT = 1 << 16;   // a bounded wait gave up
constexpr int TG_WHERE_PRODUCER = 1 << 0;    // ... in the TMA producer
constexpr int TG_WHERE_MMA = 1 << 1;         // ... in the MMA issuer
constexpr int TG_WHERE_SOFTMAX = 1 << 2;     // ... in the softmax / epilogue warps
constexpr int TG_WHERE_DRAIN = 1 << 3;       // ... while draining after an abort
constexpr int TG_DEVICE_BAD_INDEX = 1 << 17;  // (TG_DEBUG builds) an index derived from the inputs
                                              // fell outside its array; the access was skipped
constexpr int TG_WHERE_ATTENTION = 1 << 4;    // ... in an attention kernel (cu_kept vs M_total)
constexpr int TG_WHERE_SCORE = 1 << 5;        // ... in the score kernel (cu_seqlens / span vs T)

// TG_DEBUG builds: evaluate `cond` (an index bound derived from the caller's inputs); when
// it fails, record TG_DEVICE_BAD_INDEX | where in the status word and yield false, so that
// the caller skips the access.  Release builds trust the documented contract: always true.
#ifdef TG_DEBUG
#define TG_DEBUG_CHECK(cond, status, where) \
    ((cond) ? true : ((status) ? (atomicOr((status), ::tg::TG_DEVICE_BAD_INDEX | (where)), false) : false))
#else
#define TG_DEBUG_CHECK(cond, status, where) true
#endif

// ------------------------------------------------------------------ device helpers

// Order-preserving map of an fp32 score to uint32 (larger score -> larger key).
// -0 is folded onto +0 so that the two compare equal, as in fp32 comparison;
// every NaN maps to 0, below the key of -inf (0x007FFFFF).
__device__ __forceinline__ uint32_t score_key(float s) {
    if (isnan(s)) return 0u;
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// ------------------------------------------------------------------ launchers
// Each returns cudaSuccess or the launch error; arguments are validated by the
// C ABI layer before these are called.

cudaError_t launch_gate_prepare(const uint16_t* gamma, const uint16_t* W1, int D, int I, uint16_t* Wg,
                                cudaStream_t st);

// key_hist (may be NULL): [B][2048] int32, zero on entry; the kernel adds each scored row to
// bin (score_key(score) >> 21) of its sequence, the selection's first pass (select_scan with
// the same key_hist uses it and leaves it zero again).
cudaError_t launch_score(const uint16_t* hidden, const int32_t* cu_seqlens, const int32_t* span, int B,
                         int64_t T, int D, const uint16_t* Wg, const float* b1, const float* w2, float b2, int I,
                         float eps, float* scores, cudaStream_t st, int* key_hist = nullptr);

// mode 0: select by score (writes keep; the compaction outputs if non-null)
// mode 1: compaction scan from caller-given keep flags
// key_hist (may be NULL): the score kernel's first-pass histogram of these scores; the
// selection then starts from its second pass and zeroes key_hist before it exits.
// early: cu_seqlens, span, k and cu_kept are complete before the kernel's predecessor
// releases it (the caller's, behind a predecessor that waits for the caller's work before it
// releases its dependents), so the kernel reads them before its own wait.
cudaError_t launch_select_scan(int mode, const float* scores, const uint8_t* keep_in, const int32_t* cu_seqlens,
                               const int32_t* span, const int32_t* k, const int32_t* cu_kept, int B, int64_t T,
                               uint8_t* keep_out, int32_t* kept_idx, int32_t* pos, int32_t* rank, float* gls,
                               cudaStream_t st, int* key_hist = nullptr, bool early = false);

// dst[m, :] = src[kept_idx[m], :] for rows of row_bytes bytes (4, 8 or a multiple of 16;
// both pointers aligned to min(row_bytes, 16)); rows whose index lies outside [0, T) are
// left untouched
// wait_at_end: kept_idx and src were complete before the preceding kernel released its
// dependents (an attention launched with inputs_ready does so only once its own wait has
// returned); the kernel then reads at once and waits for its predecessor only before exiting.
cudaError_t launch_gather_bytes(const void* src, const int32_t* kept_idx, int64_t M_total, int64_t T,
                                int64_t row_bytes, void* dst, cudaStream_t st, bool wait_at_end = false);
// dst[idx[m], :] = src[m, :] (rows of row_bytes bytes, as for launch_gather_bytes)
cudaError_t launch_scatter_bytes(const void* src, const int32_t* idx, int64_t M, int64_t T, int64_t row_bytes,
                                 void* dst, cudaStream_t st);
cudaError_t launch_gather_rows(const uint16_t* hidden, const int32_t* kept_idx, int64_t M_total, int64_t T, int D,
                               uint16_t* hidden_kept, cudaStream_t st, bool wait_at_end = false);

// inputs_ready: q, k, v, g, c and cu_kept were complete before the kernel that precedes the
// attention on `st` started (so the attention may load them while that kernel runs; only
// pos, rank, gls and the split scratch wait for it).  Only callers that know the stream's
// history (tg_gated_prefill_layer) may set it.
//
// The gate modules whose biases add up on the attention logits: gate i
// contributes softplus(g[i][h]) * gls[i][j] (one gate is n = 1).  gls[i] is
// indexed by kept row, g[i] by query head.
constexpr int kMaxGates = 4;
struct GateSet {
    const float* gls[kMaxGates];
    const float* g[kMaxGates];
    int n;
};
inline GateSet single_gate(const float* gls, const float* g) {
    GateSet s{};
    s.gls[0] = gls;
    s.g[0] = g;
    s.n = 1;
    return s;
}

cudaError_t launch_gated_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept,
                                   int B, int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                                   const int32_t* rank, const GateSet& gates, const float* c, float sm_scale,
                                   uint16_t* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t st,
                                   bool inputs_ready = false);

// Causal work split of the attention: KV chunk length chosen for a launch,
// scratch bytes the split needs (0 when it never splits), unit count.
int attention_kv_chunk(int B, int max_M, int Hq, int Hkv, bool have_ws, bool per_unit);
// Which two-head kernel a call with a workspace runs (even GQA groups, head_dim <= 128): the
// one-CTA-per-unit kernel for a gated call over one sequence, the persistent kernel otherwise.
// Measured on B200: one CTA per unit is faster on one sequence (46.9 against 50.5 us at 32k
// tokens, K = 2000; 4.13 against 4.57 ms with every token kept), persistent CTAs on a batch of
// unequal sequences (73.7 against 86.0 us on a four-sequence batch).  The environment variable
// TG_ATTENTION_KERNEL = persistent | per_unit overrides the choice (per_unit applies to gated
// calls only: the plain, ungated attention runs persistent CTAs in every case).
bool attention_per_unit_kernel(int B, int n_gates);
cudaError_t launch_gated_attention_noalloc(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                           const int32_t* cu_kept, int B, int64_t M_total, int max_M, int Hq, int Hkv,
                                           int d, const int32_t* pos, const int32_t* rank, const GateSet& gates,
                                           const float* c, float sm_scale, uint16_t* out, float* lse,
                                           cudaStream_t st);
size_t attention_workspace_bytes(int B, int max_M, int Hq, int Hkv, int d);

// Backward of the one-gate attention (head_dim 64 or 128); ws holds
// attention_backward_workspace_bytes(M_total, Hq, Hkv, d) bytes (4 fp32 per row and head,
// plus fp32 partial dK and dV per query head of a GQA group when the group has two or more).
size_t attention_backward_workspace_bytes(int64_t M_total, int Hq, int Hkv, int d);
// gates.n (1..kMaxGates) gates: dgls[i], dg[i] per gate (device arrays), dscore may be a
// null array or hold null entries.
cudaError_t launch_gated_attention_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                            const uint16_t* out, const uint16_t* dout, const float* lse,
                                            const int32_t* cu_kept, int B, int64_t M_total, int max_M, int Hq,
                                            int Hkv, int d, const int32_t* pos, const int32_t* rank,
                                            const GateSet& gates, const float* c, float sm_scale, uint16_t* dq,
                                            uint16_t* dk, uint16_t* dv, float* const* dgls, float* const* dscore,
                                            float* const* dg, float* dc, void* ws, cudaStream_t st);
int64_t units_below_host(int x, int C);

cudaError_t launch_selftest_wait(int64_t timeout_ns, cudaStream_t st);

// y[i] = the attention softmax's FMA-pipe 2^x (exp2_poly_x2) of x[i], device arrays of n floats.
cudaError_t launch_exp2_poly_selftest(const float* x, float* y, int64_t n, cudaStream_t st);

cudaError_t read_device_status(int32_t* word, bool clear, cudaStream_t st);

}  // namespace tg
