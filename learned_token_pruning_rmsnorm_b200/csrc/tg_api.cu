// C ABI of libtokengate.so: argument validation, then the stage launches.
// Every entry point checks its arguments on the host and returns before any
// launch when they are wrong; no exception crosses the ABI.

#include <cstdarg>
#include <cstdio>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "tg_internal.cuh"

namespace {

// NVTX range over one entry point (host side: argument checks and the launches it
// enqueues), named after the call, so that a profiler's timeline shows each stage.  The
// NVTX calls are no-ops unless a profiling tool is attached.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

thread_local std::string g_last_error;

tg_status fail(tg_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

tg_status cuda_status(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return TG_OK;
    return fail(TG_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// The kernels are built for sm_100a only.
tg_status check_device() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return fail(TG_ERR_UNSUPPORTED, "device %d is sm_%d%d; libtokengate is built for sm_100a only", dev, major,
                    minor);
    return TG_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define TG_REQUIRE(cond, ...)                                   \
    do {                                                        \
        if (!(cond)) return fail(TG_ERR_INVALID_ARG, __VA_ARGS__); \
    } while (0)

#define TG_SUPPORT(cond, ...)                                   \
    do {                                                        \
        if (!(cond)) return fail(TG_ERR_UNSUPPORTED, __VA_ARGS__); \
    } while (0)

tg_status check_gate_shape(int D, int I) {
    TG_SUPPORT(D >= 64 && D <= 8192 && D % 64 == 0, "D=%d must be a multiple of 64 in [64, 8192]", D);
    TG_SUPPORT(I >= 16 && I <= 256 && I % 16 == 0, "I=%d must be a multiple of 16 in [16, 256]", I);
    return TG_OK;
}

tg_status check_attn_shape(int Hq, int Hkv, int d) {
    TG_SUPPORT(d == 64 || d == 128 || d == 256, "head_dim %d must be 64, 128 or 256", d);
    TG_REQUIRE(Hq > 0 && Hkv > 0 && Hq % Hkv == 0, "Hq=%d must be a positive multiple of Hkv=%d", Hq, Hkv);
    TG_SUPPORT(Hq <= 256, "Hq=%d above 256", Hq);
    return TG_OK;
}

tg_status do_score(const uint16_t* hidden, const int32_t* cu_seqlens, const int32_t* span, int B, int64_t T, int D,
                   const uint16_t* Wg, const float* b1, const float* w2, float b2, int I, float eps, float* scores,
                   cudaStream_t st) {
    TG_REQUIRE(B >= 0 && T >= 0, "B=%d, T=%lld must be non-negative", B, (long long)T);
    if (tg_status s = check_gate_shape(D, I)) return s;
    TG_REQUIRE(eps >= 0.f, "eps must be >= 0");
    if (B == 0 || T == 0) return TG_OK;
    TG_REQUIRE(hidden && cu_seqlens && span && Wg && b1 && w2 && scores, "null pointer argument");
    TG_REQUIRE(aligned16(hidden) && aligned16(Wg), "hidden and Wg must be 16-byte aligned");
    if (tg_status s = check_device()) return s;
    return cuda_status(tg::launch_score(hidden, cu_seqlens, span, B, T, D, Wg, b1, w2, b2, I, eps, scores, st),
                       "tg_score launch");
}

tg_status do_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept, int B,
                       int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos, const int32_t* rank,
                       const tg::GateSet& gates, const float* c, float sm_scale, uint16_t* out, float* lse,
                       void* ws, size_t ws_bytes, cudaStream_t st, bool inputs_ready = false) {
    TG_REQUIRE(B >= 0 && M_total >= 0 && max_M >= 0, "negative size");
    if (tg_status s = check_attn_shape(Hq, Hkv, d)) return s;
    TG_REQUIRE(sm_scale > 0.f, "sm_scale must be positive");
    TG_SUPPORT(gates.n >= 0 && gates.n <= tg::kMaxGates, "n_gates=%d must be in [0, %d]", gates.n, tg::kMaxGates);
    if (gates.n == 0) {
        // no gate: ordinary causal attention (bias 0, tau 1) on the persistent kernel
        TG_SUPPORT(d <= 128 && (Hq / Hkv) % 2 == 0,
                   "attention without a gate needs head_dim 64 or 128 and an even GQA group (Hq/Hkv=%d, d=%d)",
                   Hq / Hkv, d);
        TG_REQUIRE(ws != nullptr, "attention without a gate needs ws (tg_gated_attention_workspace_size bytes)");
    }
    if (B == 0 || M_total == 0) return TG_OK;
    TG_REQUIRE(max_M > 0, "max_M must bound the longest sequence");
    for (int i = 0; i < gates.n; ++i) TG_REQUIRE(gates.gls[i] && gates.g[i], "null gls or g of gate %d", i);
    TG_REQUIRE(q && k && v && cu_kept && out, "null pointer argument");
    TG_REQUIRE(gates.n == 0 || (pos && rank && c), "null pos, rank or c");
    TG_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out),
               "q, k, v and out must be 16-byte aligned");
    if (ws) {
        TG_REQUIRE((reinterpret_cast<uintptr_t>(ws) & 255u) == 0, "ws must be 256-byte aligned");
        const size_t need = tg::attention_workspace_bytes(B, max_M, Hq, Hkv, d);
        TG_REQUIRE(ws_bytes >= need, "ws holds %zu bytes, the causal split needs %zu", ws_bytes, need);
    }
    if (tg_status s = check_device()) return s;
    return cuda_status(tg::launch_gated_attention(q, k, v, cu_kept, B, M_total, max_M, Hq, Hkv, d, pos, rank, gates,
                                                  c, sm_scale, out, lse, ws, ws_bytes, st, inputs_ready),
                       "tg_gated_attention launch");
}

// The prefill layer's workspace: the attention's scratch, then (256-byte aligned) the
// selection's first-pass histogram, [B][2048] int32, which the score kernel fills and the
// selection reads and zeroes again.
size_t prefill_key_hist_offset(int B, int max_M, int Hq, int Hkv, int d, int n_layers) {
    const size_t attn = n_layers > 0 ? tg_gated_attention_workspace_size(B, max_M, Hq, Hkv, d) : 0;
    return (attn + 255) & ~static_cast<size_t>(255);
}
size_t prefill_key_hist_bytes(int B) { return static_cast<size_t>(B) * 2048 * sizeof(int32_t); }

// Scratch of tg_masked_gated_attention: keep flags, compaction map, the gathered
// Q/K/V rows, the compacted output and the attention's own split scratch, each
// 256-byte aligned.
struct MaskedWs {
    size_t keep, idx, pos, rank, gls, qc, kc, vc, oc, attn, attn_bytes, total;
};

MaskedWs masked_layout(int B, int64_t T, int64_t M, int max_M, int Hq, int Hkv, int d) {
    auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    MaskedWs L{};
    size_t o = 0;
    L.keep = o; o += al(static_cast<size_t>(T));
    L.idx = o; o += al(4 * static_cast<size_t>(M));
    L.pos = o; o += al(4 * static_cast<size_t>(M));
    L.rank = o; o += al(4 * static_cast<size_t>(M));
    L.gls = o; o += al(4 * static_cast<size_t>(M));
    L.qc = o; o += al(2 * static_cast<size_t>(M) * Hq * d);
    L.kc = o; o += al(2 * static_cast<size_t>(M) * Hkv * d);
    L.vc = o; o += al(2 * static_cast<size_t>(M) * Hkv * d);
    L.oc = o; o += al(2 * static_cast<size_t>(M) * Hq * d);
    L.attn = o;
    L.attn_bytes = B > 0 && max_M > 0 ? tg::attention_workspace_bytes(B, max_M, Hq, Hkv, d) : 0;
    o += al(L.attn_bytes);
    L.total = o;
    return L;
}

}  // namespace

extern "C" {

size_t tg_masked_gated_attention_workspace_size(int B, int64_t T, int64_t M_total, int max_M, int Hq, int Hkv, int d) {
    if (B <= 0 || T <= 0 || M_total < 0 || max_M < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 ||
        (d != 64 && d != 128 && d != 256))
        return 0;
    return masked_layout(B, T, M_total, max_M, Hq, Hkv, d).total;
}

tg_status tg_masked_gated_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* scores,
                                    const int32_t* cu_seqlens, const int32_t* span, const int32_t* kbud,
                                    const int32_t* cu_kept, int B, int64_t T, int64_t M_total, int max_M, int Hq,
                                    int Hkv, int d, const float* g, const float* c, float sm_scale, uint16_t* out,
                                    uint8_t* keep_out, void* ws, size_t ws_bytes, tg_stream_t stream) {
    NvtxRange nvtx_range("tg_masked_gated_attention");
    TG_REQUIRE(B >= 0 && T >= 0 && M_total >= 0 && M_total <= T && max_M >= 0, "bad sizes");
    if (tg_status s = check_attn_shape(Hq, Hkv, d)) return s;
    TG_REQUIRE(sm_scale > 0.f, "sm_scale must be positive");
    if (B == 0 || T == 0) return TG_OK;
    TG_REQUIRE(q && k && v && scores && cu_seqlens && span && kbud && cu_kept && g && c && out && ws,
               "null pointer argument");
    TG_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out),
               "q, k, v and out must be 16-byte aligned");
    TG_REQUIRE((reinterpret_cast<uintptr_t>(ws) & 255u) == 0, "ws must be 256-byte aligned");
    TG_REQUIRE(M_total == 0 || max_M > 0, "max_M must bound the longest kept sequence");
    const MaskedWs L = masked_layout(B, T, M_total, max_M, Hq, Hkv, d);
    TG_REQUIRE(ws_bytes >= L.total, "ws holds %zu bytes, this call needs %zu", ws_bytes, L.total);
    if (tg_status s = check_device()) return s;
    cudaStream_t st = stream;
    uint8_t* base = static_cast<uint8_t*>(ws);
    uint8_t* keep = keep_out ? keep_out : base + L.keep;
    int32_t* idx = reinterpret_cast<int32_t*>(base + L.idx);
    int32_t* pos = reinterpret_cast<int32_t*>(base + L.pos);
    int32_t* rank = reinterpret_cast<int32_t*>(base + L.rank);
    float* gls = reinterpret_cast<float*>(base + L.gls);
    uint16_t* qc = reinterpret_cast<uint16_t*>(base + L.qc);
    uint16_t* kc = reinterpret_cast<uint16_t*>(base + L.kc);
    uint16_t* vc = reinterpret_cast<uint16_t*>(base + L.vc);
    uint16_t* oc = reinterpret_cast<uint16_t*>(base + L.oc);
    // rows of pruned queries are zero; the kept rows are overwritten below
    if (tg_status s = cuda_status(cudaMemsetAsync(out, 0, static_cast<size_t>(T) * Hq * d * 2, st), "out clear"))
        return s;
    if (tg_status s = cuda_status(tg::launch_select_scan(0, scores, nullptr, cu_seqlens, span, kbud, cu_kept, B, T,
                                                         keep, idx, pos, rank, gls, st),
                                  "masked select launch"))
        return s;
    if (M_total == 0) return TG_OK;
    const int64_t qrow = static_cast<int64_t>(Hq) * d * 2, kvrow = static_cast<int64_t>(Hkv) * d * 2;
    if (tg_status s = cuda_status(tg::launch_gather_bytes(q, idx, M_total, T, qrow, qc, st), "q gather")) return s;
    if (tg_status s = cuda_status(tg::launch_gather_bytes(k, idx, M_total, T, kvrow, kc, st), "k gather")) return s;
    if (tg_status s = cuda_status(tg::launch_gather_bytes(v, idx, M_total, T, kvrow, vc, st), "v gather")) return s;
    if (tg_status s = do_attention(qc, kc, vc, cu_kept, B, M_total, max_M, Hq, Hkv, d, pos, rank,
                                   tg::single_gate(gls, g), c, sm_scale, oc, nullptr,
                                   L.attn_bytes ? base + L.attn : nullptr, L.attn_bytes, st))
        return s;
    return cuda_status(tg::launch_scatter_bytes(oc, idx, M_total, T, qrow, out, st), "out scatter");
}


int tg_abi_version(void) { return 5; }

const char* tg_last_error_string(void) { return g_last_error.c_str(); }

int64_t tg_kept_count(const int32_t* h_cu_seqlens, const int32_t* h_span, const int32_t* h_k, int B,
                      int32_t* h_cu_kept) {
    if (B < 0 || (B > 0 && (!h_cu_seqlens || !h_span || !h_k)) || !h_cu_kept) {
        fail(TG_ERR_INVALID_ARG, "tg_kept_count: bad arguments");
        return -1;
    }
    int64_t tot = 0;
    h_cu_kept[0] = 0;
    for (int b = 0; b < B; ++b) {
        const int64_t n = static_cast<int64_t>(h_cu_seqlens[b + 1]) - h_cu_seqlens[b];
        const int64_t p0 = h_span[2 * b], p1 = h_span[2 * b + 1];
        if (n < 0 || p0 < 0 || p1 < p0 || p1 > n) {
            fail(TG_ERR_INVALID_ARG, "tg_kept_count: sequence %d: length %lld, span [%lld, %lld)", b, (long long)n,
                 (long long)p0, (long long)p1);
            return -1;
        }
        const int64_t P = p1 - p0;
        const int64_t kk = (h_k[b] < 0 || h_k[b] > P) ? P : h_k[b];
        tot += (n - P) + kk;
        if (tot > INT32_MAX) {
            fail(TG_ERR_INVALID_ARG, "tg_kept_count: total above 2^31-1");
            return -1;
        }
        h_cu_kept[b + 1] = static_cast<int32_t>(tot);
    }
    return tot;
}

tg_status tg_gate_prepare(const uint16_t* gamma, const uint16_t* W1, int D, int I, uint16_t* Wg, tg_stream_t stream) {
    NvtxRange nvtx_range("tg_gate_prepare");
    if (tg_status s = check_gate_shape(D, I)) return s;
    TG_REQUIRE(gamma && W1 && Wg, "null pointer argument");
    if (tg_status s = check_device()) return s;
    return cuda_status(tg::launch_gate_prepare(gamma, W1, D, I, Wg, stream), "tg_gate_prepare launch");
}

tg_status tg_score(const uint16_t* hidden, const int32_t* cu_seqlens, const int32_t* span, int B, int64_t T, int D,
                   const uint16_t* Wg, const float* b1, const float* w2, float b2, int I, float eps, float* scores,
                   tg_stream_t stream) {
    NvtxRange nvtx_range("tg_score");
    return do_score(hidden, cu_seqlens, span, B, T, D, Wg, b1, w2, b2, I, eps, scores, stream);
}

tg_status tg_select_topk(const float* scores, const int32_t* cu_seqlens, const int32_t* span, const int32_t* k, int B,
                         int64_t T, uint8_t* keep, const int32_t* cu_kept, int32_t* kept_idx, int32_t* pos,
                         int32_t* rank, float* gls, tg_stream_t stream) {
    NvtxRange nvtx_range("tg_select_topk");
    TG_REQUIRE(B >= 0 && T >= 0, "negative size");
    if (B == 0 || T == 0) return TG_OK;
    TG_REQUIRE(scores && cu_seqlens && span && k && keep, "null pointer argument");
    const bool emit = cu_kept && kept_idx;
    TG_REQUIRE(!emit || (pos && rank && gls), "the fused compaction map needs pos, rank and gls");
    if (tg_status s = check_device()) return s;
    return cuda_status(tg::launch_select_scan(0, scores, nullptr, cu_seqlens, span, k, emit ? cu_kept : nullptr, B, T,
                                              keep, emit ? kept_idx : nullptr, pos, rank, gls, stream),
                       "tg_select_topk launch");
}

tg_status tg_compact(const uint16_t* hidden, const float* scores, const uint8_t* keep, const int32_t* cu_seqlens,
                     const int32_t* span, int B, int64_t T, int D, const int32_t* cu_kept, int64_t M_total,
                     uint16_t* hidden_kept, int32_t* pos, int32_t* rank, float* gls, int32_t* kept_idx,
                     tg_stream_t stream) {
    NvtxRange nvtx_range("tg_compact");
    TG_REQUIRE(B >= 0 && T >= 0 && M_total >= 0 && M_total <= T, "bad sizes (B=%d T=%lld M=%lld)", B, (long long)T,
               (long long)M_total);
    if (B == 0 || T == 0 || M_total == 0) return TG_OK;  // nothing is kept: no output to write
    TG_REQUIRE(kept_idx, "null kept_idx");
    if (keep) TG_REQUIRE(scores && cu_seqlens && span && cu_kept && pos && rank && gls, "null pointer argument");
    else TG_REQUIRE(hidden_kept, "keep == NULL gathers rows: hidden_kept is required");
    if (hidden_kept) {
        TG_SUPPORT(D >= 8 && D % 8 == 0, "D=%d must be a multiple of 8 for the row copy", D);
        TG_REQUIRE(hidden && aligned16(hidden) && aligned16(hidden_kept), "hidden rows must be 16-byte aligned");
    }
    if (tg_status s = check_device()) return s;
    tg_status s = TG_OK;
    if (keep)
        s = cuda_status(tg::launch_select_scan(1, scores, keep, cu_seqlens, span, nullptr, cu_kept, B, T, nullptr,
                                               kept_idx, pos, rank, gls, stream),
                        "tg_compact scan launch");
    if (s != TG_OK || !hidden_kept) return s;
    return cuda_status(tg::launch_gather_rows(hidden, kept_idx, M_total, T, D, hidden_kept, stream),
                       "tg_compact gather launch");
}

tg_status tg_gather_rows(const void* src, int64_t T, int64_t row_bytes, const int32_t* kept_idx, int64_t M, void* dst,
                         tg_stream_t stream) {
    NvtxRange nvtx_range("tg_gather_rows");
    TG_REQUIRE(T >= 0 && M >= 0 && row_bytes >= 0, "negative size");
    if (M == 0 || row_bytes == 0) return TG_OK;
    TG_REQUIRE(src && kept_idx && dst, "null pointer argument");
    TG_SUPPORT(row_bytes == 4 || row_bytes == 8 || row_bytes % 16 == 0,
               "row_bytes=%lld must be 4, 8 or a multiple of 16", (long long)row_bytes);
    const uintptr_t amask = static_cast<uintptr_t>(row_bytes < 16 ? row_bytes : 16) - 1;
    TG_REQUIRE(((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & amask) == 0,
               "src and dst must be aligned to %d bytes", static_cast<int>(amask + 1));
    // the kernels read src and write dst through restrict pointers, all of a row's loads
    // before its stores: an in-place or overlapping gather would return wrong rows
    {
        const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), d0 = reinterpret_cast<uintptr_t>(dst);
        const uintptr_t s1 = s0 + static_cast<uintptr_t>(T) * static_cast<uintptr_t>(row_bytes);
        const uintptr_t d1 = d0 + static_cast<uintptr_t>(M) * static_cast<uintptr_t>(row_bytes);
        TG_REQUIRE(s0 == d0 ? false : (s1 <= d0 || d1 <= s0), "src [T rows] and dst [M rows] must not overlap");
    }
    if (tg_status s = check_device()) return s;
    return cuda_status(tg::launch_gather_bytes(src, kept_idx, M, T, row_bytes, dst, stream), "tg_gather_rows launch");
}

tg_status tg_gated_attention_noalloc(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept,
                                     int B, int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                                     const int32_t* rank, const float* gls, const float* g, const float* c,
                                     float sm_scale, uint16_t* out, float* lse, tg_stream_t stream) {
    NvtxRange nvtx_range("tg_gated_attention_noalloc");
    TG_REQUIRE(B >= 0 && M_total >= 0 && max_M >= 0, "negative size");
    if (tg_status s = check_attn_shape(Hq, Hkv, d)) return s;
    TG_REQUIRE(sm_scale > 0.f, "sm_scale must be positive");
    if (B == 0 || M_total == 0) return TG_OK;
    TG_REQUIRE(max_M > 0, "max_M must bound the longest sequence");
    TG_REQUIRE(q && k && v && cu_kept && pos && rank && gls && g && c && out, "null pointer argument");
    TG_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out),
               "q, k, v and out must be 16-byte aligned");
    if (tg_status s = check_device()) return s;
    const tg::GateSet gates = tg::single_gate(gls, g);
    const size_t need = tg::attention_workspace_bytes(B, max_M, Hq, Hkv, d);
    TG_SUPPORT(need <= TG_NOALLOC_ATTENTION_SCRATCH_BYTES,
               "tg_gated_attention_noalloc: these sizes need %zu bytes of scratch, above the fixed %zu-byte array; "
               "use tg_gated_attention with a caller workspace",
               need, static_cast<size_t>(TG_NOALLOC_ATTENTION_SCRATCH_BYTES));
    return cuda_status(tg::launch_gated_attention_noalloc(q, k, v, cu_kept, B, M_total, max_M, Hq, Hkv, d, pos, rank,
                                                          gates, c, sm_scale, out, lse, stream),
                       "tg_gated_attention_noalloc launch");
}

size_t tg_gated_attention_workspace_size(int B, int max_M, int Hq, int Hkv, int d) {
    if (B <= 0 || max_M <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || (d != 64 && d != 128 && d != 256)) return 0;
    return tg::attention_workspace_bytes(B, max_M, Hq, Hkv, d);
}

size_t tg_gated_prefill_workspace_size(int B, int max_M, int Hq, int Hkv, int d, int n_layers) {
    if (B <= 0) return 0;
    return prefill_key_hist_offset(B, max_M, Hq, Hkv, d, n_layers) + prefill_key_hist_bytes(B);
}

tg_status tg_gated_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept, int B,
                             int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                             const int32_t* rank, const float* gls, const float* g, const float* c, float sm_scale,
                             uint16_t* out, float* lse, void* ws, size_t ws_bytes, tg_stream_t stream) {
    NvtxRange nvtx_range("tg_gated_attention");
    tg::GateSet gates = tg::single_gate(gls, g);
    if (!gls && !g && !c) gates.n = 0;  // no gate: ordinary causal attention
    return do_attention(q, k, v, cu_kept, B, M_total, max_M, Hq, Hkv, d, pos, rank, gates, c, sm_scale, out, lse, ws,
                        ws_bytes, stream);
}

tg_status tg_gated_attention_gates(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept,
                                   int B, int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                                   const int32_t* rank, int n_gates, const float* const* gls, const float* const* g,
                                   const float* c, float sm_scale, uint16_t* out, float* lse, void* ws,
                                   size_t ws_bytes, tg_stream_t stream) {
    NvtxRange nvtx_range("tg_gated_attention_gates");
    TG_SUPPORT(n_gates >= 1 && n_gates <= tg::kMaxGates, "n_gates=%d must be in [1, %d]", n_gates, tg::kMaxGates);
    TG_REQUIRE(gls && g, "null gate arrays");
    tg::GateSet gates{};
    gates.n = n_gates;
    for (int i = 0; i < n_gates; ++i) {
        gates.gls[i] = gls[i];
        gates.g[i] = g[i];
    }
    return do_attention(q, k, v, cu_kept, B, M_total, max_M, Hq, Hkv, d, pos, rank, gates, c, sm_scale, out, lse, ws,
                        ws_bytes, stream);
}

size_t tg_gated_attention_backward_workspace_size(int64_t M_total, int Hq, int Hkv, int d) {
    if (M_total <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || (d != 64 && d != 128 && d != 256)) return 0;
    return tg::attention_backward_workspace_bytes(M_total, Hq, Hkv, d);
}

}  // extern "C"

namespace {

tg_status do_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* out,
                      const uint16_t* dout, const float* lse, const int32_t* cu_kept, int B, int64_t M_total, int max_M,
                      int Hq, int Hkv, int d, const int32_t* pos, const int32_t* rank, const tg::GateSet& gates,
                      const float* c, float sm_scale, uint16_t* dq, uint16_t* dk, uint16_t* dv, float* const* dgls,
                      float* const* dscore, float* const* dg, float* dc, void* ws, size_t ws_bytes,
                      cudaStream_t stream) {
    TG_REQUIRE(B >= 0 && M_total >= 0 && max_M >= 0, "negative size");
    if (tg_status s = check_attn_shape(Hq, Hkv, d)) return s;
    TG_REQUIRE(sm_scale > 0.f, "sm_scale must be positive");
    TG_SUPPORT(gates.n >= 1 && gates.n <= tg::kMaxGates, "n_gates=%d must be in [1, %d]", gates.n, tg::kMaxGates);
    if (B == 0 || M_total == 0) return TG_OK;
    TG_REQUIRE(max_M > 0, "max_M must bound the longest sequence");
    TG_REQUIRE(q && k && v && out && dout && lse && cu_kept && pos && rank && c && dq && dk && dv && dgls && dg &&
                   dc && ws,
               "null pointer argument");
    for (int i = 0; i < gates.n; ++i)
        TG_REQUIRE(gates.gls[i] && gates.g[i] && dgls[i] && dg[i], "null gls, g, dgls or dg of gate %d", i);
    TG_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out) && aligned16(dout) && aligned16(dq) &&
                   aligned16(dk) && aligned16(dv),
               "q, k, v, out, dout, dq, dk and dv must be 16-byte aligned");
    TG_REQUIRE((reinterpret_cast<uintptr_t>(ws) & 255u) == 0, "ws must be 256-byte aligned");
    const size_t need = tg::attention_backward_workspace_bytes(M_total, Hq, Hkv, d);
    TG_REQUIRE(ws_bytes >= need, "ws holds %zu bytes, the backward needs %zu", ws_bytes, need);
    if (tg_status s = check_device()) return s;
    return cuda_status(tg::launch_gated_attention_backward(q, k, v, out, dout, lse, cu_kept, B, M_total, max_M, Hq,
                                                           Hkv, d, pos, rank, gates, c, sm_scale, dq, dk, dv, dgls,
                                                           dscore, dg, dc, ws, stream),
                       "tg_gated_attention_backward launch");
}

}  // namespace

extern "C" {

tg_status tg_gated_attention_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* out,
                                      const uint16_t* dout, const float* lse, const int32_t* cu_kept, int B,
                                      int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                                      const int32_t* rank, const float* gls, const float* g, const float* c,
                                      float sm_scale, uint16_t* dq, uint16_t* dk, uint16_t* dv, float* dgls,
                                      float* dscore, float* dg, float* dc, void* ws, size_t ws_bytes,
                                      tg_stream_t stream) {
    NvtxRange nvtx_range("tg_gated_attention_backward");
    float* dgl[1] = {dgls};
    float* dsc[1] = {dscore};
    float* dgg[1] = {dg};
    return do_backward(q, k, v, out, dout, lse, cu_kept, B, M_total, max_M, Hq, Hkv, d, pos, rank,
                       tg::single_gate(gls, g), c, sm_scale, dq, dk, dv, dgl, dsc, dgg, dc, ws, ws_bytes, stream);
}

tg_status tg_gated_attention_backward_gates(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                            const uint16_t* out, const uint16_t* dout, const float* lse,
                                            const int32_t* cu_kept, int B, int64_t M_total, int max_M, int Hq,
                                            int Hkv, int d, const int32_t* pos, const int32_t* rank, int n_gates,
                                            const float* const* gls, const float* const* g, const float* c,
                                            float sm_scale, uint16_t* dq, uint16_t* dk, uint16_t* dv,
                                            float* const* dgls, float* const* dscore, float* const* dg, float* dc,
                                            void* ws, size_t ws_bytes, tg_stream_t stream) {
    NvtxRange nvtx_range("tg_gated_attention_backward_gates");
    TG_SUPPORT(n_gates >= 1 && n_gates <= tg::kMaxGates, "n_gates=%d must be in [1, %d]", n_gates, tg::kMaxGates);
    TG_REQUIRE(gls && g && dgls && dg, "null gate arrays");
    tg::GateSet gates{};
    gates.n = n_gates;
    for (int i = 0; i < n_gates; ++i) {
        gates.gls[i] = gls[i];
        gates.g[i] = g[i];
    }
    return do_backward(q, k, v, out, dout, lse, cu_kept, B, M_total, max_M, Hq, Hkv, d, pos, rank, gates, c,
                       sm_scale, dq, dk, dv, dgls, dscore, dg, dc, ws, ws_bytes, stream);
}

tg_status tg_next_gate_span(const int32_t* h_span, const int32_t* h_k, int B, int32_t* h_span_next) {
    TG_REQUIRE(B >= 0, "negative B");
    if (B == 0) return TG_OK;
    TG_REQUIRE(h_span && h_k && h_span_next, "null pointer argument");
    for (int b = 0; b < B; ++b) {
        const int64_t p0 = h_span[2 * b], p1 = h_span[2 * b + 1];
        TG_REQUIRE(p0 >= 0 && p1 >= p0, "sequence %d: span [%lld, %lld)", b, (long long)p0, (long long)p1);
        const int64_t P = p1 - p0;
        const int64_t kk = (h_k[b] < 0 || h_k[b] > P) ? P : h_k[b];
        // every token before the span is kept, so the kept part of the span starts at p0
        // in kept order and holds the kk survivors
        h_span_next[2 * b] = static_cast<int32_t>(p0);
        h_span_next[2 * b + 1] = static_cast<int32_t>(p0 + kk);
    }
    return TG_OK;
}

tg_status tg_device_status(int32_t* h_word, int clear, tg_stream_t stream) {
    if (tg_status s = check_device()) return s;
    int32_t w = 0;
    if (tg_status s = cuda_status(tg::read_device_status(&w, clear != 0, stream), "tg_device_status")) return s;
    if (h_word) *h_word = w;
    if (w & tg::TG_DEVICE_TIMEOUT) return fail(TG_ERR_TIMEOUT, "a bounded device wait gave up (status word 0x%x)", w);
    if (w & tg::TG_DEVICE_BAD_INDEX)
        return fail(TG_ERR_INVALID_ARG, "a kernel found an input-derived index outside its array (status word 0x%x)",
                    w);
    return TG_OK;
}

tg_status tg_selftest_bounded_wait(int64_t timeout_ns, tg_stream_t stream) {
    TG_REQUIRE(timeout_ns > 0 && timeout_ns <= 10000000000LL, "timeout_ns must be in (0, 10 s]");
    if (tg_status s = check_device()) return s;
    return cuda_status(tg::launch_selftest_wait(timeout_ns, stream), "tg_selftest_bounded_wait launch");
}

tg_status tg_selftest_exp2(const float* x, float* y, int64_t n, tg_stream_t stream) {
    TG_REQUIRE(n >= 0, "negative n");
    if (n == 0) return TG_OK;
    TG_REQUIRE(x && y, "null pointer argument");
    if (tg_status s = check_device()) return s;
    return cuda_status(tg::launch_exp2_poly_selftest(x, y, n, stream), "tg_selftest_exp2 launch");
}

tg_status tg_gated_prefill_layer(const tg_prefill_layer_args* a, tg_stream_t stream) {
    NvtxRange nvtx_range("tg_gated_prefill_layer");
    TG_REQUIRE(a != nullptr, "null args");
    TG_REQUIRE(a->B >= 0 && a->T >= 0 && a->M_total >= 0 && a->M_total <= a->T && a->n_layers >= 0, "bad sizes");
    if (tg_status s = check_gate_shape(a->D, a->I)) return s;
    if (a->n_layers > 0) {
        if (tg_status s = check_attn_shape(a->Hq, a->Hkv, a->d)) return s;
        TG_REQUIRE(a->q && a->kk && a->v && a->g && a->c && a->out, "null per-layer array");
        for (int l = 0; l < a->n_layers; ++l)
            TG_REQUIRE(a->q[l] && a->kk[l] && a->v[l] && a->g[l] && a->c[l] && a->out[l],
                       "null tensor in layer %d", l);
    }
    if (a->B == 0 || a->T == 0) return TG_OK;
    TG_REQUIRE(a->hidden && a->cu_seqlens && a->span && a->k && a->Wg && a->b1 && a->w2 && a->cu_kept && a->scores &&
                   a->keep,
               "null pointer argument");
    TG_REQUIRE(a->M_total == 0 || (a->pos && a->rank && a->gls && a->kept_idx), "null compaction output");
    TG_REQUIRE(aligned16(a->hidden) && aligned16(a->Wg), "hidden and Wg must be 16-byte aligned");
    if (a->hidden_kept) TG_REQUIRE(aligned16(a->hidden_kept), "hidden_kept must be 16-byte aligned");
    TG_REQUIRE(a->n_gather >= 0, "negative n_gather");
    if (a->n_gather > 0) {
        TG_REQUIRE(a->gather_src && a->gather_dst && a->gather_row_bytes, "null gather arrays");
        for (int i = 0; i < a->n_gather; ++i) {
            TG_REQUIRE(a->gather_src[i] && a->gather_dst[i], "null gather tensor %d", i);
            TG_SUPPORT(a->gather_row_bytes[i] > 0 && a->gather_row_bytes[i] % 16 == 0,
                       "gather %d: row_bytes=%lld must be a positive multiple of 16", i,
                       (long long)a->gather_row_bytes[i]);
            TG_REQUIRE(aligned16(a->gather_src[i]) && aligned16(a->gather_dst[i]),
                       "gather %d: tensors must be 16-byte aligned", i);
        }
    }
    TG_REQUIRE(a->eps >= 0.f, "eps must be >= 0");
    if (a->attn_ws) TG_REQUIRE((reinterpret_cast<uintptr_t>(a->attn_ws) & 255u) == 0, "attn_ws must be 256-byte aligned");
    if (tg_status s = check_device()) return s;
    cudaStream_t st = stream;
    // A workspace of tg_gated_prefill_workspace_size bytes also holds the selection's
    // first-pass histogram, which the score kernel then fills (the selection skips that pass).
    int* key_hist = nullptr;
    {
        const size_t off = prefill_key_hist_offset(a->B, a->max_M, a->Hq, a->Hkv, a->d, a->n_layers);
        if (a->attn_ws && a->attn_ws_bytes >= off + prefill_key_hist_bytes(a->B))
            key_hist = reinterpret_cast<int*>(static_cast<uint8_t*>(a->attn_ws) + off);
    }
    if (tg_status s = cuda_status(tg::launch_score(a->hidden, a->cu_seqlens, a->span, a->B, a->T, a->D, a->Wg, a->b1,
                                                   a->w2, a->b2, a->I, a->eps, a->scores, st, key_hist),
                                  "score launch"))
        return s;
    if (tg_status s = cuda_status(tg::launch_select_scan(0, a->scores, nullptr, a->cu_seqlens, a->span, a->k,
                                                         a->cu_kept, a->B, a->T, a->keep, a->kept_idx, a->pos, a->rank,
                                                         a->gls, st, key_hist, true),
                                  "select launch"))
        return s;
    if (a->M_total == 0) return TG_OK;  // every token pruned: no kept rows, no attention
    // One stream, kernels chained by programmatic dependent launch:
    //   score -> select -> attention x n_layers -> row gathers.
    // Each attention layer loads its Q/K/V while its predecessor runs (they are the
    // caller's, complete before this call) and releases its dependents only once the
    // selection has completed; the row gathers (HBM-bound) therefore start during the last
    // attention layer's final wave and read the compaction map at once, waiting for the
    // attention only before they exit, so that the call's last kernel completes after all
    // of its work.
    tg_status result = TG_OK;
    for (int l = 0; l < a->n_layers && result == TG_OK; ++l) {
        float* lse = a->lse ? a->lse[l] : nullptr;
        result = do_attention(a->q[l], a->kk[l], a->v[l], a->cu_kept, a->B, a->M_total, a->max_M, a->Hq, a->Hkv,
                              a->d, a->pos, a->rank, tg::single_gate(a->gls, a->g[l]), a->c[l], a->sm_scale,
                              a->out[l], lse, a->attn_ws, a->attn_ws_bytes, st, true);
    }
    if (result != TG_OK) return result;
    const bool after_attention = a->n_layers > 0;
    if (a->hidden_kept) {
        if (tg_status s = cuda_status(tg::launch_gather_rows(a->hidden, a->kept_idx, a->M_total, a->T, a->D,
                                                             a->hidden_kept, st, after_attention),
                                      "gather launch"))
            return s;
    }
    for (int i = 0; i < a->n_gather; ++i) {
        if (tg_status s = cuda_status(tg::launch_gather_bytes(a->gather_src[i], a->kept_idx, a->M_total, a->T,
                                                              a->gather_row_bytes[i], a->gather_dst[i], st,
                                                              after_attention),
                                      "extra gather launch"))
            return s;
    }
    return result;
}

}  // extern "C"
