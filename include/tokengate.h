/*
 * tokengate.h -- C ABI of libtokengate.so, the B200 (sm_100a) implementation
 * of TokenGate's gated-prefill hot path.
 *
 * The method (TokenGate: Adapting LLMs for Fast and Memory-Efficient Prefill
 * with Learned Token Pruning; AI summary page, "Key Contributions" 1-3 and
 * "Methodology in Plain English"; README copy, "How it works"):
 *   1. at gate layer L, score every prunable token with RMSNorm followed by
 *      a small MLP over its post-attention residual          -> tg_score
 *   2. keep the K best prunable tokens plus every non-prunable one
 *                                                           -> tg_select_topk
 *   3. hand only the kept tokens, in order, to the layers above -> tg_compact
 *   4. token-gated attention in those layers: causal GQA attention over the
 *      kept tokens with a per-key, per-head gate bias and a per-query
 *      temperature                                      -> tg_gated_attention
 *   tg_gated_prefill_layer chains 1-4 on one stream.
 *
 * The pages describe the bias and the temperature only in prose ("a per-key
 * gate bias", "a learnable per-layer, per-head gain passed through softplus",
 * "a temperature scaled by the log-ratio of a query's original position to
 * its rank among kept tokens").  This library defines them as
 *     b[h,j]   = softplus(g_h) * logsigmoid(s_j)      (0 for non-prunable j)
 *     tau[q,h] = 1 + c_h * ln(pos_q / rank_q)
 *     logit    = (q.k_j * sm_scale + b[h,j]) / tau[q,h]
 * with g_h, c_h caller inputs (one per query head and layer).
 *
 * Conventions shared by every entry point
 *   - Tensors are DEVICE pointers owned by the caller; the library never
 *     allocates, frees or keeps them.  Host pointers are marked h_.
 *   - bf16 tensors are passed as uint16_t bit patterns; all layouts are
 *     row-major and densely packed.
 *   - Sequences use the varlen layout: B sequences concatenated into T
 *     tokens, cu_seqlens[B+1] (int32, device) the prefix sums of the lengths.
 *     span[2*b], span[2*b+1] (int32, device) is sequence b's prunable span
 *     [p0, p1) in sequence-local token indices (the `{state}` document).
 *     k[b] (int32, device) is the keep budget; k < 0 keeps every prunable
 *     token, k >= |P_b| too, k == 0 keeps only the non-prunable tokens.
 *   - The kept count of sequence b is M_b = (N_b - |P_b|) + min(K_b, |P_b|);
 *     it depends on no score, so the caller sizes every output on the host
 *     with tg_kept_count and passes cu_kept (device copy) back in.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Arguments are validated on the host before anything
 *     is launched; a rejected call launches nothing and returns
 *     TG_ERR_INVALID_ARG or TG_ERR_UNSUPPORTED.  TG_ERR_CUDA reports a launch
 *     error.  No exception crosses the ABI.  tg_last_error_string() describes
 *     the last failure of the calling thread.
 *   - Supported shapes: D a multiple of 64 (<= 8192); I a multiple of 16 in
 *     [16, 256]; head_dim 64, 128 or 256; Hq a multiple of Hkv; sm_100 devices.
 */
#ifndef TOKENGATE_H
#define TOKENGATE_H

#include <stddef.h>
#include <stdint.h>

/* The library is built with hidden visibility; every declaration below is
   its exported interface. */
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* tg_stream_t; /* the same type as cudaStream_t */

typedef enum tg_status {
    TG_OK = 0,
    TG_ERR_INVALID_ARG = 1, /* null pointer, bad size, inconsistent shapes */
    TG_ERR_UNSUPPORTED = 2, /* shape or device outside the supported set */
    TG_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    TG_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up (see tg_device_status) */
} tg_status;

/* Version of this ABI (incremented on any signature change). */
int tg_abi_version(void);

/* Message for the last non-OK status returned on the calling thread. */
const char* tg_last_error_string(void);

/*
 * Kept-token count (host only, no device work).
 * TokenGate README copy, "Quick start": every token outside `{state}` is
 * kept, plus max_kept_prefill_tokens=K of the state tokens (None = all).
 * h_cu_seqlens[B+1], h_span[2B], h_k[B] are host arrays; h_cu_kept[B+1]
 * (host, caller-owned) receives the prefix sums of M_b.  Returns the total
 * M = sum_b M_b, or -1 on invalid input (see tg_last_error_string).
 */
int64_t tg_kept_count(const int32_t* h_cu_seqlens, const int32_t* h_span, const int32_t* h_k, int B,
                      int32_t* h_cu_kept);

/*
 * Gate weight preparation (once per gate, not on the per-request path).
 * The RMSNorm weight gamma [D] is folded into the first gate layer
 * W1 [D, I]:  Wg[j*D + i] = bf16_rne(gamma[i] * W1[i*I + j])  ->  Wg [I, D].
 * The product of two bf16 numbers is exact in fp32, so the one rounding is
 * the final round-to-nearest-even.  RMSNorm's 1/rms factor is applied after
 * the contraction inside tg_score (AI summary, "Key Contributions" 1: MLP
 * over the RMSNorm-normalised residual).
 */
tg_status tg_gate_prepare(const uint16_t* gamma, const uint16_t* W1, int D, int I, uint16_t* Wg,
                          tg_stream_t stream);

/*
 * Stage 1: gate score of every prunable token (AI summary, "Key
 * Contributions" 1; TokenGate explained blog, "how the gate works").
 *   r_t = 1 / sqrt(mean_i x_ti^2 + eps)
 *   s_t = b2 + sum_j w2[j] * SiLU(r_t * (Wg[j,:] . x_t) + b1[j])
 * hidden [T, D] bf16; Wg [I, D] bf16 from tg_gate_prepare; b1 [I], w2 [I]
 * fp32; scores [T] fp32 (out).  Only prunable entries are written; the
 * others keep their previous contents.  The contraction runs on the tensor
 * cores in fp32 accumulation over the exact bf16 inputs.
 */
tg_status tg_score(const uint16_t* hidden, const int32_t* cu_seqlens, const int32_t* span, int B, int64_t T,
                   int D, const uint16_t* Wg, const float* b1, const float* w2, float b2, int I, float eps,
                   float* scores, tg_stream_t stream);

/*
 * Stage 2: deterministic top-K per sequence over the prunable span (AI
 * summary, "Key Contributions" 1 and "Methodology in Plain English").
 * Order: higher score first, equal scores by lower token index; -0 equals
 * +0; NaN ranks below every number.  keep [T] uint8 (out): 1 for every
 * non-prunable token and for the selected prunable ones, else 0.
 * Bit-exact and run-to-run deterministic.
 * Optional fused compaction map: when cu_kept and kept_idx are both
 * non-NULL, the same pass also writes kept_idx, pos, rank and gls exactly as
 * tg_compact defines them (pos, rank, gls must then be non-NULL too), so
 * that tg_compact(keep = NULL) only has to gather the rows.  Pass NULL for
 * all five to get the flags alone.
 */
tg_status tg_select_topk(const float* scores, const int32_t* cu_seqlens, const int32_t* span, const int32_t* k,
                         int B, int64_t T, uint8_t* keep, const int32_t* cu_kept, int32_t* kept_idx, int32_t* pos,
                         int32_t* rank, float* gls, tg_stream_t stream);

/*
 * Stage 3: stable compaction of the kept tokens (AI summary, "Key
 * Contributions" 1: the layers above L see only kept tokens and create no
 * KV entries for pruned ones).  For the m-th kept token t of sequence b
 * (m counted over the whole batch, in original order):
 *   hidden_kept[m, :] = hidden[t, :]          (bytes copied unchanged)
 *   pos[m]      = t - cu_seqlens[b] + 1       (1-indexed original position)
 *   rank[m]     = m - cu_kept[b] + 1          (1-indexed rank among kept)
 *   gls[m]      = logsigmoid(scores[t]) if t is prunable, else 0
 *   kept_idx[m] = t                           (source row; the gather map)
 * cu_kept [B+1] (device) must hold tg_kept_count's prefix sums; M_total is
 * cu_kept[B].  hidden_kept may be NULL (then only the index outputs are
 * written); pos, rank, gls, kept_idx are required.
 * keep == NULL means the compaction map was already written by
 * tg_select_topk: kept_idx is then an input and only the row gather runs
 * (scores, pos, rank, gls are not touched and may be NULL).
 * Keep flags that disagree with cu_kept never make the kernels write or
 * read outside [0, M_total) and [0, T); the affected rows are unspecified.
 */
tg_status tg_compact(const uint16_t* hidden, const float* scores, const uint8_t* keep, const int32_t* cu_seqlens,
                     const int32_t* span, int B, int64_t T, int D, const int32_t* cu_kept, int64_t M_total,
                     uint16_t* hidden_kept, int32_t* pos, int32_t* rank, float* gls, int32_t* kept_idx,
                     tg_stream_t stream);

/*
 * Stage 4: token-gated causal GQA attention over the kept tokens, one upper
 * layer (AI summary, "Key Contributions" 2 and 3; the definitions of b and
 * tau are at the top of this file).
 * q [M, Hq, d], k/v [M, Hkv, d] bf16 (M = cu_kept[B]); pos, rank [M] int32
 * and gls [M] fp32 from tg_compact; g, c [Hq] fp32; out [M, Hq, d] bf16.
 * Query i of sequence b attends to the kept keys j of b with j <= i (that
 * is rank_j <= rank_i); query head h reads KV head h / (Hq / Hkv).
 * lse [M, Hq] fp32 (optional, may be NULL): natural-log softmax
 * normaliser of each (query, head) row.  max_M is an upper bound of the
 * longest sequence's M_b (grid sizing).  sm_scale is usually 1/sqrt(d).
 * tau must stay positive: c_h >= 0 guarantees it since pos >= rank.
 * Tensor cores: bf16 operands, fp32 accumulation.
 * ws (device, 256-byte aligned, may be NULL) is scratch for the causal work
 * split: when the longest query tile would dominate the launch, long query
 * tiles are cut into two KV chunks whose partial results meet in ws, and the
 * last chunk to finish merges them.  ws_bytes must be at least
 * tg_gated_attention_workspace_size(B, max_M, Hq, Hkv, d).  ws must be
 * zero-filled before its first use; every call leaves it zero-filled again.
 * Calls that share one ws must not run concurrently.  With ws == NULL the
 * attention runs unsplit (same results, less balanced for small M).
 * Kernel choice (even GQA groups, d <= 128, ws given): one CTA per unit of
 * work for a single sequence (B == 1), persistent CTAs that take units from
 * a counter in ws for a batch; the environment variable TG_ATTENTION_KERNEL
 * set to "persistent" or "per_unit" overrides it per call (the two give the
 * same results within rounding; the workspace size may change with it).
 */
tg_status tg_gated_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept,
                             int B, int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                             const int32_t* rank, const float* gls, const float* g, const float* c, float sm_scale,
                             uint16_t* out, float* lse, void* ws, size_t ws_bytes, tg_stream_t stream);

/*
 * Several gate modules (AI summary, "Future Directions": gates at several
 * layers, each selecting from what the lower ones kept and each contributing
 * to the token-gated attention above it).  Same as tg_gated_attention with
 * the bias summed over the gates:
 *     b[h,j] = sum_i softplus(g[i][h]) * gls[i][j],  i < n_gates
 * gls and g are HOST arrays of n_gates DEVICE pointers: gls[i] [M] fp32 is
 * gate i's logsigmoid per kept row (0 for rows that gate could not prune),
 * g[i] [Hq] fp32 its gain parameters for this layer.  pos must hold the
 * ORIGINAL 1-indexed positions and rank the rank among the tokens finally
 * kept (compose them with tg_gather_rows over the later gates' kept_idx).
 * 1 <= n_gates <= 4, else TG_ERR_UNSUPPORTED; n_gates = 1 is
 * tg_gated_attention.  The gates ride in the same extra k-step of the
 * tensor-core product that carries one gate's bias, so more gates cost no
 * softmax work.
 */
tg_status tg_gated_attention_gates(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept,
                                   int B, int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                                   const int32_t* rank, int n_gates, const float* const* gls, const float* const* g,
                                   const float* c, float sm_scale, uint16_t* out, float* lse, void* ws,
                                   size_t ws_bytes, tg_stream_t stream);

/*
 * Backward of tg_gated_attention (one gate): the gradient path that makes the
 * gate trainable (AI summary, "Key Contributions" 2: the bias on the logits
 * carries the task loss's gradient back to the scoring network; 3: the gain
 * and temperature are learned; 4: training runs this attention at full budget
 * and at a sampled budget).  With l_ij = (sm q_i.k_j + softplus(g_h) gls_j) /
 * tau_ih and P = softmax(l), for the upstream gradient dout [M, Hq, d] bf16:
 *   dq [M, Hq, d], dk / dv [M, Hkv, d] bf16 (GQA: dk, dv summed over the
 *   query heads of each KV head);
 *   dgls [M] fp32 = d loss / d gls_j (summed over heads);
 *   dscore [M] fp32 (may be NULL) = dgls_j * sigmoid(-score_j), computed as
 *   dgls_j * (1 - exp(gls_j)): the gradient reaching the gate's score of kept
 *   row j (0 for rows the gate cannot prune, whose gls is 0);
 *   dg, dc [Hq] fp32 = gradients of the gain and temperature parameters.
 * q, k, v, pos, rank, gls, g, c, cu_kept, sm_scale as passed to the forward;
 * out [M, Hq, d] bf16 and lse [M, Hq] fp32 are the forward's outputs (call
 * tg_gated_attention with a non-NULL lse).  head_dim 64, 128 or 256.
 * ws: device scratch, 256-byte aligned, of at least
 * tg_gated_attention_backward_workspace_size(M_total, Hq, Hkv, d) bytes (6
 * floats per row and head, plus fp32 partial dk and dv per query head when a
 * KV head serves 3, 5, 6, 7 or more than 8 query heads, or any group of two
 * or more at head_dim 256; groups of 2, 4 and 8 at head_dim 64 and 128 add
 * theirs inside a thread-block cluster; no zeroing needed).  At head_dim 256
 * dv and dk are accumulated by two launches over the same keys (the two fp32
 * accumulators would not fit tensor memory together).  Tensor cores, no
 * atomics: the results are deterministic.
 */
size_t tg_gated_attention_backward_workspace_size(int64_t M_total, int Hq, int Hkv, int d);
tg_status tg_gated_attention_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* out,
                                      const uint16_t* dout, const float* lse, const int32_t* cu_kept, int B,
                                      int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                                      const int32_t* rank, const float* gls, const float* g, const float* c,
                                      float sm_scale, uint16_t* dq, uint16_t* dk, uint16_t* dv, float* dgls,
                                      float* dscore, float* dg, float* dc, void* ws, size_t ws_bytes,
                                      tg_stream_t stream);

/*
 * Backward of tg_gated_attention_gates: several gate modules (AI summary,
 * "Future Directions"), the logits carrying sum_i softplus(g[i][h]) gls[i][j].
 * Same arguments and outputs as tg_gated_attention_backward, with per-gate
 * HOST arrays of DEVICE pointers: gls[i] [M] and g[i] [Hq] in; dgls[i] [M]
 * (d loss / d gls_i) and dg[i] [Hq] out; dscore (may be NULL, as may any of
 * its entries) gets dscore[i][j] = dgls[i][j] * (1 - exp(gls[i][j])).
 * 1 <= n_gates <= 4, else TG_ERR_UNSUPPORTED; n_gates = 1 is
 * tg_gated_attention_backward.  Same workspace size.
 */
tg_status tg_gated_attention_backward_gates(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                            const uint16_t* out, const uint16_t* dout, const float* lse,
                                            const int32_t* cu_kept, int B, int64_t M_total, int max_M, int Hq,
                                            int Hkv, int d, const int32_t* pos, const int32_t* rank, int n_gates,
                                            const float* const* gls, const float* const* g, const float* c,
                                            float sm_scale, uint16_t* dq, uint16_t* dk, uint16_t* dv,
                                            float* const* dgls, float* const* dscore, float* const* dg, float* dc,
                                            void* ws, size_t ws_bytes, tg_stream_t stream);

/*
 * Host only: the prunable span of the NEXT gate, in the kept order of this
 * one.  All tokens before a span are kept, so sequence b's surviving span
 * tokens sit at kept indices [p0_b, p0_b + min(k_b, |P_b|)) (k_b < 0 = all).
 * h_span and h_span_next are [B, 2] int32 (may alias); h_k is [B].  With
 * cu_kept as the next gate's cu_seqlens, tg_score / tg_select_topk /
 * tg_compact run the next gate unchanged.  Returns TG_ERR_INVALID_ARG for a
 * negative or reversed span.
 */
tg_status tg_next_gate_span(const int32_t* h_span, const int32_t* h_k, int B, int32_t* h_span_next);

/* Bytes of scratch tg_gated_attention may use for these sizes on the
 * current device (0 when it does not split, or for unsupported sizes). */
size_t tg_gated_attention_workspace_size(int B, int max_M, int Hq, int Hkv, int d);

/*
 * tg_gated_attention without a caller workspace: no allocation at all.
 * (The pages describe no such entry point; it exists for callers that
 * cannot allocate device memory where they run the attention, such as a
 * serving engine that reserves all of HBM at start-up and only hands out
 * fixed buffers, or code inside a host runtime that owns the allocator.)
 * Same arguments, semantics and results as tg_gated_attention; the scratch
 * of the causal split is a fixed array of TG_NOALLOC_ATTENTION_SCRATCH_BYTES
 * in the library's device image, which every GPU that loads the library
 * keeps until the process exits.  Sizes whose split would need more
 * (tg_gated_attention_workspace_size above the limit) are rejected with
 * TG_ERR_UNSUPPORTED and nothing is launched.  The call allocates nothing
 * (no cudaMalloc, cudaFree or allocating library routine); it clears the
 * array's arrival counters with cudaMemsetAsync on `stream`.  All calls on
 * a device share the array and it keeps the last call's contents: calls
 * whose executions overlap on the GPU (other streams, other threads) race on
 * it and must be serialised by the caller.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress); make that
 * first call before any stream capture.
 */
#define TG_NOALLOC_ATTENTION_SCRATCH_BYTES (32u * 1024u * 1024u)
tg_status tg_gated_attention_noalloc(const uint16_t* q, const uint16_t* k, const uint16_t* v, const int32_t* cu_kept,
                                     int B, int64_t M_total, int max_M, int Hq, int Hkv, int d, const int32_t* pos,
                                     const int32_t* rank, const float* gls, const float* g, const float* c,
                                     float sm_scale, uint16_t* out, float* lse, tg_stream_t stream);

/*
 * The whole gated prefill at one gate layer (AI summary, "Methodology in
 * Plain English": the layers below the gate run on every token, the gate
 * scores and keeps the top-K at layer L, and the layers above run on the kept
 * tokens only; README copy, "How it works"): tg_score, tg_select_topk (which
 * also writes the compaction map), the row gather of tg_compact and n_layers
 * gated-attention layers above the gate, with no host synchronisation, all
 * on `stream`.  The kernels are chained by programmatic dependent launch:
 * each attention layer loads its q/k/v while the kernel before it runs, and
 * the row gathers run last, overlapping the final attention wave.  This
 * relies on q, k, v, g, c, hidden and cu_kept being complete before the call
 * (written by work enqueued on `stream` earlier, or already synchronised),
 * and on no other stream writing them while the call runs.  Everything the
 * call enqueues is ordered before work enqueued on `stream` afterwards, and
 * the call may be captured into a CUDA graph.  Fields mirror
 * the stage arguments above; per-layer tensors are arrays of n_layers
 * device pointers (the array itself lives in host memory).  The
 * projections that turn hidden_kept into each layer's q/k/v belong to the
 * model, not to this method, so q/k/v are inputs sized [M, ...].
 */
typedef struct tg_prefill_layer_args {
    /* stage 1-3 */
    const uint16_t* hidden;     /* [T, D] */
    const int32_t* cu_seqlens;  /* [B+1] device */
    const int32_t* span;        /* [2B] device */
    const int32_t* k;           /* [B] device */
    int B;
    int64_t T;
    int D;
    const uint16_t* Wg;         /* [I, D] */
    const float* b1;            /* [I] */
    const float* w2;            /* [I] */
    float b2;
    int I;
    float eps;
    const int32_t* cu_kept;     /* [B+1] device, from tg_kept_count */
    int64_t M_total;
    int max_M;
    float* scores;              /* [T] out */
    uint8_t* keep;              /* [T] out */
    uint16_t* hidden_kept;      /* [M, D] out, may be NULL */
    int32_t* pos;               /* [M] out */
    int32_t* rank;              /* [M] out */
    float* gls;                 /* [M] out */
    int32_t* kept_idx;          /* [M] out */
    /* stage 4, n_layers times */
    int n_layers;
    int Hq, Hkv, d;
    float sm_scale;
    const uint16_t* const* q;   /* n_layers x [M, Hq, d] */
    const uint16_t* const* kk;  /* n_layers x [M, Hkv, d] */
    const uint16_t* const* v;   /* n_layers x [M, Hkv, d] */
    const float* const* g;      /* n_layers x [Hq] */
    const float* const* c;      /* n_layers x [Hq] */
    uint16_t* const* out;       /* n_layers x [M, Hq, d] out */
    float* const* lse;          /* n_layers x [M, Hq] out, array or entries may be NULL */
    void* attn_ws;              /* scratch shared by the layers (may be NULL): see below */
    size_t attn_ws_bytes;
    /* optional: more row-major arrays gathered by the same map beside the attention, e.g. the
       KV cache of the layers below L (see tg_gather_rows); n_gather = 0 for none */
    int n_gather;
    const void* const* gather_src;    /* n_gather x [T, row_bytes] */
    void* const* gather_dst;          /* n_gather x [M, row_bytes] out */
    const int64_t* gather_row_bytes;  /* n_gather, host */
} tg_prefill_layer_args;

tg_status tg_gated_prefill_layer(const tg_prefill_layer_args* args, tg_stream_t stream);

/*
 * Bytes of args->attn_ws with which tg_gated_prefill_layer also runs the
 * selection's first bucket pass inside the score kernel: after the attention's
 * scratch (tg_gated_attention_workspace_size, rounded up to 256 bytes) the
 * workspace holds a [B][2048] int32 histogram of the top 11 bits of every
 * scored row's order-preserving key, which the score kernel fills with atomic
 * adds and the selection reads (saving a pass over the keys and a cluster
 * round trip) and zeroes again.  The same zero-on-entry contract as the
 * attention's scratch holds: zero-fill attn_ws before its first use; every
 * call leaves it zero-filled.  A smaller attn_ws (at least the attention's
 * size) runs every pass in the selection; results are identical.
 * n_layers = 0: the histogram alone.  Returns 0 for B <= 0.
 */
size_t tg_gated_prefill_workspace_size(int B, int max_M, int Hq, int Hkv, int d, int n_layers);

/*
 * Full-length (training-time) token-gated attention for a sampled budget.
 * The pages train with one full-budget forward and one forward at a smaller
 * budget drawn per step (AI summary, "Methodology in Plain English"); in the
 * full-length form of the smaller-budget pass the pruned keys are masked out
 * of every query's softmax (bias -inf) and the rows of pruned queries are
 * not computed.  This library defines, for q, k, v of full length
 * ([T, Hq, d], [T, Hkv, d], [T, Hkv, d] bf16) and the budgets kbud[B]:
 *   keep = tg_select_topk(scores, cu_seqlens, span, kbud)
 *   out[t] = 0 for every pruned t; for kept t it is the gated attention of
 *   tg_gated_attention over the kept keys j <= t of t's sequence, with
 *   pos/rank/gls from the compaction of `keep`
 * (the same numbers as compacting, attending and scattering back, which is
 * also how it runs: select, gather of the kept rows, the compacted kernel,
 * scatter; every fully masked key tile is skipped).  cu_kept / M_total /
 * max_M come from tg_kept_count(cu_seqlens, span, kbud) on the host.
 * keep_out ([T] u8) receives the flags when non-NULL.  ws (256-byte aligned,
 * zeroed once before first use; the calls leave it reusable) holds
 * tg_masked_gated_attention_workspace_size(B, T, M_total, max_M, Hq, Hkv, d)
 * bytes.  sm_scale as in tg_gated_attention.
 */
size_t tg_masked_gated_attention_workspace_size(int B, int64_t T, int64_t M_total, int max_M, int Hq, int Hkv, int d);
tg_status tg_masked_gated_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* scores,
                                    const int32_t* cu_seqlens, const int32_t* span, const int32_t* kbud,
                                    const int32_t* cu_kept, int B, int64_t T, int64_t M_total, int max_M, int Hq,
                                    int Hkv, int d, const float* g, const float* c, float sm_scale, uint16_t* out,
                                    uint8_t* keep_out, void* ws, size_t ws_bytes, tg_stream_t stream);

/*
 * Row gather by the compaction map: dst[m, :] = src[kept_idx[m], :] for
 * m < M, rows of row_bytes bytes (4, 8 or a multiple of 16; src and dst
 * aligned to min(row_bytes, 16) bytes, device; anything else is
 * TG_ERR_UNSUPPORTED or TG_ERR_INVALID_ARG before any launch).  The serving path of the pages gathers the lower
 * layers' KV cache to the kept tokens on a separate stream (AI summary,
 * "Methodology in Plain English"): with src the [T, Hkv, d] K or V cache of
 * a layer below L (row_bytes = 2 * Hkv * d for bf16) this is that gather.
 * Entries of kept_idx outside [0, T) leave their row unwritten.  src
 * ([T, row_bytes]) and dst ([M, row_bytes]) must not overlap: an in-place or
 * overlapping call is refused with TG_ERR_INVALID_ARG.
 * tg_gated_prefill_layer runs the same gather for args->gather_* beside the
 * attention.  With 4-byte rows it composes the maps of two gates: the
 * original positions of the tokens the second gate keeps are
 * pos1[kept_idx2], their first-gate logsigmoids gls1[kept_idx2].
 */
tg_status tg_gather_rows(const void* src, int64_t T, int64_t row_bytes, const int32_t* kept_idx, int64_t M,
                         void* dst, tg_stream_t stream);

/*
 * Device status word (failure detection).  Every wait inside the kernels
 * (on an mbarrier fed by TMA, by the tensor core or by other warps) is
 * bounded: after 2 s the waiting thread raises its CTA's abort flag, ORs
 * 0x10000 | <where> into the status word of the current device (where: 1 TMA
 * producer, 2 MMA issuer, 4 softmax/epilogue warps, 8 draining after an
 * abort), every role leaves its loop, copies in flight are awaited (again
 * bounded), TMEM is freed and the kernel returns, leaving the context
 * usable.  The outputs of such a call are unspecified.
 * tg_device_status synchronises `stream`, copies the word to *h_word (may be
 * NULL), clears it when `clear` is non-zero, and returns TG_ERR_TIMEOUT when
 * a timeout was recorded, else TG_OK.
 */
tg_status tg_device_status(int32_t* h_word, int clear, tg_stream_t stream);

/*
 * Diagnostic: one CTA waits on an mbarrier that nothing ever completes, with
 * the kernels' bounded-wait routine and a limit of timeout_ns (0 < t <= 10 s).
 * The wait gives up, records a timeout in the status word and the kernel
 * returns: no fault and no hang.  Used to test the failure path above.
 */
tg_status tg_selftest_bounded_wait(int64_t timeout_ns, tg_stream_t stream);

/*
 * Diagnostic: y[i] = 2^x[i] computed by the attention softmax's FMA-pipe
 * exponential (the share of the softmax's exponentials that does not go to
 * the special-function unit): Cody-Waite range reduction to f in [-0.5, 0.5]
 * and a degree-3 polynomial fitted for this library (relative error at most
 * 7.5e-5 for -125 <= x <= 0; x below -125 is clamped to -125).  x, y are
 * device arrays of n floats.  Used to test that exponential against exp2.
 */
tg_status tg_selftest_exp2(const float* x, float* y, int64_t n, tg_stream_t stream);

#ifdef __cplusplus
}
#endif

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#endif /* TOKENGATE_H */
