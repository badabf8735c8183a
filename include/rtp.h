/*
 * rtp.h -- C ABI of librtp.so: the RTPurbo sparse-attention layer on NVIDIA B200
 * (sm_100a).
 *
 * One attention layer with two kinds of heads (paper-graph-ui summary of
 * "Full Attention Strikes Back: Transferring Full Attention into Sparse within
 * Hundred Training Steps", arXiv 2605.16928, cited as [FASB §section]):
 *
 *  - retrieval heads keep the full KV cache.  A 16-dim indexer scores every
 *    causal key, s(m, n) = (W^Q q_m) . (W^K k_n)   [FASB §Low-Dimensional
 *    Projection Mechanism]; the keys are softmax-normalised on those scores and
 *    the smallest highest-scoring set whose mass reaches p is kept, ties to the
 *    lower index   [FASB §Dynamic Top-p Selection Mechanism, Eq. 5]; exact
 *    attention then runs over the kept K/V rows only (same section);
 *  - local heads attend to n_sink attention-sink tokens plus a sliding window
 *    [FASB §Local Head Attention Pattern].
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or synchronises with the host.  Every call is
 *    asynchronous on `stream` (0 = legacy default stream).
 *  - bf16 tensors are passed as void* to bf16 data (IEEE bfloat16 bits).
 *  - A strided view `rtp_view` describes a [B][L][heads][width] tensor whose
 *    (heads x width) block per row is contiguous; stride_b / stride_l are in
 *    ELEMENTS.  The base pointer and both strides must keep every row 16-byte
 *    aligned (else RTP_ERR_ALIGNMENT).
 *  - Head dimension D must be 128; indexer width is 16.
 *  - Query heads h = 0..H-1 map to kv head g = h / (H / Hkv) (GQA).
 *    kv_role (HOST array of Hkv bytes): 1 = retrieval kv head, 0 = local.  The
 *    retrieval query heads are the query heads of retrieval kv heads, numbered
 *    in increasing h as retrieval slots hr = 0..H_ret-1; q16, Wq16 and the
 *    per-row selection outputs are indexed by hr.
 *  - k16 layout: k16_per_kv_head = 0 gives one indexer key per retrieval
 *    QUERY head (H_k16 = H_ret, slot hr uses Wk16[hr]; the summary gives every
 *    retrieval head its own W^K); k16_per_kv_head = 1 gives one per retrieval
 *    KV head (H_k16 = number of retrieval kv heads, slot = rank of the kv head
 *    among retrieval kv heads, shared by its query heads).
 *  - Query row i of batch b sits at absolute position P = q_pos0 + i and sees
 *    keys 0..P (causal, the query's own key included); P must be < Lk.
 *  - Outputs of retrieval calls touch only retrieval heads of `o`, local calls
 *    only local heads, so one `o` buffer can receive both.
 *  - Arguments are validated on the host before anything is launched; an error
 *    return means nothing was enqueued.  Launch failures return RTP_ERR_CUDA.
 *  - Workspace: `ws` is caller-owned device memory of at least
 *    rtp_workspace_size(op, ...) bytes, 256-byte aligned.  Zero it once before
 *    first use (rtp_workspace_init) so the device status word starts clear; each
 *    call resets whatever it accumulates into, so one workspace may serve calls
 *    of any shape in turn.  Concurrent calls must not share a workspace.  The
 *    first 256 bytes of every workspace hold a device status word that kernels
 *    set when an internal consistency check fails; rtp_get_device_status reads
 *    it.
 */
#ifndef RTP_H_
#define RTP_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RTP_API __attribute__((visibility("default")))
#else
#define RTP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* rtp_stream_t; /* == cudaStream_t */

typedef enum rtp_status {
    RTP_OK = 0,
    RTP_ERR_INVALID_ARG = 1,         /* bad shape, null pointer, p outside [0,1], ... */
    RTP_ERR_UNSUPPORTED = 2,         /* D != 128, too many heads, device not sm_100 */
    RTP_ERR_ALIGNMENT = 3,           /* a pointer or stride breaks 16-byte row alignment */
    RTP_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes < rtp_workspace_size(...) */
    RTP_ERR_CUDA = 5,                /* a CUDA runtime call or launch failed */
    RTP_ERR_DEVICE_TIMEOUT = 6,      /* a kernel's bounded wait gave up (device status) */
    RTP_ERR_SCRATCH_LIMIT = 7        /* shape needs more than the built-in scratch array */
} rtp_status;

typedef enum rtp_op {
    RTP_OP_INDEX_SCORES = 0,
    RTP_OP_TOPP_SELECT = 1,
    RTP_OP_SPARSE_PREFILL = 2,
    RTP_OP_SPARSE_DECODE = 3,
    RTP_OP_LOCAL = 4,
    RTP_OP_DENSE = 5
} rtp_op;

typedef struct rtp_shape {
    int32_t B;      /* batch */
    int32_t Lq;     /* query rows per batch entry */
    int32_t Lk;     /* key rows per batch entry (cache length) */
    int32_t H;      /* query heads */
    int32_t Hkv;    /* kv heads; H % Hkv == 0 */
    int32_t D;      /* head dimension, must be 128 */
    int64_t q_pos0; /* absolute position of query row 0 (prefill 0, decode Lk-1) */
} rtp_shape;

typedef struct rtp_view {
    void* ptr;        /* device pointer to element [0][0][0][0] */
    int64_t stride_b; /* elements between batch entries */
    int64_t stride_l; /* elements between consecutive rows */
} rtp_view;

/* Bytes of workspace `op` needs for this shape (always >= 256). */
RTP_API size_t rtp_workspace_size(rtp_op op, const rtp_shape* shape, const uint8_t* kv_role,
                          int32_t k16_per_kv_head);

/* Zero a workspace (enqueued on `stream`). */
RTP_API rtp_status rtp_workspace_init(void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Indexer projection [FASB §Low-Dimensional Projection Mechanism]:
 *   q16[b][i][hr][c] = bf16_rn( sum_d q[b][i][h(hr)][d] * Wq16[hr][d][c] )
 *   k16[b][j][s ][c] = bf16_rn( sum_d k[b][j][g(s)][d]  * Wk16[s][d][c] )
 * with fp32 accumulation and one round-to-nearest-even to bf16.  Shapes: q has
 * shape->Lq rows of H heads, k has shape->Lk rows of Hkv heads (either count may
 * be 0 to skip that half).  Wq16 [H_ret][128][16], Wk16 [H_k16][128][16] bf16,
 * contiguous and 16-byte aligned (else RTP_ERR_ALIGNMENT).  The fp32 sum runs
 * in one fixed order for every call, so a key's k16 is the same whether it is
 * projected in a prefill or appended in a decode step.  Decode appends the new
 * key by passing views offset to the new row.  No workspace.
 */
RTP_API rtp_status rtp_index_scores(const rtp_shape* shape, const uint8_t* kv_role,
                            int32_t k16_per_kv_head, rtp_view q, rtp_view k,
                            const void* Wq16, const void* Wk16, rtp_view q16,
                            rtp_view k16, rtp_stream_t stream);

/*
 * Exact dynamic top-p per retrieval row [FASB §Dynamic Top-p Selection
 * Mechanism, Eq. 5].  For every (b, hr, i) with P = q_pos0 + i:
 *   s_j = q16[b][i][hr] . k16[b][j][slot]  for j = 0..P  (fp32),
 *   w_j = exp(s_j - max s), Z = sum w_j,
 *   kept set S = shortest prefix of the keys ordered by (s desc, j asc) whose
 *   mass reaches p*Z (p >= 1: all keys; p == 0: the argmax).
 * Outputs, [B][H_ret][Lq] contiguous:
 *   thr[]   the row threshold t (score of the last kept key; -inf when p >= 1),
 *   jtie[]  key j is kept  <=>  s_j > t  or  (s_j == t and j <= jtie),
 *   count[] |S|,
 *   mass[]  (nullable) kept mass / Z.
 * The scores are recomputed by rtp_sparse_attn_prefill with the identical
 * arithmetic, so (thr, jtie) reproduce S exactly there.
 * Workspace: rtp_workspace_size(RTP_OP_TOPP_SELECT, ...) asks for the status
 * word plus two candidate-list slots per SM (128 rows x 8128 keys x 8 bytes
 * each, about 2.5 GB on 148 SMs).  A workspace of at least 256 bytes but
 * smaller than that is accepted: the kernel then refines every dense crossing
 * range with extra sweeps instead of parked lists (same results, slower).
 */
RTP_API rtp_status rtp_topp_select(const rtp_shape* shape, const uint8_t* kv_role,
                           int32_t k16_per_kv_head, rtp_view q16, rtp_view k16, float p,
                           float* thr, int32_t* jtie, int32_t* count, float* mass,
                           void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Exact attention over each retrieval row's kept set (prefill)
 * [FASB §Dynamic Top-p Selection Mechanism, sparse attention formula]:
 *   O[b][i][h] = sum_{j in S} softmax_S(scale * q.k_j) v_j,
 * S given by (thr, jtie) from rtp_topp_select on the same q16/k16.
 * o: retrieval heads written (bf16), lse (nullable): [B][H][Lq] fp32, natural
 * log of the softmax denominator including the scale.
 * thr == jtie == NULL selects the p >= 1 case, every causal key kept: the
 * retrieval heads run on the dense tile schedule and q16/k16 are not read (may
 * be null views).  That is the prefill the summary describes, retrieval heads
 * attending densely while only the local heads are sparse [FASB
 * §Hardware-Aware Fast Top-p Decoding Kernel, "Prefill kernel"].  Passing only
 * one of the two is RTP_ERR_INVALID_ARG.
 */
RTP_API rtp_status rtp_sparse_attn_prefill(const rtp_shape* shape, const uint8_t* kv_role,
                                   int32_t k16_per_kv_head, rtp_view q, rtp_view k,
                                   rtp_view v, rtp_view q16, rtp_view k16,
                                   const float* thr, const int32_t* jtie,
                                   float softmax_scale, rtp_view o, float* lse,
                                   void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * One decode step for the retrieval heads (shape->Lq == 1, q_pos0 == Lk - 1):
 * indexer scores of the new query against the whole k16 cache (each a 16-term
 * tensor-core dot product, as in rtp_topp_select), exact top-p, union gather of
 * the kept K/V rows per kv head, exact attention, split-KV merge.  The k16 cache must already hold the new token's key (rtp_index_scores).
 * Optional outputs ([B][H_ret], nullable): thr, jtie, count, mass as in
 * rtp_topp_select.
 */
RTP_API rtp_status rtp_sparse_attn_decode(const rtp_shape* shape, const uint8_t* kv_role,
                                  int32_t k16_per_kv_head, rtp_view q, rtp_view k_cache,
                                  rtp_view v_cache, rtp_view q16, rtp_view k16_cache,
                                  float p, float softmax_scale, rtp_view o, float* lse,
                                  float* thr, int32_t* jtie, int32_t* count, float* mass,
                                  void* ws, size_t ws_bytes, rtp_stream_t stream);

/* Token selection rule of a retrieval decode step (rtp_sparse_attn_decode_select). */
typedef enum rtp_select {
    RTP_SELECT_TOPP = 0,       /* exact token-level top-p (as rtp_sparse_attn_decode) */
    RTP_SELECT_BLOCK_TOPP = 1, /* block-level approximate top-p, 64-key blocks */
    RTP_SELECT_TOPK = 2        /* static top-k */
} rtp_select;

/*
 * One decode step for the retrieval heads with a choice of selection rule; the
 * scores, the union gather and the split-KV attention are those of
 * rtp_sparse_attn_decode, which equals this call with RTP_SELECT_TOPP.
 *  - RTP_SELECT_BLOCK_TOPP [FASB §Hardware-Aware Fast Top-p Decoding Kernel,
 *    steps 1-5]: keys 0..P in blocks of 64 (the last one shorter), each
 *    reduced to its max m_b and the log-sum-exp l_b of its scores; a 256-bin
 *    histogram over [min m_b, max m_b], bin = min(255, floor(((m_b - lo) /
 *    (hi - lo)) * 256)) evaluated in fp64 from the fp32 scores (all blocks in
 *    bin 255 when hi == lo); each bin sums exp(l_b - hi); the bins are walked
 *    from the top until the running mass reaches p of the total (p >= 1: every
 *    block) and every block of that bin or above is kept, all its keys
 *    attended.  block_mask (nullable) receives, per row [B][H_ret], the
 *    ceil(ceil((P + 1) / 64) / 32) words of one bit per block (bit b % 32 of
 *    word b / 32).  count = kept keys, mass = their share of the indexer
 *    softmax mass; thr and jtie are not written.
 *  - RTP_SELECT_TOPK [FASB §5 Experimental Analysis, the method's static top-k
 *    variant, k = 4096 there]: the top_k highest scores (top_k >= 1), ties to
 *    the lower index; every key when top_k > P.  thr, jtie, count, mass as in
 *    rtp_topp_select (thr = -inf when every key is kept).  p is ignored.
 *  - scores_out (nullable): [B][H_ret][P + 1] fp32, the indexer scores the
 *    selection used (each a 16-term tensor-core dot product of bf16 q16 and
 *    k16 with fp32 accumulation), for tests and diagnostics.
 * Workspace: rtp_workspace_size(RTP_OP_SPARSE_DECODE, ...), as
 * rtp_sparse_attn_decode.
 */
RTP_API rtp_status rtp_sparse_attn_decode_select(
    const rtp_shape* shape, const uint8_t* kv_role, int32_t k16_per_kv_head, rtp_view q,
    rtp_view k_cache, rtp_view v_cache, rtp_view q16, rtp_view k16_cache, rtp_select select,
    float p, int32_t top_k, float softmax_scale, rtp_view o, float* lse, float* thr,
    int32_t* jtie, int32_t* count, float* mass, uint32_t* block_mask, float* scores_out,
    void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Local heads: keys j <= P with j < n_sink or j > P - window
 * [FASB §Local Head Attention Pattern].  Prefill (Lq > 1) and decode (Lq == 1)
 * both go through this call.  window >= 1, n_sink >= 0.
 */
RTP_API rtp_status rtp_local_attn(const rtp_shape* shape, const uint8_t* kv_role, int32_t window,
                          int32_t n_sink, rtp_view q, rtp_view k, rtp_view v,
                          float softmax_scale, rtp_view o, float* lse, void* ws,
                          size_t ws_bytes, rtp_stream_t stream);

/*
 * Window-only local-head cache [FASB §Local Head Attention Pattern, decode: the
 * local heads keep only the sink tokens and the sliding window, so their cache
 * stays O(window) however long the sequence grows].
 *
 * A ring cache holds the local kv heads only: k_ring / v_ring are
 * [B][n_sink + window][n_local_kv][128] bf16 views (rtp_view with heads =
 * number of local kv heads, in increasing kv head order).  Position j < n_sink
 * lives in row j; position j >= n_sink in row n_sink + (j - n_sink) % window.
 *
 * rtp_local_ring_write copies the local kv heads of source rows into the ring:
 * shape->Lq source rows of k / v ([B][Lq][Hkv][128], row i = absolute position
 * shape->q_pos0 + i; shape->Lk is not used).  Only the sinks and the last
 * `window` positions of the range are copied (earlier ones would be
 * overwritten): after a prefill, write rows 0..L-1 once; each decode step then
 * writes its new token (Lq = 1, q_pos0 = its position).  Positions must be
 * written in increasing order over calls.  No workspace.
 */
RTP_API rtp_status rtp_local_ring_write(const rtp_shape* shape, const uint8_t* kv_role,
                                        int32_t window, int32_t n_sink, rtp_view k, rtp_view v,
                                        rtp_view k_ring, rtp_view v_ring, rtp_stream_t stream);

/*
 * Local-head decode from a ring cache: as rtp_local_attn with shape->Lq == 1
 * (query at P = shape->q_pos0, shape->Lk >= P + 1), keys j <= P with
 * j < n_sink or j > P - window read from k_ring / v_ring, which must hold every
 * such position (rtp_local_ring_write up to P).  The keys are visited in the
 * same order as rtp_local_attn over a full cache, so the result is the same bit
 * for bit.  Workspace: rtp_workspace_size(RTP_OP_LOCAL, ...).
 */
RTP_API rtp_status rtp_local_attn_decode_ring(const rtp_shape* shape, const uint8_t* kv_role,
                                              int32_t window, int32_t n_sink, rtp_view q,
                                              rtp_view k_ring, rtp_view v_ring,
                                              float softmax_scale, rtp_view o, float* lse,
                                              void* ws, size_t ws_bytes, rtp_stream_t stream);

/*
 * Local-head decode that allocates nothing (the paper has no counterpart; this
 * is a deployment variant of rtp_local_attn with shape->Lq == 1).
 *
 * For callers that cannot hand the library a workspace: code that runs under a
 * memory allocator it does not own (a host framework's fixed pool, a plugin
 * interface that passes only inputs and outputs) or in a phase where device
 * allocation is not allowed.  The split-KV partials live in
 * one file-scope device array of RTP_NOALLOC_SCRATCH_BYTES (8 MiB) that every GPU
 * which loads the library holds until the process exits.
 *  - Same arguments and results as rtp_local_attn for one decode token, minus
 *    the workspace.  Shapes whose partials exceed the array return
 *    RTP_ERR_SCRATCH_LIMIT before anything is enqueued.  The need is 256 bytes
 *    plus 8448 bytes per (batch entry, local kv head, split), with
 *    min(256, ceil(296 / (B * local_kv_heads)), ceil(n_keys / 64)) splits, at
 *    least 1; n_keys is the number of sink and window keys, at most
 *    window + n_sink.
 *  - Every call looks the array's device address up (cudaGetSymbolAddress)
 *    on the current device, so a device reset is harmless.  The first call on
 *    a device also loads the library's device code there; make that first call
 *    outside any stream capture.
 *  - Every call reuses the same array and overwrites what the last call left
 *    there (nothing in it needs clearing between calls); calls that overlap on
 *    the GPU (other streams, other threads) race on it and must be serialised
 *    by the caller.
 *  - Never calls cudaMalloc, cudaFree or any allocating routine.
 */
#define RTP_NOALLOC_SCRATCH_BYTES (8u << 20)
RTP_API rtp_status rtp_local_attn_decode_noalloc(const rtp_shape* shape, const uint8_t* kv_role,
                                                 int32_t window, int32_t n_sink, rtp_view q,
                                                 rtp_view k, rtp_view v, float softmax_scale,
                                                 rtp_view o, float* lse, rtp_stream_t stream);

/*
 * Baseline: dense causal softmax attention on every head (keys 0..P).
 */
RTP_API rtp_status rtp_dense_attn(const rtp_shape* shape, rtp_view q, rtp_view k, rtp_view v,
                          float softmax_scale, rtp_view o, float* lse, void* ws,
                          size_t ws_bytes, rtp_stream_t stream);

/* Human-readable name of a status code (static storage). */
RTP_API const char* rtp_status_string(rtp_status status);

/* Synchronises `stream`, reads and clears the device status word at the start
 * of `ws`; RTP_OK if no kernel gave up a bounded wait since the last read. */
RTP_API rtp_status rtp_get_device_status(void* ws, rtp_stream_t stream);

/*
 * Kernel trace (no counterpart in the paper; a measurement aid).  While
 * enabled, every kernel the library launches is bracketed by two CUDA events
 * recorded on its launch stream (inside a stream capture they become external
 * event-record nodes, so each replay of the graph re-times its kernels).
 * rtp_trace_read synchronises those events and returns, per kernel name, the
 * number of recorded launches and their summed device time (ms) as of the last
 * time each event completed.  Not thread-safe against concurrent enable/reset;
 * costs nothing while disabled.
 */
typedef struct rtp_trace_entry {
    char name[48];
    int64_t launches;
    double total_ms;
} rtp_trace_entry;

/* One recorded launch: start and end, in ms after the start of the first
 * launch recorded since the last rtp_trace_reset (as of its last completion). */
typedef struct rtp_trace_launch {
    char name[48];
    double start_ms;
    double end_ms;
} rtp_trace_launch;

RTP_API void rtp_trace_enable(int on);
RTP_API void rtp_trace_reset(void);
/* Fills up to max_entries entries; returns the number filled, or -1 on a CUDA error. */
RTP_API int rtp_trace_read(rtp_trace_entry* out, int max_entries);
/* The recorded launches in recording order (up to max_entries); returns the
 * number filled, or -1 on a CUDA error. */
RTP_API int rtp_trace_timeline(rtp_trace_launch* out, int max_entries);

/*
 * Measurement aid (no counterpart in the paper): launches `blocks` CTAs of 256
 * threads that each issue iters x 8 dependent-chain ex2.approx.f32
 * instructions (blocks * 2048 * iters in all), for timing the device's exp
 * rate with CUDA events.  `out`: device buffer of blocks * 256 floats, never
 * written in practice.
 */
RTP_API rtp_status rtp_probe_ex2(int32_t blocks, int32_t iters, float* out, rtp_stream_t stream);

/* Library version, e.g. "0.1.0". */
RTP_API const char* rtp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RTP_H_ */
