/*
 * moe_nonexpand.h -- C ABI of the local MoE expert forward on the "non-expand"
 * routed layout, for NVIDIA B200 (sm_100a).
 *
 * The problem statement follows sonic-moe issue #68 ("End-to-end DeepEP v2
 * non-expand + SonicMoE integration"):
 *   - input layout (the non-expand receive block): x [N,H], topk_idx [N,K]
 *     holding a local expert id or -1 for an invalid slot, topk_w [N,K];
 *   - the proposed entry point moe_deepep_nonexpand_inputs(recv_x,
 *     recv_topk_idx, recv_topk_weights, total_pairs, w1, b1, w2, b2, E,
 *     stream_id, activation_type, ...), which these calls follow;
 *   - the list of metadata the entry point builds directly from [N,K]
 *     (expert_frequency, expert_frequency_offset, x_gather_idx,
 *     s_scatter_idx, s_reverse_scatter_idx,
 *     num_activated_expert_per_token_offset, compact router_scores [P]);
 *   - the target dataflow: the local expert compute yields local_out [N,H].
 * The expert MLP is the gated up projection with "silu times up" and the down
 * projection (qwen3_5.py commit notes, CCCL segmented-sort recipe, steps 3-5;
 * sonic-moe write-up, "The MoE class takes a routing count and a kernel
 * backend": SWIGLU and optional biases).  The gate/up columns of w1 are
 * interleaved (g0,u0,g1,u1,...) or concatenated (all gates, then all ups)
 * (sonic-moe write-up, "Interleaved by default, concatenated if your model
 * is HuggingFace").
 *
 * Definitions used throughout:
 *   pair q     -- the q-th valid slot in row-major (token, slot) order; a slot
 *                 is valid when 0 <= topk_idx[t,k] < E.  P = number of pairs.
 *   position p -- index in the stable expert-sorted order of the pairs
 *                 (expert ascending, then q ascending).
 *   out[t,:]   = sum over token t's pairs q, in q order, of
 *                topk_w[t,k(q)] * ( silu(g) * u ) . w2[e] + b2[e] ),
 *                with [g|u] taken from x[t,:] . w1[e] + b1[e].
 *                A token without a valid slot gets a zero row.
 *
 * Conventions:
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise, and
 *     every buffer is owned by the caller.  The library allocates nothing and
 *     keeps no state besides per-device launch settings.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Only moe_nonexpand_read_error synchronises the host.
 *   - Layouts are dense row-major; x, w1, w2, out must be 16-byte aligned.
 *   - Dtypes: x, w1, b1, w2, b2, out are bf16; topk_idx int32; topk_w fp32.
 *   - Return value: MOE_OK or one of the MOE_ERR_* codes below; on error
 *     nothing has been enqueued.  Errors found on the device (bad expert ids,
 *     a pair count that disagrees with total_pairs, an internal wait that
 *     timed out) are recorded in the workspace's device error word and read
 *     with moe_nonexpand_read_error.
 *   - Supported sizes: N >= 0, 1 <= K <= 32, 1 <= E <= 1024, N*K < 2^31,
 *     H and I multiples of 64 (tensor-memory-access and MMA alignment), and
 *     P_cap * max(H, I) < 2^31 where P_cap is total_pairs when it is given
 *     and N*K otherwise.
 */
#ifndef MOE_NONEXPAND_H
#define MOE_NONEXPAND_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Host return codes. */
#define MOE_OK 0
#define MOE_ERR_ARG 1         /* null required pointer, bad N/K/E, bad enum, misaligned pointer */
#define MOE_ERR_SHAPE 2       /* H or I not a multiple of 64, or sizes overflow 32-bit indexing */
#define MOE_ERR_WS 3          /* workspace too small (or null) */
#define MOE_ERR_CUDA 4        /* a CUDA runtime call or launch failed */
#define MOE_ERR_DEVICE 5      /* current device is not sm_100 (B200-class) */

/* Bits of the device error word (moe_nonexpand_read_error). */
#define MOE_DEVERR_BAD_EXPERT_ID 0x1u /* an id outside {-1} U [0,E) was seen; that slot was skipped */
#define MOE_DEVERR_PAIR_COUNT 0x2u    /* counted P != total_pairs (total_pairs >= 0) or P > P_cap */
#define MOE_DEVERR_TIMEOUT 0x4u       /* an internal pipeline wait gave up; outputs are invalid */
#define MOE_DEVERR_ABORTED 0x8u       /* P > P_cap: GEMMs and combine were skipped, out unwritten */
#define MOE_DEVERR_BAD_TOKEN 0x10u    /* pair list: a token id outside [0,N) (that pair was skipped)
                                         or token ids not in ascending order (offsets unspecified) */

/* activation argument */
#define MOE_ACT_SWIGLU 0
/* gate_up_layout argument */
#define MOE_LAYOUT_INTERLEAVED 0
#define MOE_LAYOUT_CONCATENATED 1

/* The routing metadata of issue #68's list, in caller-owned device memory.
 * P_cap = total_pairs if total_pairs >= 0, else N*K. */
typedef struct moe_meta_t {
    int32_t *expert_frequency;         /* [E]     pairs per expert                          */
    int32_t *expert_frequency_offset;  /* [E+1]   exclusive prefix sum; [E] = P             */
    int32_t *x_gather_idx;             /* [P_cap] token (row of x) at sorted position p     */
    int32_t *s_scatter_idx;            /* [P_cap] pair index q at sorted position p         */
    int32_t *s_reverse_scatter_idx;    /* [P_cap] sorted position p of pair q               */
    int32_t *token_offset;             /* [N+1]   num_activated_expert_per_token_offset:
                                          pairs of token t are q in [off[t], off[t+1])      */
    float *scores;                     /* [P_cap] compact router scores, scores[q]          */
} moe_meta_t;

/* Opaque CUDA handles, ABI-compatible with cudaStream_t / cudaEvent_t. */
typedef struct CUstream_st *moe_stream_t;
typedef struct CUevent_st *moe_event_t;

/*
 * Bytes of workspace needed by moe_nonexpand_forward for these sizes (pass
 * H = I = 0 for what moe_nonexpand_metadata alone needs).  The workspace
 * holds the per-tile histograms, the GEMM tile table, the metadata when the
 * caller does not provide it, and the intermediates h [P_cap,I] (bf16) and
 * y [P_cap,H] (fp16 with a power-of-two exponent per 32-column block).  Its
 * contents need no initialisation: every call writes what
 * it reads.  One workspace must not be used by two calls that can run at the
 * same time.
 * Returns 0 for arguments outside the supported sizes.
 */
MOE_API size_t moe_nonexpand_workspace_bytes(int64_t N, int32_t H, int32_t I, int32_t E, int32_t K,
                                     int64_t total_pairs);

/*
 * Routing metadata only (issue #68 metadata list), built from [N,K]:
 * histogram, exclusive offsets, stable counting sort of the pairs by expert,
 * per-token pair offsets and compact scores.  Results are bit-exact and
 * deterministic.  `meta` (host struct of device pointers) must be non-null
 * with every field set.  Invalid slots' weights are loaded with their ids
 * but never used: any value, NaN included, leaves every result unchanged.
 */
MOE_API int moe_nonexpand_metadata(const int32_t *topk_idx, const float *topk_w,
                           int64_t N, int32_t K, int32_t E, int64_t total_pairs,
                           const moe_meta_t *meta, void *ws, size_t ws_bytes,
                           moe_stream_t stream);

/*
 * moe_nonexpand_metadata without a workspace: the same metadata, bit for bit,
 * for callers that cannot allocate device memory when they call in -- for
 * example a serving process whose memory pool is sized and frozen at start-up,
 * or a plugin whose host framework owns every device allocation -- and so
 * cannot provide the `ws` buffer the other entry points need.  The pages have
 * no counterpart to this call; it exists for those callers only.
 *
 * Scratch: a fixed 160 KiB array in device memory that belongs to the library
 * (a file-scope __device__ array: every GPU that loads the library keeps it
 * until the process exits).  It holds what the metadata kernels need besides
 * their inputs and outputs -- a header with the device error word, the
 * per-tile histogram table (at most 32768 entries: the tiling keeps
 * tiles x E within that), per-tile counts and the GEMM tile table -- which
 * fits for every supported size (E <= 1024); a size that would not fit
 * returns MOE_ERR_WS.  The call allocates nothing: no cudaMalloc, cudaFree or
 * allocating library routine.  Argument checks are those of
 * moe_nonexpand_metadata (sizes, null and misaligned pointers give
 * MOE_ERR_ARG before any CUDA call).
 *
 * The first call on a device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture.  All calls share the one array, which keeps the last call's
 * contents (the kernels write every scratch byte they read, so nothing has to
 * be cleared): calls that can overlap on the GPU -- on different streams, or
 * on one device from several host threads without ordering -- race and must
 * not be issued.  Device-side error bits (bad ids, pair-count mismatch) land
 * in the scratch's error word, which every call rewrites whole; read them with
 * moe_nonexpand_metadata_noalloc_read_error.  The outputs follow the same
 * rules as moe_nonexpand_metadata.
 */
MOE_API int moe_nonexpand_metadata_noalloc(const int32_t *topk_idx, const float *topk_w,
                                   int64_t N, int32_t K, int32_t E, int64_t total_pairs,
                                   const moe_meta_t *meta, moe_stream_t stream);

/*
 * The device error word (MOE_DEVERR_* bits) of the last
 * moe_nonexpand_metadata_noalloc call on the current device, copied to the
 * host pointer *err_word after `stream` has been synchronised -- the
 * counterpart of moe_nonexpand_read_error for the library's own scratch.
 * Call it on the stream of that metadata call (or after it has finished).
 * Like the call it reports on, it has no counterpart on the pages.
 */
MOE_API int moe_nonexpand_metadata_noalloc_read_error(moe_stream_t stream, uint32_t *err_word);

/*
 * The whole local expert forward: metadata, gathered grouped GEMM up with
 * bias and SwiGLU fused in its epilogue (rows of x are gathered straight
 * through x_gather_idx; no permuted copy of x is made), grouped GEMM down
 * with bias, and the deterministic score-weighted combine (each token sums
 * its pairs in slot order through s_reverse_scatter_idx; no atomics).
 *   x    [N,H]   bf16       w1 [E,H,2I] bf16     b1 [E,2I] bf16 or NULL
 *   w2   [E,I,H] bf16       b2 [E,H]    bf16 or NULL
 *   out  [N,H]   bf16 (written; rounded to nearest even from an fp32 sum)
 *   meta_out: NULL keeps the metadata inside the workspace; otherwise the
 *             metadata is also left in the caller's buffers.
 * Intermediates: h = silu(g)*u is stored as bf16; y = h.w2 + b2 as fp16
 * scaled by a power of two per row and 32-column block (11 significant bits
 * at bf16's range; moe_ws_layout_t.y and .y_scale), which the combine reads.
 */
MOE_API int moe_nonexpand_forward(const void *x, const int32_t *topk_idx, const float *topk_w,
                          int64_t N, int32_t H, int32_t I, int32_t E, int32_t K,
                          int64_t total_pairs,
                          const void *w1, const void *b1, const void *w2, const void *b2,
                          int32_t activation, int32_t gate_up_layout,
                          void *out, const moe_meta_t *meta_out,
                          void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Same as moe_nonexpand_forward, and records five caller-created CUDA events
 * on `stream` (a host array of 5 moe_event_t, none null): before the
 * metadata, after the metadata, after the GEMM up, after the GEMM down and
 * after the combine.  Used to time each stage on the launching stream.
 */
MOE_API int moe_nonexpand_forward_timed(const void *x, const int32_t *topk_idx, const float *topk_w,
                                int64_t N, int32_t H, int32_t I, int32_t E, int32_t K,
                                int64_t total_pairs,
                                const void *w1, const void *b1, const void *w2, const void *b2,
                                int32_t activation, int32_t gate_up_layout,
                                void *out, const moe_meta_t *meta_out,
                                void *ws, size_t ws_bytes, moe_stream_t stream,
                                const moe_event_t *stage_events);

/*
 * The combine step alone (issue #68 dataflow, local_out [N,H]):
 *   out[t,:] = bf16( sum over q in [token_offset[t], token_offset[t+1]), in q
 *              order, of scores[q] * y[s_reverse_scatter_idx[q], :] )
 * with an fp32 accumulator.  y is [P_cap,H] bf16 in expert-sorted order.
 * Reads only the token_offset, s_reverse_scatter_idx and scores fields of
 * `meta`.  No workspace is used.
 */
MOE_API int moe_nonexpand_combine(const void *y, const moe_meta_t *meta, int64_t N, int32_t H,
                          void *out, moe_stream_t stream);

/*
 * Routing input in either of two layouts, for the moe_nonexpand_routed_* calls.
 *
 *   MOE_ROUTING_TOPK   the non-expand table of sonic-moe issue #68:
 *                      expert_idx = topk_idx [N,K] (-1 = invalid slot),
 *                      weights = topk_w [N,K], token_idx = NULL, K slots per
 *                      token, pairs = total_pairs (>= 0) or -1 when unknown.
 *   MOE_ROUTING_PAIRS  the compact pair list of sonic-moe's general routing API
 *                      (issue #68: token_indices / expert_indices /
 *                      router_scores [P], one entry per (token, expert) pair):
 *                      token_idx = token_indices [P], ascending, each in
 *                      [0,N); expert_idx = expert_indices [P]; weights =
 *                      router_scores [P]; pairs = P; K is ignored.  Pair q of
 *                      the metadata is the q-th entry that is kept.
 *
 * index_dtype gives the dtype of expert_idx and token_idx (int32 or int64;
 * int64 ids outside the int32 range are invalid).  An expert id outside
 * [0,E) other than -1 sets MOE_DEVERR_BAD_EXPERT_ID and a token id outside
 * [0,N) sets MOE_DEVERR_BAD_TOKEN; either way that entry is skipped.  A pair
 * list whose tokens are not ascending sets MOE_DEVERR_BAD_TOKEN and leaves
 * token_offset unspecified.  All arrays are device memory, caller-owned.
 */
#define MOE_ROUTING_TOPK 0
#define MOE_ROUTING_PAIRS 1
#define MOE_INDEX_INT32 0
#define MOE_INDEX_INT64 1

typedef struct moe_routing_t {
    int32_t kind;              /* MOE_ROUTING_TOPK or MOE_ROUTING_PAIRS */
    int32_t index_dtype;       /* MOE_INDEX_INT32 or MOE_INDEX_INT64 */
    int64_t N;                 /* tokens: rows of x and out */
    int32_t K;                 /* TOPK: slots per token (1..32); PAIRS: ignored */
    int64_t pairs;             /* TOPK: total_pairs or -1; PAIRS: P >= 0 */
    const void *expert_idx;    /* TOPK: [N,K]; PAIRS: [P] */
    const float *weights;      /* TOPK: [N,K]; PAIRS: [P] */
    const void *token_idx;     /* PAIRS: [P] ascending; TOPK: NULL */
} moe_routing_t;

/* Workspace bytes for a routed call (H = I = 0: metadata only); 0 = invalid. */
MOE_API size_t moe_nonexpand_routed_workspace_bytes(const moe_routing_t *routing, int32_t H, int32_t I,
                                                    int32_t E);

/* moe_nonexpand_metadata for either routing layout (P_cap = pairs for a pair
 * list, as for the table). */
MOE_API int moe_nonexpand_routed_metadata(const moe_routing_t *routing, int32_t E, const moe_meta_t *meta,
                                  void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_nonexpand_forward for either routing layout: out[t,:] sums, in pair
 * order, the score-weighted expert rows of the pairs of token t. */
MOE_API int moe_nonexpand_routed_forward(const void *x, const moe_routing_t *routing, int32_t H, int32_t I,
                                 int32_t E, const void *w1, const void *b1, const void *w2, const void *b2,
                                 int32_t activation, int32_t gate_up_layout, void *out,
                                 const moe_meta_t *meta_out, void *ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Training: forward that keeps what the backward needs, and the backward.
 *
 * The pages leave the backward open (sonic-moe issue #68 asks how the routing
 * scores' gradient gets back to [N_recv,K]; the write-up names the layer a
 * training layer).  These calls apply the chain rule to the forward above,
 * for the non-expand [N,K] routing:
 *   dy_q  = s_q dout_t               (the pair's share of out_t = sum_q s_q y_q)
 *   ds_q  = <dout_t, y_q>            -> dtopk_w[t,k] of the slot of q (0 at invalid slots)
 *   dh_q  = dy_q . W2[e]^T
 *   dg    = dh u silu'(g), du = dh silu(g), silu'(g) = sig(g)(1 + g(1 - sig(g)))
 *   dz_q  = (dg, du) at the gate/up columns of the layout
 *   dW2[e] = sum h_q^T dy_q,  db2[e] = sum dy_q,
 *   dW1[e] = sum x_t^T dz_q,  db1[e] = sum dz_q,  dx_t = sum over t's pairs of dz_q . W1[e]^T
 * (sums over the pairs q of expert e, or of token t).
 *
 * moe_nonexpand_train_workspace_bytes: a larger workspace that also holds z
 * (fp32 [P_cap,2I], bias included: the SwiGLU derivative is sensitive to the
 * gate's precision near silu's minimum), dz (bf16 [P_cap,2I]) and dy (bf16
 * [P_cap,H]).
 *
 * moe_nonexpand_forward_train: moe_nonexpand_forward that keeps the metadata,
 * h, y and z in the training workspace for the backward.
 *
 * moe_nonexpand_backward: the gradients, given dout [N,H] bf16 and the
 * training workspace of a forward_train call with the same x, routing,
 * weights, layout and sizes (nothing in between may use that workspace).
 * Outputs (device, caller-owned, all written): dx [N,H], dw1 [E,H,2I],
 * dw2 [E,I,H] bf16; dtopk_w [N,K] fp32; db1 [E,2I] and db2 [E,H] bf16 when
 * not NULL.  The workspace's dy, dz and y regions are overwritten.  Products
 * accumulate in fp32; dh is computed from dout and the weights (bf16 inputs)
 * with the score applied in fp32; dy, dz and the per-pair dx rows are stored
 * in bf16.
 * Deterministic: no atomics decide any sum.  Enqueued on stream, no sync.
 * Same return codes as moe_nonexpand_forward; MOE_ERR_WS for a workspace
 * smaller than the training size.
 */
MOE_API size_t moe_nonexpand_train_workspace_bytes(int64_t N, int32_t H, int32_t I, int32_t E, int32_t K,
                                                   int64_t total_pairs);

MOE_API int moe_nonexpand_forward_train(const void *x, const int32_t *topk_idx, const float *topk_w, int64_t N,
                                        int32_t H, int32_t I, int32_t E, int32_t K, int64_t total_pairs,
                                        const void *w1, const void *b1, const void *w2, const void *b2,
                                        int32_t activation, int32_t gate_up_layout, void *out, void *ws,
                                        size_t ws_bytes, moe_stream_t stream);

MOE_API int moe_nonexpand_backward(const void *dout, const void *x, const int32_t *topk_idx, const float *topk_w,
                                   int64_t N, int32_t H, int32_t I, int32_t E, int32_t K, int64_t total_pairs,
                                   const void *w1, const void *w2, int32_t activation, int32_t gate_up_layout,
                                   void *dx, void *dw1, void *db1, void *dw2, void *db2, float *dtopk_w,
                                   void *ws, size_t ws_bytes, moe_stream_t stream);

/* moe_nonexpand_backward plus eight events recorded on the stream around its
 * seven steps: score gradients and dy, dh + SwiGLU backward, dW2, dW1 (with
 * the gather of x rows it reads), dx rows, the dx combine, the bias
 * gradients. */
MOE_API int moe_nonexpand_backward_timed(const void *dout, const void *x, const int32_t *topk_idx,
                                         const float *topk_w, int64_t N, int32_t H, int32_t I, int32_t E,
                                         int32_t K, int64_t total_pairs, const void *w1, const void *w2,
                                         int32_t activation, int32_t gate_up_layout, void *dx, void *dw1,
                                         void *db1, void *dw2, void *db2, float *dtopk_w, void *ws,
                                         size_t ws_bytes, moe_stream_t stream, const moe_event_t *stage_events);

/*
 * Training for either routing layout (moe_routing_t; see the routed calls):
 * the same computation as moe_nonexpand_forward_train / moe_nonexpand_backward.
 * dweights has the shape of routing->weights ([N,K] for the table, [P] for a
 * pair list) and receives each slot's score gradient, 0 at slots that are no
 * pair (expert -1, bad ids, bad tokens).
 */
MOE_API size_t moe_nonexpand_routed_train_workspace_bytes(const moe_routing_t *routing, int32_t H, int32_t I,
                                                          int32_t E);

MOE_API int moe_nonexpand_routed_forward_train(const void *x, const moe_routing_t *routing, int32_t H, int32_t I,
                                               int32_t E, const void *w1, const void *b1, const void *w2,
                                               const void *b2, int32_t activation, int32_t gate_up_layout,
                                               void *out, void *ws, size_t ws_bytes, moe_stream_t stream);

MOE_API int moe_nonexpand_routed_backward(const void *dout, const void *x, const moe_routing_t *routing, int32_t H,
                                          int32_t I, int32_t E, const void *w1, const void *w2, int32_t activation,
                                          int32_t gate_up_layout, void *dx, void *dw1, void *db1, void *dw2,
                                          void *db2, float *dweights, void *ws, size_t ws_bytes,
                                          moe_stream_t stream);

/*
 * Router top-k: router logits [N,E] -> the routing table topk_idx [N,K] /
 * topk_w [N,K] that moe_nonexpand_forward takes (sonic-moe write-up, "Three
 * routing strategies, selected on the command line": TC top-K routing is the
 * softmax over the top-k logits; Qwen3-style routing is the top-k of the
 * softmax over all experts, with optional renormalisation of the chosen
 * probabilities).
 *
 *   MOE_ROUTER_SOFTMAX_TOPK         w = softmax over the K chosen logits
 *   MOE_ROUTER_TOPK_SOFTMAX         w = softmax over all E logits, at the chosen
 *   MOE_ROUTER_TOPK_SOFTMAX_RENORM  the same, divided by its sum over the K chosen
 *
 * The chosen experts are the K largest logits (softmax is increasing, so all
 * modes choose alike), compared as given: fp32, or bf16 widened exactly.
 * Slot k holds the k-th largest; equal logits go to the lower expert id
 * (-0.0 equals +0.0).  A NaN logit is read as -inf.  A token whose chosen
 * logits are all -inf gets NaN weights.  Weights are computed in fp32: expf
 * of the chosen logits' differences to the largest, and for the softmax over
 * all E the fast exponential (relative error a few 1e-6) in its sum.
 *
 * logits: device, [N,E] row-major, dtype MOE_DTYPE_F32 or MOE_DTYPE_BF16.
 * topk_idx: device int32 [N,K]; topk_w: device fp32 [N,K]; both written.
 * 1 <= K <= min(E, 32), 1 <= E <= 1024.  Enqueued on stream, no sync; one
 * kernel launch.  Returns MOE_ERR_ARG for bad sizes, modes, dtypes, null or
 * misaligned pointers.
 */
#define MOE_ROUTER_SOFTMAX_TOPK 0
#define MOE_ROUTER_TOPK_SOFTMAX 1
#define MOE_ROUTER_TOPK_SOFTMAX_RENORM 2
#define MOE_DTYPE_F32 0
#define MOE_DTYPE_BF16 1

MOE_API int moe_router_topk(const void *logits, int32_t logits_dtype, int64_t N, int32_t E, int32_t K,
                            int32_t mode, int32_t *topk_idx, float *topk_w, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * Expert-parallel dispatch and combine around the local path (non-expand).
 *
 * The dataflow of "End-to-end DeepEP v2 non-expand + SonicMoE integration
 * #68": a non-expand dispatch hands every rank recv_x [N_recv,H],
 * recv_topk_idx [N_recv,K] (local expert ids, -1 for a slot whose expert
 * lives on another rank) and recv_topk_weights; the local expert compute
 * (moe_nonexpand_forward) turns them into local_out [N_recv,H]; the combine
 * returns routed_out [T,H] in the source's token order.  Non-expand: a token
 * row travels once to each rank that owns at least one of its experts.
 *
 * Conventions (readings where the pages leave the layout open):
 *  - R ranks of E_local experts each; global expert e lives on rank
 *    e / E_local as local expert e % E_local;
 *  - a destination's receive rows are blocks by source rank in rank order,
 *    the source's tokens ascending inside its block; the block of source s
 *    on rank d starts at row_off = sum over s' < s of counts[s'][d], where
 *    counts[s][d] is send_count[d] of source s (exchanged between ranks by
 *    the caller, e.g. an all-gather of the R send counts);
 *  - the combine adds the destinations' rows in ascending rank order, in
 *    fp32, with one bf16 rounding: deterministic, no atomics.
 *
 * Peer buffers: entry d of the pointer tables below is rank d's buffer as
 * seen from the calling GPU (a peer pointer, through CUDA IPC or symmetric
 * memory, when d is another GPU; plain loads and stores over NVLink, no TMA
 * and no multicast).  The caller orders the phases across ranks: every
 * rank's dispatch completes before any rank reads its receive buffers, and
 * every rank's local forward completes before any rank's combine reads it.
 * All calls are enqueued on `stream` without a host sync.
 * ------------------------------------------------------------------------- */
#define MOE_EP_MAX_RANKS 32

/*
 * Layout on one source rank.  topk_idx: device int32 [T,K] global expert ids
 * (-1: empty slot; any other id outside [0, R*E_local) is not sent and sets
 * MOE_DEVERR_BAD_EXPERT_ID in *err_word).  Writes send_idx: device int32
 * [T,R], the token's row inside its block for destination d, or -1 when d
 * owns none of its experts; send_count: device int32 [R], rows per
 * destination.  err_word: device uint32 or NULL (bits are OR-ed in, never
 * cleared).  1 <= R <= MOE_EP_MAX_RANKS, 1 <= K <= 32, E_local >= 1,
 * R*E_local < 2^31, T*R < 2^31.  One kernel launch (one CTA).
 */
MOE_API int moe_ep_layout(const int32_t *topk_idx, int64_t T, int32_t K, int32_t R, int32_t E_local,
                          int32_t *send_idx, int32_t *send_count, uint32_t *err_word, moe_stream_t stream);

/* Receive buffers of every rank, as seen from the calling (source) rank.  A row
 * at or past recv_rows[d] is never written: it sets MOE_DEVERR_ABORTED in
 * *err_word (device uint32, may be NULL) instead. */
typedef struct moe_ep_peers_t {
    void *recv_x[MOE_EP_MAX_RANKS];      /* rank d: bf16 [recv_rows_d, H], 16-byte aligned */
    int32_t *recv_idx[MOE_EP_MAX_RANKS]; /* rank d: int32 [recv_rows_d, K] local ids or -1 */
    float *recv_w[MOE_EP_MAX_RANKS];     /* rank d: fp32 [recv_rows_d, K], 0 where -1      */
    int64_t row_off[MOE_EP_MAX_RANKS];   /* first row of this source's block on rank d    */
    int64_t recv_rows[MOE_EP_MAX_RANKS]; /* rows rank d's buffers hold                     */
    uint32_t *err_word;                  /* this rank's device error word, or NULL         */
} moe_ep_peers_t;

/*
 * Dispatch on one source rank: for every token t and destination d with
 * send_idx[t,d] >= 0, row row_off[d] + send_idx[t,d] of rank d's buffers gets
 * x[t,:] (copied exactly), the local ids of t's experts on d (-1 elsewhere)
 * and their weights (0 elsewhere).  x: device bf16 [T,H] (16-byte aligned,
 * H % 8 == 0); topk_idx / topk_w: device [T,K]; send_idx: device [T,R] from
 * moe_ep_layout; peers: host struct (copied; entries d < R must be non-null).
 * One kernel launch.
 */
MOE_API int moe_ep_dispatch(const void *x, const int32_t *topk_idx, const float *topk_w, const int32_t *send_idx,
                            int64_t T, int32_t H, int32_t K, int32_t R, int32_t E_local,
                            const moe_ep_peers_t *peers, moe_stream_t stream);

/* local_out buffers of every rank, as seen from the calling (source) rank.  A row
 * at or past rows[d] is never read: it counts as 0 and sets MOE_DEVERR_ABORTED in
 * *err_word (device uint32, may be NULL). */
typedef struct moe_ep_sources_t {
    const void *local_out[MOE_EP_MAX_RANKS]; /* rank d: bf16 [rows_d, H], 16-byte aligned */
    int64_t row_off[MOE_EP_MAX_RANKS];       /* first row of this source's block on rank d */
    int64_t rows[MOE_EP_MAX_RANKS];          /* rows rank d's local_out holds              */
    uint32_t *err_word;                      /* this rank's device error word, or NULL     */
} moe_ep_sources_t;

/*
 * Combine on one source rank: out[t,:] = sum over d ascending with
 * send_idx[t,d] >= 0 of local_out_d[row_off[d] + send_idx[t,d], :], summed in
 * fp32 and rounded once to bf16; a token sent nowhere gets 0.  out: device
 * bf16 [T,H] (16-byte aligned, H % 8 == 0); src: host struct (copied).  One
 * kernel launch.
 */
MOE_API int moe_ep_combine(const moe_ep_sources_t *src, const int32_t *send_idx, int64_t T, int32_t H, int32_t R,
                           void *out, moe_stream_t stream);

/* Byte offsets of the workspace's internal arrays (for inspection and tests).
 * Offsets of arrays that the given sizes do not need are 0. */
typedef struct moe_ws_layout_t {
    size_t total;              /* == moe_nonexpand_workspace_bytes(...)       */
    size_t header;             /* 256-byte header; error word at byte 4       */
    size_t tile_hist;          /* int32 [T,E] per-tile expert histograms      */
    size_t tile_valid;         /* int32 [T]   valid slots per tile            */
    size_t tile_err;           /* int32 [T]   error bits per tile             */
    size_t gemm_tile_offset;   /* int32 [E+1] prefix of ceil(freq/256)        */
    size_t meta_freq, meta_off, meta_x_gather, meta_s_scatter, meta_s_rev,
           meta_token_offset, meta_scores;  /* metadata kept in the workspace */
    size_t h;                  /* bf16 [P_cap,I] */
    size_t y;                  /* fp16 bits [P_cap,H]: y (+ b2) per expert-sorted row, each 32-column
                                  block scaled by a power of two: value = fp16 * 2^y_scale */
    int64_t p_cap;
    int32_t meta_tiles;        /* T */
    int32_t meta_tile_slots;   /* slots per metadata tile */
    size_t z;                  /* training workspace: bf16 [P_cap,2I], w1 column order: u silu'(g) at the
                                  gate columns, silu(g) at the up columns, saved by the forward */
    size_t dz;                 /* training workspace: bf16 [P_cap,2I], dz of the backward */
    size_t dy;                 /* training workspace: bf16 [P_cap,H], dy of the backward */
    size_t slot_pair;          /* training workspace: int32 [slots], the pair of each routing slot or -1 */
    size_t ds;                 /* training workspace: fp32 [P_cap], score gradients in pair order */
    size_t train_total;        /* == moe_nonexpand_train_workspace_bytes(...) */
    size_t y_scale;            /* int8 [P_cap,H/32]: the exponent e of each row's 32-column block of y,
                                  e in [-100,113], every |y| * 2^-e at most 2^15 (the grouped GEMM puts
                                  the block's largest in [2^14, 2^15); decode-sized batches share e
                                  over up to 32 rows of one expert) */
} moe_ws_layout_t;

MOE_API int moe_nonexpand_workspace_layout(int64_t N, int32_t H, int32_t I, int32_t E, int32_t K,
                                   int64_t total_pairs, moe_ws_layout_t *layout_out);

/*
 * Copies the device error word of the last call that used `ws` to *err_word
 * (MOE_DEVERR_* bits; 0 = no error) after synchronising `stream`.  This is
 * the only call that blocks the host.
 */
MOE_API int moe_nonexpand_read_error(const void *ws, moe_stream_t stream, uint32_t *err_word);

/*
 * Self-test of the device failure path (no counterpart on the pages): launches
 * one bounded pipeline wait that nothing completes, with a limit of
 * `timeout_us` microseconds (1 .. 2,000,000).  When the wait gives up, the
 * kernel records MOE_DEVERR_TIMEOUT in the error word of `ws` (cleared first)
 * and returns; read it with moe_nonexpand_read_error.  The GEMM kernels take
 * the same path, with a 4 s limit, if a pipeline stage never completes.  Only
 * the 256-byte header of `ws` is used.
 */
MOE_API int moe_nonexpand_selftest_wait_timeout(void *ws, size_t ws_bytes, uint32_t timeout_us,
                                        moe_stream_t stream);

/* Static string for a MOE_OK / MOE_ERR_* code. */
MOE_API const char *moe_nonexpand_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_NONEXPAND_H */
