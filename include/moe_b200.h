/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) Mixture-of-Experts layer library.
 *
 * One MoE FFN layer forward pass on one GPU, in five steps:
 *   route    logits = x . W_r (+ bias), top-K, softmax over the K kept logits
 *   permute  group the (token, slot) assignments by expert (histogram, scan,
 *            stable token-order ranks, capacity drop, row gather)
 *   expert   per expert: H = silu(X W1) * (X W3); Y = H W2  (tcgen05 GEMMs)
 *   combine  y[t] = sum_k w[t,k] * Y[row(t,k)]  (deterministic gather)
 *   stats    counts, f_i, P_i, aux = E * sum f_i P_i, the top-K-only balance
 *            statistic and the router z-loss; aux-free bias update
 * moe_layer_forward runs all five on one stream; moe_layer_forward_chunked
 * runs the same layer over token chunks in a chunk-sized workspace.
 *
 * Sources (web pages; cited by title and section):
 *   [P1] "MoE serving essay", dpshk.com/news/3211971
 *   [P2] "MoE computation notes", cf-1.com/news/5905749
 *   [P3] "MoE inference engineering in practice", ybb.press/quantum-computing/18594
 *
 * Conventions for every entry point
 *   - All array arguments are DEVICE pointers to memory the caller owns; the
 *     library allocates nothing on these paths and keeps no pointer after a
 *     call returns.  Scratch space is the caller's workspace (`ws`, sized by
 *     moe_workspace_size).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *     only enqueues work on it and returns; results are ready when the stream
 *     reaches that point.  No call synchronises the device.
 *   - Layouts are dense row-major.  bf16 values are passed as their 16-bit
 *     patterns (moe_bf16).  Pointers must be 16-byte aligned; d_model and
 *     d_ff must be multiples of 16.
 *   - Status codes are returned (MOE_OK = 0, negative on error); nothing is
 *     thrown across the ABI and a failed argument check enqueues no work.
 *     Device-side failures (a bounded wait that ran out) set a flag in the
 *     workspace that moe_get_device_status reads.
 *   - Inputs must be finite; NaN or Inf in x or the weights gives unspecified
 *     routing.
 *   - Limits: 1 <= K <= E <= 256, 1 <= T <= 2^24.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

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

typedef uint16_t moe_bf16; /* bfloat16 bit pattern */

/* Problem statement of one layer call ([P2] section 3.1 names T, K, E and the
 * capacity factor; [P2] section 2 names d_model; the FFN width is d_ff).
 *   T                 tokens in the batch, exactly (no padding tokens: [P2]
 *                     section 4.3 warns that padded tokens get routed too)
 *   d_model, d_ff     hidden and expert FFN widths
 *   E, K              experts and experts per token
 *   capacity_factor   <= 0: no per-expert limit.  Otherwise each expert keeps
 *                     at most C = ceil(capacity_factor * T * K / E) assignments
 *                     (the ceiling of the exact value of the double), the
 *                     earliest tokens first ([P2] section 3.1). */
typedef struct moe_dims {
    int64_t T;
    int32_t d_model;
    int32_t d_ff;
    int32_t E;
    int32_t K;
    double capacity_factor;
} moe_dims;

enum {
    MOE_OK = 0,
    MOE_EINVAL = -1,       /* bad argument: NULL where required, size out of range */
    MOE_EUNSUPPORTED = -2, /* valid but not supported by this build (alignment, widths) */
    MOE_ECUDA = -3,        /* a CUDA runtime call failed (launch error, no device) */
    MOE_EWORKSPACE = -4,   /* workspace too small */
    MOE_ETIMEOUT = -5,     /* a device-side bounded wait ran out (from moe_get_device_status) */
    MOE_ESCRATCH = -6,     /* batch too large for the static scratch of moe_permute_noalloc */
    MOE_EINDEX = -7,       /* a dispatch input named an expert outside [0, E) (from moe_get_device_status) */
};

/* Human-readable name of a status code.  Never NULL. */
MOE_API const char* moe_status_str(int status);

/* Library ABI version (major * 100 + minor). */
MOE_API int moe_version(void);

/* Testing the device-side timeouts (no counterpart on the source pages).
 * Sets, for the expert-GEMM launches enqueued afterwards by this process,
 * the poll limit of every bounded wait (wait_polls) and of the down
 * projection's readiness wait (dependency_polls); a value <= 0 restores the
 * default (2^26 polls, seconds), other values are clamped to [1024, 2^31].
 * With dependency_never_ready != 0 the readiness target of every
 * down-projection tile is made unreachable, so those waits run out: the
 * launch ends early, with MOE_ETIMEOUT and detail 6 in the workspace status
 * flag, after its abort and drain paths have run; its outputs are undefined.
 * Lets a test exercise those paths without faulting or hanging anything.
 * Process-wide and not synchronised with launches in flight on other
 * threads: call it only between launches. */
MOE_API int moe_test_set_wait_limits(int64_t wait_polls, int64_t dependency_polls, int dependency_never_ready);

/* Capacity C of [P2] section 3.1 for these dims: -1 when there is no limit,
 * else ceil(capacity_factor * T * K / E) >= 1.  Returns < -1 on bad dims. */
MOE_API int64_t moe_capacity(const moe_dims* dims);

/* Bytes of device workspace that moe_layer_forward and the step entry points
 * need for these dims.  *bytes receives the size.  Host only. */
MOE_API int moe_workspace_size(const moe_dims* dims, size_t* bytes);

/* Zero the workspace's device status flag (enqueued on `stream`). */
MOE_API int moe_reset_device_status(void* ws, void* stream);

/* Read the workspace's device status flag: synchronises `stream`, then
 * *status = MOE_OK; MOE_ETIMEOUT with *detail naming the wait that ran out
 * (a small integer, 1..6); or MOE_EINDEX (*detail = 7) when a dispatch input
 * named an expert outside [0, E).  The first failure recorded wins; the
 * flag stays set until moe_reset_device_status.  MOE_EINDEX with detail 8
 * means an expert with rows had no valid cache slot (moe_expert_ffn_slots). */
MOE_API int moe_get_device_status(const void* ws, void* stream, int* status, int* detail);

/* Bytes of the packed expert weights moe_pack_weights writes for these dims:
 * *w13_bytes for the gate/up weights, *w2_bytes for the down weights.  Host
 * only. */
MOE_API int moe_packed_weight_bytes(const moe_dims* dims, size_t* w13_bytes, size_t* w2_bytes);

/* One-time re-layout of the expert weights for the tensor-core GEMMs.
 *   W1, W3  [E, d_model, d_ff]   (x . W1 is the gate, x . W3 the up projection)
 *   W2      [E, d_ff, d_model]   (down projection)
 *   W13p    out, moe_packed_weight_bytes(..)->w13_bytes bytes: per expert the
 *           K-major gate/up matrix [2*d_ff rows, d_model] whose rows
 *           32b..32b+15 are W1[:, 16b..16b+15]^T and rows 32b+16..32b+31 are
 *           W3[:, 16b..16b+15]^T, stored as 128-row x 64-column tiles (16 KB,
 *           row-block-major, then column-block) with the 128-byte swizzle of
 *           the tensor-core operand layout inside each tile; padding is zero
 *   W2p     out, w2_bytes bytes: per expert W2^T [d_model rows, d_ff] in the
 *           same tiled form
 * The expert FFN is the SwiGLU form y = (silu(x W1) * (x W3)) W2 ([P2]
 * section 2: each expert is an FFN).  A weight tile is one contiguous 16 KB
 * block, so the GEMMs stream weights with plain bulk copies.  This is a
 * load-time step, outside the per-batch path; the caller may free W1/W3/W2
 * afterwards. */
MOE_API int moe_pack_weights(const moe_dims* dims, const moe_bf16* W1, const moe_bf16* W3,
                     const moe_bf16* W2, moe_bf16* W13p, moe_bf16* W2p, void* stream);

/* Step 1+2: router logits, top-K and renormalisation ([P2] sections 1.2, 2
 * and 2.1; [P3] sections 1 and 1.2).
 *   x          [T, d_model] bf16 tokens
 *   Wr         [d_model, E] bf16 router weight
 *   bias       [E] fp32 or NULL: added (in fp32) to the logits before
 *              selection; the weights use the biased logits too
 *   logits     [T, E] fp32 out (unbiased logits) or NULL
 *   topk_idx   [T, K] int32 out: selected experts, descending biased logit,
 *              equal values ranked by lower expert index
 *   topk_w     [T, K] fp32 out: softmax over the K selected (biased) logits
 *   prob_mean  [E] fp32 out or NULL: P_i = mean over tokens of the full
 *              softmax of the unbiased logits ([P2] section 1.2)
 *   ws         workspace of at least ws_bytes = moe_workspace_size bytes */
MOE_API int moe_route(const moe_dims* dims, const moe_bf16* x, const moe_bf16* Wr, const float* bias,
              float* logits, int32_t* topk_idx, float* topk_w, float* prob_mean,
              void* ws, size_t ws_bytes, void* stream);

/* Step 2 alone, from given fp32 logits [T, E] (same outputs and rules as
 * moe_route).  Lets the selection be checked bit for bit on logits both
 * sides share.  prob_mean may be NULL. */
MOE_API int moe_route_from_logits(const moe_dims* dims, const float* logits, const float* bias,
                          int32_t* topk_idx, float* topk_w, float* prob_mean,
                          void* ws, size_t ws_bytes, void* stream);

/* Step 3: dispatch ([P2] section 2.1: group by expert via sort and cumsum;
 * section 3.1: capacity drop).
 *   topk_idx  [T, K] int32 in: entries should lie in [0, E).  An entry
 *             outside that range is never used as an address: its slot is
 *             skipped (not counted, inv = -1, no row) and the workspace
 *             status flag records MOE_EINDEX (moe_get_device_status).  The
 *             router writes K distinct experts per token; a token that lists
 *             an expert twice is treated as two assignments, ranked in slot
 *             order.
 *   x         [T, d_model] bf16 in, or NULL to skip the row gather
 *   counts    [E] int32 out: selections per expert before drops
 *   kept      [E] int32 out: min(counts, C)
 *   offsets   [E+1] int32 out: exclusive cumsum of kept (offsets[E] = N_kept)
 *   inv       [T, K] int32 out: row of (t, k) in x_perm, or -1 if dropped
 *   src       [T*K] int32 out: token of each row (rows >= N_kept untouched)
 *   x_perm    [T*K, d_model] bf16 out (rows >= N_kept untouched), or NULL
 *   n_dropped [1] int32 out or NULL
 * The rank of (t, k) within its expert is the number of assignments
 * (t', k') before it in token-major order that chose the same expert (for
 * distinct experts per token: the tokens t' < t that chose it); rows are
 * expert-major, token-ascending. */
MOE_API int moe_permute(const moe_dims* dims, const int32_t* topk_idx, const moe_bf16* x,
                int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* inv, int32_t* src,
                moe_bf16* x_perm, int32_t* n_dropped, void* ws, size_t ws_bytes, void* stream);

/* Step 3 for callers that cannot allocate: the same dispatch as
 * moe_permute (same arguments, outputs and ordering, bit for bit) with no
 * workspace argument.  Some callers cannot hand the library device memory:
 * a plugin or runtime that owns every device buffer and exposes no
 * allocator to its extensions, or a serving loop where an allocation (or
 * the device synchronisation an allocator may trigger) is not allowed
 * between steps.  This entry point allocates nothing and calls no
 * allocating routine.
 *
 * Its scratch (the per-block histogram, ceil(T / 256) * E int32 values) is
 * a fixed 256 KB array inside the library, held by every GPU that loads the
 * library until the process exits.  Batches with ceil(T / 256) * E > 65536
 * are rejected with MOE_ESCRATCH (e.g. T <= 65536 tokens at E = 256).
 * Batches of at most 1024 tokens need no scratch at all.
 *
 * The first call on each device looks up the array's device address (a
 * one-time host-side set-up, with that device current), so make that first
 * call before any stream capture.  All calls share the array and it keeps
 * the last call's contents; every value a call reads is written earlier in
 * the same call, so no clearing is needed, but calls whose work overlaps on
 * the same GPU (for example on two streams) race on it: serialise them.
 * The looked-up address is kept for the life of the process, so do not use
 * this entry point across a cudaDeviceReset (or any other teardown of the
 * device's primary context) in the same process.
 *
 * An out-of-range expert index is skipped as in moe_permute, but with no
 * workspace there is no status flag to record it: validate topk_idx first
 * where it does not come from moe_route.
 *
 * There is no counterpart of this entry point on the source pages; it
 * exists for the callers described above. */
MOE_API int moe_permute_noalloc(const moe_dims* dims, const int32_t* topk_idx, const moe_bf16* x,
                                int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* inv,
                                int32_t* src, moe_bf16* x_perm, int32_t* n_dropped, void* stream);

/* Step 4: grouped SwiGLU expert FFN on the rows of each expert ([P2]
 * section 2 step 3; section 2.2: experts only see their own tokens).
 *   x_perm   [T*K, d_model] bf16 in (rows 0..offsets[E]-1 are used)
 *   offsets  [E+1] int32 in (device; read by the kernels, never by the host)
 *   W13p, W2p packed weights from moe_pack_weights
 *   h        [T*K, d_ff] bf16 out: silu(X W1) * (X W3) rounded to bf16
 *   y_perm   [T*K, d_model] fp32 out: h W2, fp32 accumulation */
MOE_API int moe_expert_ffn(const moe_dims* dims, const moe_bf16* x_perm, const int32_t* offsets,
                   const moe_bf16* W13p, const moe_bf16* W2p, moe_bf16* h, float* y_perm,
                   void* ws, size_t ws_bytes, void* stream);

/* Step 5: combine ([P2] section 2 step 4 and section 2.3: weighted sum back
 * in token order; section 2.2: unselected experts add nothing).
 *   y[t] = sum_{k=0..K-1, inv[t,k] >= 0} topk_w[t,k] * y_perm[inv[t,k]]
 * summed in k order in fp32 (fused multiply-adds); a dropped slot adds
 * nothing and the remaining weights are not renormalised.
 *   y           [T, d_model] out: fp32 when y_is_bf16 == 0; bf16 otherwise,
 *               each value the round-to-nearest-even of the fp32 sum (the
 *               activation type an inference engine passes on; the fp32 form
 *               is the parity output). */
MOE_API int moe_combine(const moe_dims* dims, const float* y_perm, const int32_t* inv,
                const float* topk_w, void* y, int y_is_bf16, void* stream);

/* Load statistics ([P2] section 1.2): f_i = counts_i / (T K),
 * P_i = prob_mean_i, aux = E * sum_i f_i P_i.  Any output may be NULL. */
MOE_API int moe_load_stats(const moe_dims* dims, const int32_t* counts, const float* prob_mean,
                   float* f, float* aux, void* stream);

/* Aux-free bias update ([P3] section 1.2): for each expert, b -= alpha if
 * counts*E > T*K (above the target load T*K/E), b += alpha if below,
 * unchanged if equal.  One fp32 add per expert; bias [E] fp32 in/out. */
MOE_API int moe_bias_update(const moe_dims* dims, const int32_t* counts, float alpha, float* bias,
                    void* stream);

/* Optional outputs of moe_layer_forward: device pointers, each may be NULL
 * (the value then stays in the workspace). */
typedef struct moe_layer_outputs {
    int32_t* topk_idx;  /* [T, K] */
    float* topk_w;      /* [T, K] */
    float* logits;      /* [T, E] unbiased */
    int32_t* counts;    /* [E] before drops */
    int32_t* kept;      /* [E] */
    int32_t* offsets;   /* [E+1] */
    int32_t* inv;       /* [T, K] */
    int32_t* n_dropped; /* [1] */
    float* f;           /* [E] */
    float* P;           /* [E] */
    float* aux;         /* [1] */
    /* Caller-created CUDA events (cudaEvent_t), or NULL.  When set, the
     * layer records, on `stream`: [0] before routing, [1] after routing,
     * [2] after dispatch, [3] after the expert GEMMs (gate/up and down run
     * in one launch), [4] after combine, [5] after statistics and the bias
     * update (these run in one extra CTA of the combine launch, so [4] and
     * [5] mark the same point).  For per-stage timing. */
    void* const* stage_events; /* [MOE_NUM_STAGE_EVENTS] */
    /* Further router statistics ([P2] section 3.2), computed with P_i:
     * P_topk[i] = (1/T) * sum of the renormalised top-K weights w[t,k] of
     * the slots that chose expert i (the cheaper balance statistic that
     * counts only the selected experts' probabilities); aux_topk =
     * E * sum_i f_i P_topk[i]; z_loss = (1/T) * sum_t (log sum_e
     * exp(logits[t,e]))^2 over the unbiased logits (router z-loss). */
    float* P_topk;      /* [E] */
    float* aux_topk;    /* [1] */
    float* z_loss;      /* [1] */
} moe_layer_outputs;

#define MOE_NUM_STAGE_EVENTS 6

/* Which grouped-GEMM kernel moe_expert_ffn and moe_layer_forward launch for
 * these dims: 0 = single-CTA tiles (grouped_gemm_kernel), 1 = CTA-pair tiles
 * on tcgen05 cta_group::2 (grouped_gemm_2sm_kernel).  The choice depends on
 * the shape only.  Host only (at most a query of the current device's SM
 * count); MOE_EINVAL on bad dims. */
MOE_API int moe_ffn_kernel(const moe_dims* dims);

/* Number of kernel launches one moe_layer_forward call enqueues for these
 * dims and options (stats = P_i / f_i / aux requested, bias_update = bias
 * non-NULL and alpha != 0; neither adds a launch, both run in one extra CTA
 * of the combine launch).  Host only; < 0 on bad dims. */
MOE_API int moe_layer_launch_count(const moe_dims* dims, int stats, int bias_update);

/* The whole layer: route -> permute -> expert FFN -> combine (-> stats, bias
 * update), all enqueued on `stream` with no host synchronisation.
 *   x [T, d_model] bf16, Wr [d_model, E] bf16, W13p/W2p from moe_pack_weights
 *   bias  [E] fp32 or NULL; if non-NULL and alpha != 0 it is updated in place
 *         after routing (so the routing of this call uses the old value)
 *   y     [T, d_model] out: fp32, or bf16 with y_is_bf16 != 0 (RNE of the
 *         fp32 result, as in moe_combine)
 *   out   optional extra outputs (NULL = none)
 * [P1] section 2 lists the same sequence: score, select, dispatch, expert
 * FFN, gather back. */
MOE_API int moe_layer_forward(const moe_dims* dims, const moe_bf16* x, const moe_bf16* Wr, float* bias,
                      float alpha, const moe_bf16* W13p, const moe_bf16* W2p, void* y, int y_is_bf16,
                      const moe_layer_outputs* out, void* ws, size_t ws_bytes, void* stream);

/* Chunked MoE ([P2] section 4.3: prefill tokens go through the MoE step in
 * chunks, so the expert stage never holds the whole batch and the memory
 * peak drops).  The same layer as moe_layer_forward for dims without a
 * capacity (a capacity is defined over the whole batch: capacity_factor > 0
 * returns MOE_EUNSUPPORTED):
 *   1. routing, statistics rows and top-K of all T tokens (small state);
 *   2. for each chunk of at most chunk_tokens consecutive tokens: dispatch,
 *      both expert GEMMs and the combine into y's rows of that chunk, in one
 *      chunk-sized workspace region;
 *   3. the whole batch's counts, f_i, P_i, aux, P_topk, aux_topk, z_loss and
 *      the bias update (with alpha != 0), from the whole batch's routing.
 * Routing, statistics and the bias update equal moe_layer_forward's; y rows
 * agree within floating-point reordering (the GEMM tiling follows the chunk's
 * groups).  out->offsets and out->inv are not written (rows are chunk-local);
 * out->kept receives the counts and out->n_dropped 0.  stage_events are
 * ignored.  ws: moe_chunked_workspace_size bytes (host query); d_model % 8 == 0. */
MOE_API int moe_chunked_workspace_size(const moe_dims* dims, int64_t chunk_tokens, size_t* bytes);
/* Kernel launches one moe_layer_forward_chunked call enqueues (host only;
 * < 0 on bad arguments). */
MOE_API int moe_layer_chunked_launch_count(const moe_dims* dims, int64_t chunk_tokens, int stats, int bias_update);
MOE_API int moe_layer_forward_chunked(const moe_dims* dims, int64_t chunk_tokens, const moe_bf16* x,
                                      const moe_bf16* Wr, float* bias, float alpha, const moe_bf16* W13p,
                                      const moe_bf16* W2p, void* y, int y_is_bf16, const moe_layer_outputs* out,
                                      void* ws, size_t ws_bytes, void* stream);

/* Expert parallelism ([P2] section 4.2; [P3] section 2.2: experts spread over
 * GPUs, token rows exchanged by all-to-all before and after the expert
 * computation).  The exchanges themselves are the caller's (NCCL through
 * torch.distributed in the Python layer); this call is the receiving rank's
 * one local step that has no single-GPU counterpart: it regroups the
 * received rows by local expert.
 *   n_ranks, E_local  ranks and experts per rank (n_ranks * E_local <= 2048)
 *   recv_counts  [n_ranks, E_local] int32 (device): rows received from each
 *                source rank for each local expert
 *   rows_in      [n_rows, d_model] bf16: the received rows, source-major (a
 *                source's rows for local expert 0, 1, .., in the order sent);
 *                n_rows = sum of recv_counts
 *   rows_out     [n_rows, d_model] bf16 out: expert-major; within an expert,
 *                by source rank, then in the order received
 *   offsets      [E_local + 1] int32 out: exclusive prefix of the per-expert
 *                row totals (the group offsets moe_expert_ffn takes)
 *   row_of       [n_rows] int32 out: the output row of each received row (to
 *                return results in the received order, e.g. moe_combine with
 *                K = 1, inv = row_of and unit weights, an exact copy)
 * d_model % 8 == 0; pointers 16-byte aligned. */
MOE_API int moe_ep_regroup(int n_ranks, int E_local, const int32_t* recv_counts, int64_t n_rows, int d_model,
                           const moe_bf16* rows_in, moe_bf16* rows_out, int32_t* offsets, int32_t* row_of,
                           void* stream);

/* Expert offloading ([P3] section 3.2: when the experts do not all fit in
 * GPU memory, keep some in host memory, group-wise quantized to INT4 to cut
 * the transfer volume, with an LRU cache of experts in GPU memory and
 * prefetching predicted from the routing history).  The cache's bookkeeping
 * (which expert sits in which slot) is the caller's; these calls move and
 * use the weights.
 *
 * INT4 format.  Codes follow the packed weight layout of moe_pack_weights:
 * for every 128-row x 64-column tile of an expert's packed matrix, 4096
 * bytes of 4-bit two's-complement codes (tile element i, in the tile's own
 * swizzled order, in the low nibble of byte i / 2 for even i, the high
 * nibble for odd i) and 128 fp32 scales, one per tile row.  A tile row's 64
 * elements form one group: 64 consecutive weights along the reduction axis
 * of one output column.  Per group, in fp32: s = amax / 7, q =
 * clamp(round_half_even(w / s), -8, 7) (correctly rounded divisions); an
 * all-zero group has s = 0.  The weight a GEMM uses is bf16(q * s), the
 * fp32 product rounded to nearest even.  Requires d_model % 64 == 0 and
 * d_ff % 64 == 0.
 *
 * moe_int4_bytes: sizes of the codes and scales of all E experts (host only).
 * moe_int4_pack: quantize W1, W3 [E, d_model, d_ff] and W2 [E, d_ff, d_model]
 *   (bf16, device) into q13/s13 and q2/s2 (device); a load-time step.
 * moe_int4_unpack: for each job j, expand expert job_expert[j]'s codes into
 *   cache slot job_slot[j] of W13c / W2c (each n_slots experts of packed
 *   weights, moe_packed_weight_bytes / E bytes per slot).  job_expert and
 *   job_slot are HOST arrays of n_jobs entries, checked against E and
 *   n_slots before any launch.  q13, s13, q2, s2 may be device memory or
 *   page-locked host memory mapped into the device's address space (read
 *   directly by the kernel over the host link: no staging copy); other host
 *   memory is refused with MOE_EUNSUPPORTED before any launch.
 * moe_expert_ffn_slots: moe_expert_ffn with the weights of expert e read
 *   from slot expert_slot[e] ([E] int32, device) of W13c / W2c.  The slot
 *   MOE_SLOT_SKIP skips expert e: its rows of h and y_perm are left as they
 *   are (a second call with the complementary table fills them, so the
 *   resident experts can run while the others are still loading).  Any other
 *   slot outside [0, n_slots) of an expert with rows is never used as an
 *   address: slot 0 is read instead and the workspace status flag records
 *   MOE_EINDEX (detail 8). */
#define MOE_SLOT_SKIP (-2)
MOE_API int moe_int4_bytes(const moe_dims* dims, size_t* q13_bytes, size_t* s13_bytes, size_t* q2_bytes,
                           size_t* s2_bytes);
MOE_API int moe_int4_pack(const moe_dims* dims, const moe_bf16* W1, const moe_bf16* W3, const moe_bf16* W2,
                          uint8_t* q13, float* s13, uint8_t* q2, float* s2, void* stream);
MOE_API int moe_int4_unpack(const moe_dims* dims, int n_jobs, const int32_t* job_expert, const int32_t* job_slot,
                            const uint8_t* q13, const float* s13, const uint8_t* q2, const float* s2, int n_slots,
                            moe_bf16* W13c, moe_bf16* W2c, void* stream);
MOE_API int moe_expert_ffn_slots(const moe_dims* dims, const moe_bf16* x_perm, const int32_t* offsets,
                                 const int32_t* expert_slot, int n_slots, const moe_bf16* W13c, const moe_bf16* W2c,
                                 moe_bf16* h, float* y_perm, void* ws, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
