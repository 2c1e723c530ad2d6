// Host-side interface between the library's translation units.
#pragma once
#include <cstdint>
#include <cstddef>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <atomic>

namespace moe {

using bf16 = __nv_bfloat16;

// ------------------------------------------------------------ grouped GEMM
enum GemmEpilogue : int {
    EPI_SWIGLU_BF16 = 0,  // D columns are interleaved (gate x16, up x16) blocks -> bf16 silu(g)*u
    EPI_F32 = 1,          // D stored as fp32
};

// One matrix product over all groups: out[rows of g] = tok[rows of g] . w[g]^T.
// Raise `func`'s dynamic shared memory limit to `bytes` on the current device,
// once per device (`done` holds one bit per device id < 64).  0, or -3 when
// the runtime refuses.
inline int smem_attr_once(const void* func, int bytes, std::atomic<unsigned long long>& done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -3;
    const unsigned long long bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return 0;
    if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return -3;
    if (bit) done.fetch_or(bit, std::memory_order_release);
    return 0;
}

// Programmatic dependent launch (a kernel may begin while the previous one
// on the stream drains; every kernel calls pdl_wait() before using earlier
// results, so it stays correct either way).  Off: with it on, the layer
// steps measured slower (DeepSeek-like layer 5.42 -> 5.29 ms per step,
// Qwen-like 0.57 -> 0.55 ms, Mixtral decode unchanged at 0.485 ms): the next
// kernel's CTAs became resident early and held SM resources while the
// current kernel still ran.  pdl_wait() returns at once without it.
constexpr bool kProgrammaticLaunch = false;

// Launch `kernel`, with programmatic stream serialization when
// kProgrammaticLaunch is set: it must call pdl_wait() before using the
// previous kernel's results (see ptx.cuh).
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
    cfg.numAttrs = kProgrammaticLaunch ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

struct GemmPhase {
    const bf16* tok;      // [tok_rows, Kdim] bf16, K contiguous
    int64_t tok_rows;
    const bf16* w;        // per group a K-major [N, Kdim] matrix in 128 x 64 swizzled tiles
                          // (tiled_offset), groups ceil(N/128) * ceil(Kdim/64) tiles apart
    int N;                // weight rows per group
    int N_store;          // output columns actually written (<= N)
    int Kdim;
    int ksplit;           // reduction split into partial slices (every tile of the phase)
    int epi;
    void* out;
    int64_t ldo;          // output row stride (elements)
    int64_t split_stride; // elements between partial slices
};

struct GemmLaunch {
    int G;
    // Groups: rows group_off[g] .. group_off[g+1]-1 of the token matrices
    // (device array), or a single group of dense_rows rows when NULL.
    const int32_t* group_off;
    int64_t dense_rows;
    int64_t max_group_rows;  // host-known upper bound on any group's rows
    int swap_max_rows;       // groups with at most this many rows use weight-major tiles
    bool small_groups;       // mean group below 128 rows: keep token-major tiles narrow
    int bn_max;              // cap on token-major BN (0 = none)
    int nphase;              // 1, or 2: phase 1 of group g starts after phase 0 of g
    GemmPhase ph[2];
    int* status;             // device status word
    int* sched;              // gemm_sched_bytes(G) bytes, zero at launch
    // Bounded waits (0 = the default limit of ptx.cuh), and a value added to
    // the phase-1 readiness target (0 in production; a test of the timeout
    // paths makes the target unreachable).
    uint32_t wait_limit = 0;
    uint32_t dep_wait_limit = 0;
    int dep_extra = 0;
    // Expert cache: group g's weights are matrix w_slot[g] of the phase's
    // buffer, which holds w_slots matrices (nullptr: matrix g of G).
    const int32_t* w_slot = nullptr;
    int w_slots = 0;
};

// Staged fp32 output stores (gemm.cu): whether a phase qualifies, the rows
// of its output map, and the map itself (box {32, 32}, 128-byte swizzle).
bool out_map_ok(const GemmPhase& g);
uint64_t out_map_rows(const GemmPhase& g, int ksplit);
bool h_map_ok(const GemmPhase& g);
bool make_out_map(CUtensorMap* m, void* base, uint64_t rows, uint64_t cols, uint64_t ld, bool bf16_out);

// Test-only settings of the expert-GEMM launches (see moe_test_set_wait_limits
// in the header); all zero in production.
struct WaitSettings {
    uint32_t wait_limit, dep_wait_limit;
    int dep_never_ready;
};
WaitSettings wait_settings();

size_t gemm_sched_bytes(int G);
// CTA-pair (cta_group::2) kernel: 256-wide tiles, so both phases' widths
// must be multiples of 256.
bool gemm_2sm_supported(const GemmLaunch& L);
int launch_grouped_gemm_2sm(const GemmLaunch& L, cudaStream_t st);
int launch_grouped_gemm(const GemmLaunch& L, cudaStream_t st);
int num_sms();

// ------------------------------------------------------------ routing
int launch_route_fused(const bf16* x, const bf16* Wr, const float* bias, int64_t T, int d, int E,
                       int K, float* logits, int32_t* idx, float* w, float* prob_part, int nblocks,
                       cudaStream_t st);
int route_fused_supported(int d, int E);
int route_blocks(int64_t T);
// Top-K from the sum of nsplit partial logits slices [nsplit][T][E] (slice
// order); logits_out (or nullptr) receives the sums.
int launch_topk_from_logits(const float* logits, int nsplit, int64_t split_stride, float* logits_out,
                            const float* bias, int64_t T, int E, int K, int32_t* idx, float* w, float* prob_part,
                            int nblocks, cudaStream_t st);
// WrT: the router weight as a K-major [E_pad, d] matrix in 128 x 64 swizzled tiles.
int launch_transpose_router(const bf16* Wr, int d, int E, int E_pad, bf16* WrT, cudaStream_t st);
int launch_prob_finalize(const float* prob_part, int nblocks, int E, int64_t T, float* prob_mean,
                         cudaStream_t st);

// ------------------------------------------------------------ permutation
int permute_blocks(int64_t T);
int launch_permute(const int32_t* idx, const bf16* x, int64_t T, int d, int E, int K, int64_t C,
                   int32_t* block_hist, int32_t* counts, int32_t* kept, int32_t* offsets,
                   int32_t* inv, int32_t* src, bf16* x_perm, int32_t* n_dropped, int32_t* zero_out,
                   int zero_count, int* status, cudaStream_t st);

// ------------------------------------------------------------ combine / stats
// Work folded into the combine launch as one extra CTA: the load statistics
// (P_i from the router's per-block sums, f_i, aux) and the aux-free bias
// update.  Both need only routing results, which are complete when the
// combine starts.
struct StatsTail {
    const float* part;      // router per-block rows [nblocks, 2 E + 1]: probability sums, top-K weight
                            // sums, squared log-sum-exp sum; nullptr: no statistics
    int nblocks;
    const int32_t* counts;  // nullptr: no tail CTA at all
    float* P;               // required with part
    float* f;               // may be nullptr
    float* aux;             // may be nullptr
    float* P_topk;          // may be nullptr
    float* aux_topk;        // may be nullptr
    float* z_loss;          // may be nullptr
    float* bias;            // updated in place when non-null and alpha != 0
    float alpha;
    int E;
    int64_t T;              // tokens the statistics cover (0: the combine's own T)
};

// y [T, d]: fp32, or bf16 (each value RNE of the fp32 sum) when y_bf16.
int launch_combine(const float* y_perm, int nsplit, int64_t split_stride, const int32_t* inv,
                   const float* w, int64_t T, int d, int K, void* y, bool y_bf16, cudaStream_t st,
                   const StatsTail* tail = nullptr);
// dst[e] = (first ? 0 : dst[e]) + src[e] for e < E (a batch's counts from its chunks').
int launch_accumulate_counts(int32_t* dst, const int32_t* src, int E, bool first, cudaStream_t st);
int launch_reduce_splits(const float* part, int nsplit, int64_t split_stride, const int32_t* offsets,
                         int E, int d, float* y_perm, cudaStream_t st);
int launch_stats(const int32_t* counts, const float* prob_mean, int64_t T, int E, int K,
                 float* f, float* aux, const float* alpha_bias_unused, cudaStream_t st);
int launch_count(int64_t T);  // kernels launch_permute enqueues before the row gather
// The layer's small-batch dispatch: counts, ranks and the row gather in one
// launch (results identical to launch_permute's).
bool dispatch_gather_fused_supported(int64_t T, int E, int K);
int launch_dispatch_gather_small(const int32_t* idx, const bf16* x, int64_t T, int d, int E, int K, int64_t C,
                                 int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* inv, int32_t* src,
                                 bf16* x_perm, int32_t* n_dropped, int32_t* zero_out, int zero_count,
                                 int* status, cudaStream_t st);
int64_t permute_static_max_hist();
int launch_permute_static(const int32_t* idx, const bf16* x, int64_t T, int d, int E, int K, int64_t C,
                          int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* inv, int32_t* src,
                          bf16* x_perm, int32_t* n_dropped, cudaStream_t st);
int launch_bias_update(const int32_t* counts, int64_t T, int E, int K, float alpha, float* bias,
                       cudaStream_t st);

// ------------------------------------------------------------ expert parallelism
int ep_regroup_max_blocks();
int launch_ep_regroup(const int32_t* counts, int G, int El, int64_t n, const bf16* in, int d, bf16* out,
                      int32_t* offsets, int32_t* row_of, cudaStream_t st);

// ------------------------------------------------------------ offloaded experts (INT4)
void int4_sizes(int E, int d, int f, size_t* q13, size_t* s13, size_t* q2, size_t* s2);
int launch_int4_pack(const bf16* W1, const bf16* W3, const bf16* W2, int E, int d, int f, uint8_t* q13, float* s13,
                     uint8_t* q2, float* s2, cudaStream_t st);
int launch_int4_unpack(int n_jobs, const int32_t* job_expert, const int32_t* job_slot, int d, int f,
                       const uint8_t* q13, const float* s13, const uint8_t* q2, const float* s2, bf16* W13c,
                       bf16* W2c, cudaStream_t st);

// ------------------------------------------------------------ packing
int launch_pack(const bf16* W1, const bf16* W3, const bf16* W2, int E, int d, int f, bf16* W13p,
                bf16* W2p, cudaStream_t st);
size_t packed_w13_bytes(int E, int d, int f);
size_t packed_w2_bytes(int E, int d, int f);

}  // namespace moe
