// Grouped GEMM for large expert groups on CTA pairs (tcgen05 cta_group::2).
//
// Same computation as gemm.cu ("MoE computation notes", cf-1.com/news/5905749,
// section 2.1: one matrix product per expert group), for launches where every
// group is large enough for token-major tiles (prefill-sized batches).  Each
// cluster of two CTAs owns one 256 x 256 output tile at a time:
//   - CTA r loads token rows m0 + 128 r .. +127 (the M half of A) and weight
//     rows n0 + 128 r .. +127 (the N half of B) into its own shared memory;
//   - the leader (rank 0) issues one 256 x 256 x 16 tcgen05.mma per k-step,
//     which reads A and B halves from both CTAs and accumulates rows
//     128 r .. of D into CTA r's TMEM;
//   - each CTA's epilogue drains its own TMEM rows.
// Per CTA and k-block this moves 32 KB into shared memory for the FLOPs that
// a single-CTA 128 x 256 tile needed 48 KB for, so the ring is deeper and the
// weight tile is fetched by half as many CTAs.
//
// Small groups use weight-major pair tiles instead: the MMA's M side is 256
// weight rows (CTA r loads the 128-row weight tile n0 + 128 r), its N side
// the group's tokens, of which each CTA loads half.  Against single-CTA
// weight-major tiles this halves the token traffic and the MMA instructions
// per SM.  Where the phase has tiles to spare, a weight-major pair tile
// covers two such 256-row sub-tiles that share one token load, issuing two
// MMAs into two TMEM accumulators, which halves the token traffic again.
// The down projection's reduction can be split as in gemm.cu.
//
// Where weight-major tiles are enabled (mixed group sizes), a token-major
// group's last chunk of at most 128 rows takes a 128-row tile instead of a
// 256-row one: tcgen05.mma cta_group::2 with M = 128, each CTA loading 64
// token rows; a CTA's accumulator then holds its 64 rows in TMEM lanes 0-63
// for output columns 0-127 and in lanes 64-127 for columns 128-255.  This is
// the kHalfTiles instance of the kernel.
//
// Two tile queues.  Token-major tiles (large groups) and weight-major tiles
// (small groups) are numbered in separate queues, each phase 0 then phase 1
// in group order, with a tile counter each.  At kernel start every CTA
// computes both queues' tiles and the same split of the pairs between them
// (split_pairs: in proportion to the queues' work); a pair serves one queue
// with a ring shaped for it: token-major pairs put two k-blocks in each of
// three stages, weight-major pairs one k-block in each of five or more.  So
// the tensor-bound and the stream-bound tiles of a mixed launch run side by
// side, each kind with its better ring (DeepSeek-shaped layer: expert GEMMs
// 5.13-5.17 -> 4.90-4.94 ms on one box).  A launch with one kind of tile
// puts every pair on its queue.
//
// fp32 output of token-major tiles (the down projection) leaves through a
// 4 KB staging buffer per epilogue warp and one TMA tile store per 32 x 32
// block, as in gemm.cu; the buffers sit after the token-major ring (two per
// warp where they fit, else one).
//
// Stage layout (per CTA and k-block): token-major tiles put their 128 token
// rows at 0 and their 128 weight rows at 16 KB; weight-major tiles put
// weight sub-tile j at 16 KB j and their token rows at xoff.  A stage holds
// one or two such k-blocks (kpb) that complete on one barrier phase.
//
// Pair protocol (barriers live in each CTA; "leader" means rank 0's copy):
//   full[s]    leader only: the leader registers the pair's bytes, both CTAs'
//              TMA loads complete on it
//   empty[s]   both CTAs: the leader's MMA commit arrives on both
//   tfull[b]   both CTAs: the leader's MMA commit arrives on both
//   tempty[b]  leader: all 8 epilogue warps of the pair arrive
//   ring       the leader claims tiles and writes them into both CTAs' rings;
//              the pair's 10 consumers free a slot on the leader's rempty
// Every wait is bounded.  No TMA multicast is used.
//
// Failure handling.  A wait that runs out records its code in the status
// word and raises the abort flag of BOTH CTAs (the peer's by a store into
// its shared memory), so every role of the pair stops within one poll
// interval.  Before the pair passes its final cluster barrier, every copy
// either CTA issued must have landed.  The peer's copies complete on the
// leader's full[] barriers, which the leader alone arms, so the leader
// reconciles with the peer: once its producer stops, the peer reports how
// many stage uses it issued and their byte counts; the leader arms the uses
// the peer issued beyond its own (expecting the peer's bytes only),
// completes by hand the peer's half of the uses it armed that the peer never
// issued, and then waits for every stage's last phase.  The MMA issuer waits
// for its last MMAs before TMEM is freed.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kBK = 64;
constexpr int kThreads = 192;
constexpr uint32_t kHalf = 128u * 128u;  // 128 rows x 64 bf16 = 16 KB
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxGroups = 256;
constexpr int kRing = 8;

struct Phase2 {
    const bf16* w;  // packed weights (read only for the L2 prefetch; loads go through the tensor map)
    int N, k_blocks, epi;
    int64_t nb;  // 128-row weight blocks per group
    int ksplit, kb_per_split;  // reduction split (every tile of the phase)
    int wt;                    // weight-major tiles: 256-row weight sub-tiles per pair tile (1 or 2)
    void* out;
    int64_t ldo;
    int64_t split_stride;
    int tma_out;         // fp32 token-major tiles store full 32-row slabs by TMA (Maps2::out)
    int64_t split_rows;  // rows between partial slices in the output map
};

struct Args2 {
    const int32_t* group_off;
    int G;
    int nphase;
    int dep;
    int swap_max_rows;  // groups with at most this many rows take weight-major pair tiles
    int BNs;            // weight-major: tokens per pair tile (multiple of 32, <= 128)
    Phase2 ph[2];
    // Ring of a pair serving the token-major queue [0] or the weight-major queue [1]
    int stages[2];
    uint32_t stage_bytes[2];  // per k-block and CTA
    int kpb[2];               // k-blocks per stage (1 or 2)
    size_t ring_bytes;        // shared memory of the larger ring (token-major: with its output staging)
    int stg_bufs;             // token-major pairs: 4 KB output staging buffers per epilogue warp (0: none)
    uint32_t stg_off;         // offset of the staging buffers (after the token-major ring)
    uint32_t xoff;            // weight-major tiles: offset of the token rows in a k-block
    int* status;
    int* sched;  // [0] token-major tile counter, [1 + g] phase-0 stores of group g, [G + 1] weight-major tile counter
    uint32_t wait_limit;      // polls of a bounded mbarrier or drain wait
    uint32_t dep_wait_limit;  // polls of the phase-1 readiness wait
    int dep_extra;            // added to the phase-1 readiness target (0; a test makes it unreachable)
    int prefetch_kb;          // k-blocks of the first-round weight tiles pulled into L2 before the wait (0: none)
    const int32_t* w_slot;    // group -> weight matrix (expert cache slot), or nullptr
    int w_slots;
};

constexpr int kMaxStages = 16;
// The peer's report to the leader at the end of its producer loop (in the
// leader's shared memory): stage uses issued, done flag, and the bytes of
// its last use of each stage.
struct PeerReport {
    uint32_t uses;
    uint32_t done;
    uint32_t bytes[kMaxStages];
};

struct Maps2 {
    CUtensorMap tok[2];  // token rows, box 128, 128-byte swizzle
    CUtensorMap tok16[2];  // token rows, box 16, 128-byte swizzle (weight-major halves)
    CUtensorMap tok64[2];  // token rows, box 64, 128-byte swizzle (weight-major halves of >= 64 rows)
    CUtensorMap w[2];    // tiled weights as [rows, 64], box 128, no swizzle (tiles are pre-swizzled)
    CUtensorMap out[2];  // fp32 output rows, box {32 columns, 32 rows}, 128-byte swizzle (phases with tma_out)
};

struct Tile2 {
    int phase, g, swap;
    int64_t row0;  // first token row of the pair's tile
    int rows;      // valid token rows (<= 256 token-major, <= BNs weight-major)
    int n0;        // first weight row (multiple of 256)
    int kb0, kb1, split;
    int wt;    // weight sub-tiles (weight-major tiles), else 1
    int half;  // token-major tile of 128 rows (M = 128: 64 token rows per CTA)
};

// ---- cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(addr), "r"(rank));
    return out;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void remote_arrive(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void remote_store(uint32_t cluster_addr, int v) {
    asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_cluster(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.cluster.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}
__device__ __forceinline__ void fence_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
                 : "memory");
}
// TMA tile load into this CTA's shared memory, completing on the leader's barrier.
__device__ __forceinline__ void tma_load_pair(const CUtensorMap* map, void* smem_dst, uint32_t leader_bar, int32_t x,
                                              int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(leader_bar),
          "l"(policy)
        : "memory");
}
__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}
// Arrive on the barrier at this offset in both CTAs of the pair once all
// previously issued pair MMAs are complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(smem_u32(bar)), "h"(static_cast<uint16_t>(3))
                 : "memory");
}

// A bounded wait whose failure (its own, or an abort seen) also raises the
// other CTA's abort flag.
__device__ __forceinline__ bool pwait(uint64_t* bar, uint32_t parity, const Args2& a, int code,
                                      volatile int* abort_flag, uint32_t peer_abort) {
    if (mbar_wait(bar, parity, a.status, code, abort_flag, a.wait_limit)) return true;
    *abort_flag = 1;
    remote_store(peer_abort, 1);
    return false;
}

__device__ __forceinline__ bool swaps2(const Args2& a, int64_t rows) { return rows <= a.swap_max_rows; }

__device__ __forceinline__ int tiles_of2(const Args2& a, int p, int64_t rows) {
    if (rows <= 0) return 0;
    const Phase2& ph = a.ph[p];
    if (!swaps2(a, rows)) return static_cast<int>(((rows + 255) / 256) * (ph.N / 256) * ph.ksplit);
    return static_cast<int>(((rows + a.BNs - 1) / a.BNs) * (ph.N / (256 * ph.wt)) * ph.ksplit);
}

// Tiles of a group of `rows` rows in queue q (0: token-major, 1: weight-major).
__device__ __forceinline__ int tiles_in_queue(const Args2& a, int q, int p, int64_t rows) {
    return (swaps2(a, rows) ? 1 : 0) == q ? tiles_of2(a, p, rows) : 0;
}

// Cost of a token-major k-block relative to a weight-major k-block of one
// 256-row weight sub-tile when the two kinds run side by side on separate
// pairs (DeepSeek-shaped layer, clock-counter instrumentation: 813 against
// 600 cycles; the token-major loads then wait behind the weight stream).
constexpr float kTokenMajorCost = 1.35f;

// Pairs serving the token-major queue.  Token-major tiles are bound by the
// tensor pipe, weight-major tiles by the weight stream, and the two kinds run
// side by side on separate pairs, each with its own ring (token-major pairs
// use two k-blocks per stage).  The pairs are split in proportion to the
// queues' work: k-blocks per 256-row weight (sub-)tile, token-major ones
// weighted by kTokenMajorCost, of which the k-blocks of 128-row tiles
// (half_kb) count three quarters (their operand bytes per k-block).  An empty
// queue gets no pair.
__device__ __forceinline__ int split_pairs(const Args2& a, const int* tstart_all, int npairs, int half_kb) {
    const int G = a.G;
    float w[2] = {0.f, 0.f};
    for (int q = 0; q < 2; ++q)
        for (int p = 0; p < a.nphase; ++p) {
            const int* ts = tstart_all + (2 * q + p) * (G + 1);
            const float tiles = static_cast<float>(ts[G] - ts[0]);
            w[q] += tiles * static_cast<float>(a.ph[p].kb_per_split) * static_cast<float>(q == 1 ? a.ph[p].wt : 1);
        }
    w[0] = (w[0] - 0.25f * static_cast<float>(half_kb)) * kTokenMajorCost;
    if (w[0] <= 0.f) return 0;
    if (w[1] <= 0.f || npairs < 2) return npairs;
    int x = __float2int_rn(static_cast<float>(npairs) * w[0] / (w[0] + w[1]));
    return x < 1 ? 1 : (x > npairs - 1 ? npairs - 1 : x);
}

template <bool kHalfTiles>
__device__ __forceinline__ Tile2 decode2(const Args2& a, int tile, const int* tstart, const int64_t* off) {
    Tile2 t;
    const int G = a.G;
    int p = 0;
    if (a.nphase > 1 && tile >= tstart[G]) p = 1;
    const int* ts = tstart + p * (G + 1);
    int lo = 0, hi = G;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ts[mid] <= tile) lo = mid; else hi = mid;
    }
    const Phase2& ph = a.ph[p];
    t.phase = p;
    t.g = lo;
    const int local = tile - ts[lo];
    const int64_t base = off[lo];
    const int64_t rows_g = off[lo + 1] - base;
    t.swap = swaps2(a, rows_g) ? 1 : 0;
    t.wt = t.swap ? ph.wt : 1;
    // reduction split fastest, then the token chunk (the weight tile is
    // reused from L2), then the weight tile
    const int chunk = t.swap ? a.BNs : 256;
    const int nch = static_cast<int>((rows_g + chunk - 1) / chunk);
    const int sp = local % ph.ksplit;
    const int rest = local / ph.ksplit;
    const int c = rest % nch;
    const int64_t r0 = static_cast<int64_t>(c) * chunk;
    t.row0 = base + r0;
    t.rows = static_cast<int>(rows_g - r0 < chunk ? rows_g - r0 : chunk);
    t.half = (kHalfTiles && !t.swap && t.rows <= 128) ? 1 : 0;
    t.n0 = (rest / nch) * 256 * t.wt;
    t.kb0 = sp * ph.kb_per_split;
    t.kb1 = min(ph.k_blocks, t.kb0 + ph.kb_per_split);
    t.split = sp;
    return t;
}

__device__ __forceinline__ int ld_acquire2(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// silu(g) = g / (1 + e^-g) with the fast exp and divide intrinsics: the
// result is rounded to bf16 (8-bit mantissa) right after, far coarser than
// their few-ulp error.  For g < -87, e^-g overflows to inf and the quotient
// is 0, the limit of silu.
__device__ __forceinline__ float silu2(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

// kHalfTiles: token-major chunks of <= 128 rows take 128-row (M = 128) tiles.
// A separate instantiation because the 256-row-only kernel measured 1.5 %
// faster on launches without such chunks.
template <bool kHalfTiles>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_2sm_kernel(const __grid_constant__ Maps2 maps, const Args2 a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int Smax = a.stages[0] > a.stages[1] ? a.stages[0] : a.stages[1];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.ring_bytes);
    uint64_t* empty = full + Smax;
    uint64_t* tfull = empty + Smax;
    uint64_t* tempty = tfull + 2;
    uint64_t* rfull = tempty + 2;
    uint64_t* rempty = rfull + kRing;
    uint64_t* drain = rempty + kRing;
    int* ring = reinterpret_cast<int*>(drain + 1);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring + kRing);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int64_t* off = reinterpret_cast<int64_t*>(tmem_slot + 2);
    int* tstart_all = reinterpret_cast<int*>(off + a.G + 1);  // [queue][phase][G + 1]
    int* role_split = tstart_all + 4 * (a.G + 1);            // pairs serving the token-major queue
    PeerReport* report = reinterpret_cast<PeerReport*>(role_split + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = a.G;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Smax; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        for (int r = 0; r < kRing; ++r) {
            mbar_init(&rfull[r], 1);
            mbar_init(&rempty[r], 10);  // leader: MMA + 4 epilogue warps; peer: producer + 4 epilogue warps
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        report->uses = 0;
        report->done = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0)
        for (int p = 0; p < a.nphase; ++p) {
            tma_prefetch_desc(&maps.tok[p]);
            tma_prefetch_desc(&maps.tok16[p]);
            tma_prefetch_desc(&maps.tok64[p]);
            tma_prefetch_desc(&maps.w[p]);
        }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    // Weight tiles depend on no earlier kernel.  Under programmatic launch,
    // while the router and the dispatch finish, pull the first k-blocks of
    // the first round of weight-major tiles into L2: cluster c takes tile c
    // of the first phase, as if every group had one token chunk (the decode
    // case); whichever cluster claims that tile later finds them in L2.  A
    // hint only: no result depends on it, and every address lies inside the
    // packed weights.
    if (a.prefetch_kb > 0 && warp == 0 && lane == 0) {
        const Phase2& p0 = a.ph[0];
        const int tpg = (p0.N / (256 * p0.wt)) * p0.ksplit;  // tiles per group with one token chunk
        const int tile = static_cast<int>(blockIdx.x >> 1);
        const int g = tile / tpg;
        if (g < G) {
            const int local = tile - g * tpg;
            const int kb0 = (local % p0.ksplit) * p0.kb_per_split;
            const int kb1 = min(p0.k_blocks, min(kb0 + p0.kb_per_split, kb0 + a.prefetch_kb));
            const int n0 = (local / p0.ksplit) * 256 * p0.wt;
            const int64_t wblk0 = static_cast<int64_t>(g) * p0.nb + (n0 + 128 * static_cast<int>(rank)) / 128;
            for (int j = 0; j < p0.wt; ++j)
                for (int kb = kb0; kb < kb1; ++kb)
                    prefetch_l2(p0.w + ((wblk0 + 2 * j) * p0.k_blocks + kb) * 8192, 16384u);
        }
    }
    // group offsets, scheduler words and token rows come from earlier kernels
    pdl_wait();
    // Under programmatic launch (kProgrammaticLaunch, off by default) the
    // next kernel may launch once every CTA has run out of tiles (its
    // producer sees the end marker, below), so its CTAs do not sit resident
    // on the SMs through the whole launch, only through the last tiles.
    for (int g = threadIdx.x; g <= G; g += blockDim.x) off[g] = static_cast<int64_t>(a.group_off[g]);
    __syncthreads();
    // rows of group g in this launch (0 for a group the slot table skips)
    auto rows_of = [&](int g) -> int64_t { return group_skipped(a.w_slot, g) ? 0 : off[g + 1] - off[g]; };
    if (warp == 0) {
        // Tile numbering per queue (0: token-major groups, 1: weight-major
        // groups), phase 0 then phase 1, groups in order; each lane scans a
        // contiguous span of groups.
        const int span = (G + 31) / 32;
        const int g0 = min(G, lane * span), g1 = min(G, g0 + span);
        for (int q = 0; q < 2; ++q) {
            int carry = 0;
            for (int p = 0; p < a.nphase; ++p) {
                int sum = 0;
                for (int g = g0; g < g1; ++g) sum += tiles_in_queue(a, q, p, rows_of(g));
                int incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int v = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += v;
                }
                int run = carry + incl - sum;
                int* ts = tstart_all + (2 * q + p) * (G + 1);
                for (int g = g0; g < g1; ++g) {
                    ts[g] = run;
                    run += tiles_in_queue(a, q, p, rows_of(g));
                }
                const int tot = __shfl_sync(0xffffffffu, incl, 31);
                if (lane == 0) ts[G] = carry + tot;
                carry += tot;
            }
        }
        // k-blocks of the token-major queue's 128-row tiles (chunks of <= 128 rows)
        int half_kb = 0;
        if (kHalfTiles)
            for (int g = g0; g < g1; ++g) {
                const int64_t rows = rows_of(g);
                const int64_t rem = rows & 255;
                if (rows > 0 && !swaps2(a, rows) && rem > 0 && rem <= 128)
                    for (int p = 0; p < a.nphase; ++p)
                        half_kb += (a.ph[p].N / 256) * a.ph[p].ksplit * a.ph[p].kb_per_split;
            }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) half_kb += __shfl_xor_sync(0xffffffffu, half_kb, o);
        __syncwarp();
        if (lane == 0) *role_split = split_pairs(a, tstart_all, static_cast<int>(gridDim.x >> 1), half_kb);
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // this pair's queue and ring (both CTAs of a pair compute the same)
    const int queue = static_cast<int>(blockIdx.x >> 1) < *role_split ? 0 : 1;
    const int S = a.stages[queue];
    const int kpb = a.kpb[queue];
    const uint32_t sbytes = a.stage_bytes[queue];
    const int* tstart = tstart_all + 2 * queue * (G + 1);
    const int total = tstart[(a.nphase - 1) * (G + 1) + G];
    int* const counter = a.sched + (queue == 0 ? 0 : G + 1);
    const uint32_t leader_rempty0 = mapa_shared(smem_u32(rempty), 0);
    const uint32_t leader_tempty0 = mapa_shared(smem_u32(tempty), 0);
    const uint32_t leader_full0 = mapa_shared(smem_u32(full), 0);
    const uint32_t peer_abort = mapa_shared(smem_u32(const_cast<int*>(abort_flag)), rank ^ 1u);

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------- scheduler (leader) + producer (both)
            const uint64_t pol_first = policy_evict_first();
            const uint64_t pol_last = policy_evict_last();
            uint32_t s = 0, ph = 0, r = 0, rph = 0;
            bool ok = true;
            uint32_t uses = 0;                 // stage uses this CTA issued (armed, on the leader)
            uint32_t use_bytes[kMaxStages];    // bytes of the pair's (leader) or own (peer) last use per stage
            int next = leader ? atomicAdd(counter, 1) : 0;
            const uint32_t peer_ring = mapa_shared(smem_u32(ring), 1);
            const uint32_t peer_rfull = mapa_shared(smem_u32(rfull), 1);
            while (ok) {
                int tile;
                if (leader) {
                    tile = next < total ? next : -1;
                    if (tile >= 0) next = atomicAdd(counter, 1);
                    if (!pwait(&rempty[r], rph ^ 1u, a, DEV_TIMEOUT_PRODUCER_EMPTY, abort_flag, peer_abort)) {
                        ok = false;
                        break;
                    }
                    ring[r] = tile;
                    remote_store(peer_ring + 4u * r, tile);
                    mbar_arrive(&rfull[r]);
                    remote_arrive(peer_rfull + 8u * r);
                } else {
                    if (!pwait(&rfull[r], rph, a, DEV_TIMEOUT_MMA_FULL, abort_flag, peer_abort)) {
                        ok = false;
                        break;
                    }
                    tile = ring[r];
                    remote_arrive(leader_rempty0 + 8u * r);
                }
                if (++r == kRing) { r = 0; rph ^= 1u; }
                if (tile < 0) {  // the end marker
                    pdl_trigger();
                    break;
                }
                const Tile2 t = decode2<kHalfTiles>(a, tile, tstart, off);
                const Phase2& pa = a.ph[t.phase];
                if (t.phase == 1 && a.dep) {
                    const int need = 8 * (tstart[t.g + 1] - tstart[t.g]) + a.dep_extra;
                    uint32_t i = 0;
                    while (ld_acquire2(&a.sched[1 + t.g]) < need) {
                        if (*abort_flag) {
                            ok = false;
                            break;
                        }
                        if (++i > a.dep_wait_limit) {
                            atomicCAS(a.status, 0, DEV_TIMEOUT_DEPENDENCY);
                            *abort_flag = 1;
                            remote_store(peer_abort, 1);
                            ok = false;
                            break;
                        }
                        if (i > 64) __nanosleep(128);
                    }
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    if (!ok) break;
                }
                // this CTA's 128-row weight block of (sub-)tile j: rows n0 + 256 j + 128 rank
                const int wg = weight_slot(a.w_slot, a.w_slots, t.g, a.status);
                const int64_t wblk0 = static_cast<int64_t>(wg) * pa.nb + (t.n0 + 128 * static_cast<int>(rank)) / 128;
                // weight-major: the MMA's N is the tile's tokens rounded up to 16;
                // this CTA holds N / 2 of them (a multiple of 8), loaded in 64-row
                // boxes and the rest in 16-row boxes (fewer copies to issue; a
                // box at a 1 KB boundary lays rows out as the 16-row boxes would)
                const int half = t.swap ? ((t.rows + 15) / 16) * 8 : 0;
                const int n64 = half / 64;
                const int nb16 = (half - 64 * n64 + 15) / 16;
                // each CTA loads exactly half of the pair's bytes
                const uint32_t pair_bytes =
                    t.swap ? 2u * (static_cast<uint32_t>(t.wt) * kHalf + static_cast<uint32_t>(n64) * 8192u +
                                   static_cast<uint32_t>(nb16) * 2048u)
                           : (t.half ? 3u * kHalf : 4u * kHalf);
                for (int kb0 = t.kb0; kb0 < t.kb1; kb0 += kpb) {
                    const int nk = min(kpb, t.kb1 - kb0);
                    if (!pwait(&empty[s], ph ^ 1u, a, DEV_TIMEOUT_PRODUCER_EMPTY, abort_flag, peer_abort)) {
                        ok = false;
                        break;
                    }
                    if (leader) mbar_arrive_expect_tx(&full[s], pair_bytes * static_cast<uint32_t>(nk));
                    const uint32_t bar = leader_full0 + 8u * s;
                    for (int h = 0; h < nk; ++h) {
                        const int kb = kb0 + h;
                        uint8_t* stage = smem + (static_cast<size_t>(s) * kpb + h) * sbytes;
                        if (!t.swap) {
                            if (t.half)  // 64 token rows per CTA
                                tma_load_pair(&maps.tok64[t.phase], stage, bar, kb * kBK,
                                              static_cast<int32_t>(t.row0 + 64 * rank), pol_last);
                            else
                                tma_load_pair(&maps.tok[t.phase], stage, bar, kb * kBK,
                                              static_cast<int32_t>(t.row0 + 128 * rank), pol_last);
                            tma_load_pair(&maps.w[t.phase], stage + kHalf, bar, 0,
                                          static_cast<int32_t>((wblk0 * pa.k_blocks + kb) * 128), pol_first);
                        } else {
                            for (int j = 0; j < t.wt; ++j)
                                tma_load_pair(&maps.w[t.phase], stage + j * kHalf, bar, 0,
                                              static_cast<int32_t>(((wblk0 + 2 * j) * pa.k_blocks + kb) * 128), pol_first);
                            const int64_t trow = t.row0 + static_cast<int64_t>(rank) * half;
                            for (int j = 0; j < n64; ++j)
                                tma_load_pair(&maps.tok64[t.phase], stage + a.xoff + j * 8192, bar, kb * kBK,
                                              static_cast<int32_t>(trow + 64 * j), pol_last);
                            for (int j = 0; j < nb16; ++j)
                                tma_load_pair(&maps.tok16[t.phase], stage + a.xoff + n64 * 8192 + j * 2048, bar, kb * kBK,
                                              static_cast<int32_t>(trow + 64 * n64 + 16 * j), pol_last);
                        }
                    }
                    use_bytes[s] = (leader ? pair_bytes : pair_bytes / 2u) * static_cast<uint32_t>(nk);
                    ++uses;
                    if (++s == static_cast<uint32_t>(S)) { s = 0; ph ^= 1u; }
                }
            }
            if (!leader) {
                // report to the leader: this CTA issues no more copies
                const uint32_t rep = mapa_shared(smem_u32(report), 0);
                remote_store(rep, static_cast<int>(uses));
                for (int i = 0; i < S; ++i)
                    remote_store(rep + 8u + 4u * i, static_cast<int>(use_bytes[i]));
                fence_cluster();
                remote_store(rep + 4u, 1);
            } else {
                // Drain (leader): reconcile with the peer's report, then wait
                // for every stage's last phase, so that no copy of either CTA
                // is in flight when the pair passes its final cluster barrier.
                bool have = false;
                for (uint32_t i = 0; i < a.wait_limit; ++i) {
                    if (ld_acquire_cluster(&report->done) != 0u) {
                        have = true;
                        break;
                    }
                    if (i > 64) __nanosleep(128);
                }
                fence_cluster();
                uint32_t last = uses;  // stage uses whose phases are armed
                if (!have) {
                    atomicCAS(a.status, 0, DEV_TIMEOUT_DRAIN);
                    *abort_flag = 1;
                    remote_store(peer_abort, 1);
                } else {
                    const uint32_t np = report->uses;
                    if (np > uses && np - uses <= static_cast<uint32_t>(S)) {
                        // uses the peer issued and the leader never armed: arm them
                        // for the peer's bytes alone
                        for (uint32_t u = uses; u < np; ++u) {
                            const uint32_t st = u % static_cast<uint32_t>(S);
                            mbar_arrive_expect_tx(&full[st], report->bytes[st]);
                        }
                        last = np;
                    } else if (np < uses && uses - np <= static_cast<uint32_t>(S)) {
                        // uses the leader armed that the peer never issued: the
                        // peer's half will not arrive, complete it by hand
                        for (uint32_t u = np; u < uses; ++u) {
                            const uint32_t st = u % static_cast<uint32_t>(S);
                            mbar_complete_tx(&full[st], use_bytes[st] / 2u);
                        }
                    } else if (np != uses) {
                        atomicCAS(a.status, 0, DEV_TIMEOUT_DRAIN);  // inconsistent report: drain what is known
                    }
                }
                // the last armed phase of every stage (use u of stage u % S has parity (u / S) & 1)
                const uint32_t first = last > static_cast<uint32_t>(S) ? last - static_cast<uint32_t>(S) : 0u;
                for (uint32_t u = first; u < last; ++u)
                    mbar_drain(&full[u % static_cast<uint32_t>(S)], (u / static_cast<uint32_t>(S)) & 1u, a.status,
                               DEV_TIMEOUT_DRAIN, a.wait_limit);
            }
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {
            // ------------------------------------------------ pair MMA issuer (leader only)
            uint32_t s = 0, ph = 0, r = 0, rph = 0;
            int it = 0;
            bool ok = true;
            while (ok) {
                if (!pwait(&rfull[r], rph, a, DEV_TIMEOUT_MMA_FULL, abort_flag, peer_abort)) break;
                const int tile = ring[r];
                mbar_arrive(&rempty[r]);
                if (++r == kRing) { r = 0; rph ^= 1u; }
                if (tile < 0) break;
                const Tile2 t = decode2<kHalfTiles>(a, tile, tstart, off);
                const int buf = it & 1;
                const uint32_t use = static_cast<uint32_t>(it >> 1);
                ++it;
                if (!pwait(&tempty[buf], (use & 1u) ^ 1u, a, DEV_TIMEOUT_MMA_TEMPTY, abort_flag, peer_abort)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf) * 256u;
                const uint32_t n_mma = t.swap ? static_cast<uint32_t>((t.rows + 15) / 16) * 16u : 256u;
                const uint32_t idesc = umma_idesc_bf16(t.half ? 128 : 256, n_mma);
                for (int kb0 = t.kb0; kb0 < t.kb1; kb0 += kpb) {
                    const int nk = min(kpb, t.kb1 - kb0);
                    if (!pwait(&full[s], ph, a, DEV_TIMEOUT_MMA_FULL, abort_flag, peer_abort)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int h = 0; h < nk; ++h) {
                        const int kb = kb0 + h;
                        const uint32_t stage = smem_u32(smem + (static_cast<size_t>(s) * kpb + h) * sbytes);
                        if (!t.swap) {
#pragma unroll
                            for (int kk = 0; kk < kBK / 16; ++kk)
                                umma_pair(d_tmem, umma_desc_sw128(stage + kk * 32), umma_desc_sw128(stage + kHalf + kk * 32),
                                          idesc, (kb > t.kb0 || kk > 0) ? 1u : 0u);
                        } else {
                            // sub-tile j accumulates into columns 128 j .. of the buffer
                            for (int j = 0; j < t.wt; ++j) {
#pragma unroll
                                for (int kk = 0; kk < kBK / 16; ++kk)
                                    umma_pair(d_tmem + 128u * j, umma_desc_sw128(stage + j * kHalf + kk * 32),
                                              umma_desc_sw128(stage + a.xoff + kk * 32), idesc,
                                              (kb > t.kb0 || kk > 0) ? 1u : 0u);
                            }
                        }
                    }
                    umma_commit_pair(&empty[s]);
                    if (++s == static_cast<uint32_t>(S)) { s = 0; ph ^= 1u; }
                }
                if (ok) umma_commit_pair(&tfull[buf]);
            }
            // all issued MMAs (into both CTAs' TMEM) complete before TMEM is freed
            asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                         ::"r"(smem_u32(drain)) : "memory");
            mbar_drain(drain, 0, a.status, DEV_TIMEOUT_DRAIN, a.wait_limit);
        }
    } else {
        // ---------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;
        uint32_t r = 0, rph = 0;
        int it = 0;
        uint32_t nst = 0;  // staged tile stores this warp issued
        for (;;) {
            if (!pwait(&rfull[r], rph, a, DEV_TIMEOUT_EPI_TFULL, abort_flag, peer_abort)) break;
            const int tile = ring[r];
            __syncwarp();
            if (lane == 0) remote_arrive(leader_rempty0 + 8u * r);
            if (++r == kRing) { r = 0; rph ^= 1u; }
            if (tile < 0) break;
            const Tile2 t = decode2<kHalfTiles>(a, tile, tstart, off);
            const Phase2& pa = a.ph[t.phase];
            const int buf = it & 1;
            const uint32_t use = static_cast<uint32_t>(it >> 1);
            ++it;
            if (!pwait(&tfull[buf], use & 1u, a, DEV_TIMEOUT_EPI_TFULL, abort_flag, peer_abort)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + static_cast<uint32_t>(buf) * 256u + (static_cast<uint32_t>(q * 32) << 16);
            float v[32];
            if (!t.swap) {
                // Rows of the pair's tile this warp holds (slab0 + lane) and their
                // output columns (col0 + 32 c).  A 256-row tile: CTA r holds rows
                // 128 r .., lane quarter q rows 32 q .., all 256 columns.  A 128-row
                // tile (M = 128): CTA r holds rows 64 r .., TMEM lanes 0-63 its rows
                // with columns 0-127, lanes 64-127 the same rows with columns 128-255.
                const int slab0 = t.half ? static_cast<int>(rank) * 64 + (q & 1) * 32
                                         : static_cast<int>(rank) * 128 + q * 32;
                const int col0 = t.n0 + (t.half ? (q >> 1) * 128 : 0);
                const int nchunks = t.half ? 4 : 8;
                const int rr = slab0 + lane;  // row within the pair's tile
                const bool valid = rr < t.rows;
                const int64_t grow = t.row0 + rr;
                // fp32 output of a slab whose 32 rows all belong to the group: staged
                // in shared memory and written by one TMA tile store per chunk
                const bool staged = pa.tma_out && a.stg_bufs > 0 && slab0 + 32 <= t.rows;
                for (int c = 0; c < nchunks; ++c) {
                    tmem_ld32(taddr + static_cast<uint32_t>(c * 32), v);
                    if (staged) {
                        uint8_t* stg = smem + a.stg_off +
                                       static_cast<size_t>(q * a.stg_bufs + static_cast<int>(nst % a.stg_bufs)) * 4096;
                        if (lane == 0) {
                            // the store that last used this buffer has read it
                            if (a.stg_bufs > 1) bulk_wait_read<1>(); else bulk_wait_read<0>();
                        }
                        __syncwarp();
                        stage_row_f32_sw128(stg, lane, v);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&maps.out[t.phase], stg, col0 + c * 32,
                                         static_cast<int32_t>(t.split * pa.split_rows + t.row0 + slab0));
                            bulk_commit();
                        }
                        ++nst;
                        continue;
                    }
                    if (!valid) continue;
                    if (pa.epi == EPI_SWIGLU_BF16) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            pk[i] = pack2(silu2(v[2 * i]) * v[16 + 2 * i], silu2(v[2 * i + 1]) * v[16 + 2 * i + 1]);
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<bf16*>(pa.out) + grow * pa.ldo +
                                                              (col0 / 2 + c * 16));
                        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    } else {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(pa.out) +
                                                                static_cast<int64_t>(t.split) * pa.split_stride +
                                                                grow * pa.ldo + col0 + c * 32);
#pragma unroll
                        for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                    }
                }
            } else {
                // accumulator `sub`: lanes are this CTA's 128 weight rows n0 + 256 sub + 128 rank + ..,
                // columns 128 sub + (the tile's tokens)
                const int nbk = (t.rows + 31) / 32;
                for (int cc = 0; cc < t.wt * nbk; ++cc) {
                    const int sub = cc / nbk, c = cc - sub * nbk;
                    const int nwr = t.n0 + 256 * sub + 128 * static_cast<int>(rank);
                    tmem_ld32(taddr + static_cast<uint32_t>(128 * sub + c * 32), v);
                    if (pa.epi == EPI_SWIGLU_BF16) {
                        // lane l < 16 holds gate row f0 + l and lane l + 16 the up
                        // row of the same f, each for 32 tokens.  The half-warps
                        // split the tokens: lane l finishes token j, lane l + 16
                        // token j + 16, after one exchange per token pair, so each
                        // lane computes 16 SiLUs and every store writes for both.
                        const bool hi = lane >= 16;
                        const int f = nwr / 2 + q * 16 + (lane & 15);
                        const int tok0 = c * 32 + (hi ? 16 : 0);
                        bf16* H = static_cast<bf16*>(pa.out) + (t.row0 + tok0) * pa.ldo + f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float other = __shfl_xor_sync(0xffffffffu, hi ? v[j] : v[j + 16], 16);
                            const float g = hi ? other : v[j];
                            const float u = hi ? v[j + 16] : other;
                            if (tok0 + j < t.rows) H[static_cast<int64_t>(j) * pa.ldo] = __float2bfloat16_rn(silu2(g) * u);
                        }
                    } else {
                        float* Y = static_cast<float*>(pa.out) + static_cast<int64_t>(t.split) * pa.split_stride;
                        const int col = nwr + q * 32 + lane;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int tok = c * 32 + j;
                            if (tok < t.rows) Y[(t.row0 + tok) * pa.ldo + col] = v[j];
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                remote_arrive(leader_tempty0 + 8u * buf);
                if (t.phase == 0 && a.dep) {
                    asm volatile("fence.proxy.async.global;" ::: "memory");
                    __threadfence();
                    atomicAdd(&a.sched[1 + t.g], 1);
                }
            }
        }
    }

    // staged output stores complete (and stop reading shared memory) before the CTA exits
    if (warp >= 2 && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // the peer's TMEM and shared memory stay alive until the leader is done
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder2() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool map2(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows, bool swizzle) {
    auto enc = encoder2();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows < 1 ? 1 : rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64u, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool gemm_2sm_supported(const GemmLaunch& L) {
    if (L.nphase < 1 || L.nphase > 2 || L.G < 1 || L.G > kMaxGroups || L.group_off == nullptr) return false;
    for (int p = 0; p < L.nphase; ++p) {
        const GemmPhase& g = L.ph[p];
        if (g.N % 256 != 0 || g.Kdim % 8 != 0 || g.Kdim < 16 || g.N_store != g.N || (g.ldo & 3) != 0) return false;
        if (g.ksplit > 1 && g.epi != EPI_F32) return false;  // SwiGLU needs the whole reduction
    }
    return true;
}

int launch_grouped_gemm_2sm(const GemmLaunch& L, cudaStream_t st) {
    if (!gemm_2sm_supported(L) || !L.sched) return -2;
    Args2 a{};
    a.group_off = L.group_off;
    a.G = L.G;
    a.nphase = L.nphase;
    a.dep = L.nphase == 2 ? 1 : 0;
    a.status = L.status;
    a.sched = L.sched;
    a.wait_limit = L.wait_limit ? L.wait_limit : kWaitLimit;
    a.dep_wait_limit = L.dep_wait_limit ? L.dep_wait_limit : kWaitLimit;
    a.dep_extra = L.dep_extra;
    a.w_slot = L.w_slot;
    a.w_slots = L.w_slots;
    if (L.w_slot && L.w_slots < 1) return -2;
    const int64_t mx = L.max_group_rows < 1 ? 1 : L.max_group_rows;
    a.swap_max_rows = L.swap_max_rows < 0 ? 0 : L.swap_max_rows;
    {
        const int64_t lim = mx < a.swap_max_rows ? mx : a.swap_max_rows;
        a.BNs = static_cast<int>(lim >= 128 ? 128 : ((lim + 31) / 32) * 32);
        if (a.BNs < 32) a.BNs = 32;
    }
    const bool weight_major_possible = a.swap_max_rows > 0;
    const int sms = num_sms();
    if (sms <= 1) return -3;
    const int clusters = sms / 2;
    if (clusters < 2) return -2;  // the two tile queues need a pair each
    Maps2 maps;
    std::memset(&maps, 0, sizeof(maps));
    for (int p = 0; p < L.nphase; ++p) {
        const GemmPhase& g = L.ph[p];
        Phase2& ph = a.ph[p];
        ph.w = g.w;
        ph.N = g.N;
        ph.k_blocks = (g.Kdim + kBK - 1) / kBK;
        ph.epi = g.epi;
        ph.nb = g.N / 128;
        ph.out = g.out;
        ph.ldo = g.ldo;
        ph.split_stride = g.split_stride;
        int ks = g.ksplit < 1 ? 1 : g.ksplit;
        if (ks > ph.k_blocks) ks = ph.k_blocks;
        ph.kb_per_split = (ph.k_blocks + ks - 1) / ks;
        ph.ksplit = (ph.k_blocks + ph.kb_per_split - 1) / ph.kb_per_split;
        // Two 256-row weight sub-tiles per weight-major tile when the width
        // allows and the phase still has at least 3 tiles per cluster with
        // every group active.  (Single sub-tiles for the groups scheduled
        // last, to shorten the final tiles, measured slower at the Mixtral
        // decode shape: their extra token reads cost more than the shorter
        // tail saved.)
        ph.wt = (weight_major_possible && g.N % 512 == 0 &&
                 static_cast<int64_t>(L.G) * (g.N / 512) * ph.ksplit >= 3LL * clusters) ? 2 : 1;
        const uint64_t trows = static_cast<uint64_t>(g.tok_rows);
        if (!map2(&maps.tok[p], g.tok, trows, g.Kdim, 128u, true)) return -3;
        if (!map2(&maps.tok16[p], g.tok, trows, g.Kdim, 16u, true)) return -3;
        if (!map2(&maps.tok64[p], g.tok, trows, g.Kdim, 64u, true)) return -3;
        const uint64_t wmats = static_cast<uint64_t>(L.w_slot ? L.w_slots : L.G);
        const uint64_t wrows = wmats * ph.nb * ph.k_blocks * 128;
        if (!map2(&maps.w[p], g.w, wrows, 64, 128u, false)) return -3;
        ph.tma_out = out_map_ok(g) ? 1 : 0;  // cleared below if no staging fits
        ph.split_rows = ph.tma_out && ph.ksplit > 1 ? g.split_stride / g.ldo : 0;
        if (ph.tma_out && !make_out_map(&maps.out[p], g.out, out_map_rows(g, ph.ksplit), g.N, g.ldo, false)) return -3;
    }
    const size_t fixed = 1024 + static_cast<size_t>(2 * kMaxStages + 4 + 2 * kRing + 1) * 8 + kRing * 4 + 16 +
                         static_cast<size_t>(L.G + 1) * (8 + 4 * 4) + 4 + sizeof(PeerReport) + 64;
    // stage: token-major tiles need 2 x 16 KB; weight-major tiles wt x 16 KB
    // of weights and BNs / 2 token rows
    int wt_max = 1;
    for (int p = 0; p < L.nphase; ++p) wt_max = a.ph[p].wt > wt_max ? a.ph[p].wt : wt_max;
    a.xoff = static_cast<uint32_t>(wt_max) * kHalf;
    // decode-sized launches (weight-major tiles for groups of <= 128 rows)
    // under programmatic launch: prefetch up to 16 k-blocks of each
    // first-round weight tile.  Without it the prefetch cannot overlap the
    // earlier kernels and measured slightly slower at decode (0.488-0.490 vs
    // 0.485-0.488 ms per step), so it is off.
    a.prefetch_kb = (kProgrammaticLaunch && weight_major_possible && L.w_slot == nullptr)
                        ? (a.ph[0].k_blocks < 16 ? a.ph[0].k_blocks : 16) : 0;
    // Rings.  Token-major pairs: 32 KB per k-block and CTA, two k-blocks per
    // stage where three such stages fit (a producer thread's copies issued
    // after a barrier wait are serviced about one stage at a time, so fewer,
    // larger stages move more bytes per stage cycle: prefill-sized layer,
    // expert GEMMs 3-6 % faster).  Weight-major pairs: wt weight sub-tiles and
    // BNs / 2 token rows per k-block, one k-block per stage and a deeper ring
    // (two k-blocks there measured slower).  Both rings are always set up;
    // the kernel splits the pairs between the queues at run time.
    const size_t avail = 227 * 1024 - fixed;
    a.stage_bytes[0] = 2u * kHalf;
    a.stage_bytes[1] = a.xoff + static_cast<uint32_t>(a.BNs) * 64u;
    size_t ring = 0, ring_q[2] = {0, 0};
    for (int q = 0; q < 2; ++q) {
        a.kpb[q] = (q == 0 && avail / (2 * static_cast<size_t>(a.stage_bytes[0])) >= 3) ? 2 : 1;
        int stages = static_cast<int>(avail / (a.kpb[q] * static_cast<size_t>(a.stage_bytes[q])));
        if (stages > kMaxStages) stages = kMaxStages;
        if (stages < 2) return -2;
        a.stages[q] = stages;
        ring_q[q] = static_cast<size_t>(stages) * a.kpb[q] * a.stage_bytes[q];
    }
    // Output staging of token-major pairs (4 epilogue warps x 4 KB per buffer)
    // after their ring: two buffers per warp, else one, in the room the ring
    // leaves.  Weight-major pairs never touch it (their epilogue stores
    // columns of 32 tokens, already whole rows), so it may overlap their ring.
    bool want_stg = false;
    for (int p = 0; p < L.nphase; ++p) want_stg = want_stg || a.ph[p].tma_out;
    a.stg_bufs = 0;
    for (int nb = 2; want_stg && nb >= 1 && a.stg_bufs == 0; --nb)
        if (ring_q[0] + static_cast<size_t>(nb) * 4 * 4096 <= avail) a.stg_bufs = nb;
    if (a.stg_bufs == 0)
        for (int p = 0; p < L.nphase; ++p) a.ph[p].tma_out = 0;
    a.stg_off = static_cast<uint32_t>(ring_q[0]);
    ring = ring_q[0] + static_cast<size_t>(a.stg_bufs) * 4 * 4096;
    if (ring_q[1] > ring) ring = ring_q[1];
    a.ring_bytes = ring;
    const size_t smem = fixed + ring;
    // 128-row tiles where groups of mixed sizes are expected (weight-major
    // tiles enabled): the token-major groups' last chunks are often <= 128 rows
    const bool half_tiles = weight_major_possible;
    void (*kern)(Maps2, Args2) = half_tiles ? grouped_gemm_2sm_kernel<true> : grouped_gemm_2sm_kernel<false>;
    static std::atomic<unsigned long long> attr_done[2] = {{0}, {0}};
    if (smem_attr_once(reinterpret_cast<const void*>(kern), 227 * 1024, attr_done[half_tiles ? 1 : 0]) != 0) return -3;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attrs[2];
    attrs[0].id = cudaLaunchAttributeClusterDimension;
    attrs[0].val.clusterDim.x = 2;
    attrs[0].val.clusterDim.y = 1;
    attrs[0].val.clusterDim.z = 1;
    attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // pdl_wait in the kernel
    attrs[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attrs;
    cfg.numAttrs = kProgrammaticLaunch ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, kern, maps, a) != cudaSuccess) return -3;
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace moe
