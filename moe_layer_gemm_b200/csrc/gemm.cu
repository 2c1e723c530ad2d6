// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), fed by
// TMA, for the expert FFN of an MoE layer: each expert g multiplies its own
// contiguous group of token rows by its own weight matrix ("MoE computation
// notes", cf-1.com/news/5905749, section 2.1: permute tokens so each expert
// gets one contiguous batch and run one matrix product per group; section
// 2.2: experts never see tokens that did not choose them).
//
// One persistent CTA per SM.  Up to two phases run in one launch: the
// gate/up projection with its SwiGLU epilogue (phase 0) and the down
// projection (phase 1).  Tiles are handed out by a global atomic counter in
// phase order, and a phase-1 tile of expert g waits (bounded) until every
// phase-0 tile of g has stored its H rows, so the down projection of early
// experts overlaps the gate/up projection of late ones and there is one
// tail instead of two.  Roles per CTA (224 threads):
//   warp 0        scheduler + producer 0 (one elected thread): claims tiles
//                 and broadcasts them through a shared-memory ring
//   warps 0, 6    producers (one elected thread each): fill a multi-stage
//                 operand ring, alternating stage uses (producer k issues
//                 the uses u with u % 2 == k, so it owns the stages of that
//                 parity): token rows by TMA tile loads, weight tiles by
//                 contiguous 16 KB bulk copies of the pre-tiled,
//                 pre-swizzled packed weights
//   warp 1        TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2..5    epilogue: TMEM -> registers -> SwiGLU / fp32 -> global.
//                 Rows of token-major tiles go through a 4 KB staging buffer
//                 per warp and one TMA tile store per 32 x 32 fp32 block (or
//                 32 x 64 bf16 block of H): stored from registers, each
//                 16-byte store touched 32 rows, and the down projection's
//                 short tiles (reduction d_ff) could not hide them (Qwen-like
//                 layer: expert GEMMs 0.430 -> 0.411 ms; with no output
//                 stores at all, 0.39)
// Two producers: with 16 KB stages a probe measured one issuing thread at
// about one stage per 0.4 us whatever the ring depth, and two threads at
// twice that; with this kernel's 48 KB stages the probe's rate no longer
// depends on the number of issuing threads (the copy engine's throughput,
// about 140 GB/s per SM with every SM loading, binds), and the second
// producer measured 2-3 % faster at the Qwen-like shape.
// The accumulator is double-buffered in TMEM (2 x 256 fp32 columns).
//
// Tile orientation is chosen per group:
//   token-major:  D[128 tokens x BN weight rows]   (groups with many tokens)
//   weight-major: D[128 weight rows x n tokens], n <= 128 a multiple of 32
//                 (small groups: no tensor-core rows spent on padding; the
//                 weight stream dominates).  In phase 1 the reduction of a
//                 weight-major tile can be split into slices written to
//                 separate partial buffers and summed later in slice order.
// No TMA multicast is used anywhere.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kBK = 64;                        // reduction elements per stage (one 128 B swizzle row)
constexpr int kThreads = 224;
constexpr int kProducer1Warp = 6;
constexpr uint32_t kTileABytes = 128u * 128u;  // 128 rows x 64 bf16
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxGroups = 256;
constexpr int kRing = 8;                       // scheduled tiles buffered between roles

struct PhaseArgs {
    const bf16* w;  // tiled weights (tiled_offset), groups w_group_elems apart
    int64_t w_group_elems;
    int N;        // weight rows per group
    int N_store;  // output columns written (router: E of E_pad)
    int k_blocks;
    int ksplit;   // reduction split (partial slices), every tile of the phase
    int kb_per_split;
    int epi;
    int BN;       // token-major: weight rows per tile
    void* out;
    int64_t ldo;
    int64_t split_stride;
    int tma_out;         // fp32 token-major tiles store full 32-row slabs by TMA (Maps::out)
    int tma_h;           // SwiGLU token-major tiles store full 32-row slabs of H by TMA (Maps::out)
    int64_t split_rows;  // rows between partial slices in the output map (split_stride / ldo)
};

struct DevArgs {
    const int32_t* group_off;
    int G;
    int64_t dense_rows;
    int swap_max_rows;  // groups with rows <= this use weight-major tiles
    int BNs;            // weight-major: max tokens per tile (multiple of 32, <= 128)
    int nphase;
    int dep;            // phase-1 tiles of g wait for all phase-0 tiles of g
    PhaseArgs ph[2];
    int stages;                 // operand ring depth; a stage holds one weight and one token slot
    uint32_t wslot, xslot;      // bytes per weight / token slot
    int stg_bufs;               // 4 KB output staging buffers per epilogue warp (0: none)
    int* status;
    int* sched;         // [0] tile counter, [1..G] phase-0 tiles done per group (x4 warps)
    uint32_t wait_limit;      // polls of a bounded mbarrier or drain wait
    uint32_t dep_wait_limit;  // polls of the phase-1 readiness wait
    int dep_extra;            // added to the phase-1 readiness target (0; a test makes it unreachable)
    const int32_t* w_slot;    // group -> weight matrix (expert cache slot), or nullptr
    int w_slots;
};

struct Maps {
    CUtensorMap tokA[2];  // token rows, box 128 (token-major A)
    CUtensorMap tokB[2];  // token rows, box 32  (weight-major B)
    CUtensorMap out[2];   // output rows, 128-byte swizzle: fp32 box {32, 32} (tma_out) or bf16 box {64, 32} (tma_h)
};

struct Tile {
    int phase;
    int g;
    int swap;
    int64_t row0;  // first token row
    int rows;      // valid token rows
    int n0;        // first weight row within the group
    int kb0, kb1;
    int split;
};

__device__ __forceinline__ bool group_swaps(const DevArgs& a, int p, int64_t rows) {
    return rows <= a.swap_max_rows && a.ph[p].N % 128 == 0;
}

__device__ __forceinline__ int tiles_of(const DevArgs& a, int p, int64_t rows) {
    if (rows <= 0) return 0;
    const PhaseArgs& ph = a.ph[p];
    if (!group_swaps(a, p, rows)) return static_cast<int>(((rows + 127) / 128) * (ph.N / ph.BN) * ph.ksplit);
    return static_cast<int>(((rows + a.BNs - 1) / a.BNs) * (ph.N / 128) * ph.ksplit);
}

// tstart[p*(G+1) + g]: first tile of group g in phase p (global numbering).
__device__ __forceinline__ Tile decode_tile(const DevArgs& a, int tile, const int* tstart, const int64_t* off) {
    Tile t;
    const int G = a.G;
    int p = 0;
    if (a.nphase > 1 && tile >= tstart[G]) p = 1;
    const int* ts = tstart + p * (G + 1);
    int lo = 0, hi = G;  // ts[lo] <= tile < ts[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ts[mid] <= tile) lo = mid; else hi = mid;
    }
    const PhaseArgs& ph = a.ph[p];
    t.phase = p;
    t.g = lo;
    const int local = tile - ts[lo];
    const int64_t base = off[lo];
    const int64_t rows_g = off[lo + 1] - base;
    t.swap = group_swaps(a, p, rows_g) ? 1 : 0;
    if (!t.swap) {
        // a reduction split applies to every tile of the phase, so each
        // partial slice is written for every row
        const int s = local % ph.ksplit;
        const int rest = local / ph.ksplit;
        const int mt = static_cast<int>((rows_g + 127) / 128);
        const int n = rest / mt, m = rest - n * mt;  // m fastest: weight tile reused from L2
        const int64_t r0 = static_cast<int64_t>(m) * 128;
        t.row0 = base + r0;
        t.rows = static_cast<int>(rows_g - r0 < 128 ? rows_g - r0 : 128);
        t.n0 = n * ph.BN;
        t.kb0 = s * ph.kb_per_split;
        t.kb1 = min(ph.k_blocks, t.kb0 + ph.kb_per_split);
        t.split = s;
    } else {
        const int nch = static_cast<int>((rows_g + a.BNs - 1) / a.BNs);
        const int s = local % ph.ksplit;
        const int rest = local / ph.ksplit;
        const int c = rest % nch;
        const int w = rest / nch;
        const int64_t r0 = static_cast<int64_t>(c) * a.BNs;
        t.row0 = base + r0;
        t.rows = static_cast<int>(rows_g - r0 < a.BNs ? rows_g - r0 : a.BNs);
        t.n0 = w * 128;
        t.kb0 = s * ph.kb_per_split;
        t.kb1 = min(ph.k_blocks, t.kb0 + ph.kb_per_split);
        t.split = s;
    }
    return t;
}

// silu(g) = g / (1 + e^-g) with the fast exp and divide intrinsics: the
// result is rounded to bf16 (8-bit mantissa) right after, far coarser than
// their few-ulp error.  For g < -87, e^-g overflows to inf and the quotient
// is 0, the limit of silu.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

// Rows n .. n+rows-1 (rows <= 128, n a multiple of 8, within one 128-row
// block) of k-block kb of group g's tiled weights: one contiguous range.
__device__ __forceinline__ const bf16* weight_rows(const PhaseArgs& pa, int g, int n, int kb) {
    return pa.w + static_cast<int64_t>(g) * pa.w_group_elems + tiled_offset(n, static_cast<int64_t>(kb) * 64, pa.k_blocks);
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ Maps maps, const DevArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int S = a.stages;
    uint8_t* sW = smem;                                               // [S][wslot]
    uint8_t* sX = smem + static_cast<size_t>(S) * a.wslot;            // [S][xslot]
    uint8_t* sStg = sX + static_cast<size_t>(S) * a.xslot;           // [4 warps][stg_bufs][4 KB]
    uint64_t* full = reinterpret_cast<uint64_t*>(sStg + static_cast<size_t>(a.stg_bufs) * 4 * 4096);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;
    uint64_t* tempty = tfull + 2;
    uint64_t* rfull = tempty + 2;
    uint64_t* rempty = rfull + kRing;
    uint64_t* drain = rempty + kRing;
    int* ring = reinterpret_cast<int*>(drain + 1);                   // [kRing]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring + kRing);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int64_t* off = reinterpret_cast<int64_t*>(tmem_slot + 2);        // [G+1]
    int* tstart = reinterpret_cast<int*>(off + a.G + 1);             // [2][G+1]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = a.G;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        for (int r = 0; r < kRing; ++r) {
            mbar_init(&rfull[r], 1);
            mbar_init(&rempty[r], 6);  // producer 1 + MMA thread + 4 epilogue warps
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int p = 0; p < a.nphase; ++p) {
            tma_prefetch_desc(&maps.tokA[p]);
            tma_prefetch_desc(&maps.tokB[p]);
        }
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    // group offsets, scheduler words and token rows come from earlier kernels
    pdl_wait();
    // Under programmatic launch (kProgrammaticLaunch, off by default) the
    // next kernel may launch once every CTA has run out of tiles (its
    // producer sees the end marker, below), so its CTAs do not sit resident
    // on the SMs through the whole launch, only through the last tiles.
    for (int g = threadIdx.x; g <= G; g += blockDim.x)
        off[g] = a.group_off ? static_cast<int64_t>(a.group_off[g]) : (g == 0 ? 0 : a.dense_rows);
    __syncthreads();
    // rows of group g in this launch (0 for a group the slot table skips)
    auto rows_of = [&](int g) -> int64_t { return group_skipped(a.w_slot, g) ? 0 : off[g + 1] - off[g]; };
    if (warp == 0) {
        // tile prefix over (phase, group): each lane scans a contiguous span of groups
        const int span = (G + 31) / 32;
        const int g0 = min(G, lane * span), g1 = min(G, g0 + span);
        int carry = 0;
        for (int p = 0; p < a.nphase; ++p) {
            int sum = 0;
            for (int g = g0; g < g1; ++g) sum += tiles_of(a, p, rows_of(g));
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            int run = carry + incl - sum;
            int* ts = tstart + p * (G + 1);
            for (int g = g0; g < g1; ++g) {
                ts[g] = run;
                run += tiles_of(a, p, rows_of(g));
            }
            const int tot = __shfl_sync(0xffffffffu, incl, 31);
            if (lane == 0) ts[G] = carry + tot;
            carry += tot;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = tstart[(a.nphase - 1) * (G + 1) + G];

    if (warp == 0 || warp == kProducer1Warp) {
        if (lane == 0) {
            // ------------------------------------- scheduler + producers
            const uint32_t me = warp == 0 ? 0u : 1u;
            const uint64_t pol_first = policy_evict_first();
            const uint64_t pol_last = policy_evict_last();
            uint32_t s = 0, ph = 0, r = 0, rph = 0, u = 0;
            uint32_t issued_mask = 0, issued_ph = 0;
            bool ok = true;
            // claims run one tile ahead so the atomic's round trip overlaps
            // the loads of the current tile
            int next = me == 0 ? atomicAdd(&a.sched[0], 1) : 0;
            while (ok) {
                int tile;
                if (me == 0) {
                    tile = next < total ? next : -1;
                    if (tile >= 0) next = atomicAdd(&a.sched[0], 1);
                    if (!mbar_wait(&rempty[r], rph ^ 1u, a.status, DEV_TIMEOUT_PRODUCER_EMPTY, abort_flag,
                                   a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    ring[r] = tile;
                    mbar_arrive(&rfull[r]);
                } else {
                    if (!mbar_wait(&rfull[r], rph, a.status, DEV_TIMEOUT_PRODUCER_EMPTY, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    tile = ring[r];
                    mbar_arrive(&rempty[r]);
                }
                if (++r == kRing) { r = 0; rph ^= 1u; }
                if (tile < 0) {  // the end marker
                    pdl_trigger();
                    break;
                }
                const Tile t = decode_tile(a, tile, tstart, off);
                const PhaseArgs& pa = a.ph[t.phase];
                if (t.phase == 1 && a.dep) {
                    // all phase-0 tiles of this group must have stored their rows
                    const int need = 4 * (tstart[t.g + 1] - tstart[t.g]) + a.dep_extra;
                    uint32_t i = 0;
                    while (ld_acquire(&a.sched[1 + t.g]) < need) {
                        if (*abort_flag) {
                            ok = false;
                            break;
                        }
                        if (++i > a.dep_wait_limit) {
                            atomicCAS(a.status, 0, DEV_TIMEOUT_DEPENDENCY);
                            *abort_flag = 1;
                            ok = false;
                            break;
                        }
                        if (i > 64) __nanosleep(128);
                    }
                    fence_proxy_async_global();
                    if (!ok) break;
                }
                const int wg = weight_slot(a.w_slot, a.w_slots, t.g, a.status);
                const int nb = t.swap ? (t.rows + 31) / 32 : 0;
                const uint32_t wbytes = t.swap ? 16384u : static_cast<uint32_t>(pa.BN) * 128u;
                const uint32_t xbytes = t.swap ? static_cast<uint32_t>(nb) * 4096u : kTileABytes;
                for (int kb = t.kb0; kb < t.kb1; ++kb, ++u) {
                    const uint32_t cs = s, cph = ph;  // this use's stage and phase
                    if (++s == static_cast<uint32_t>(S)) { s = 0; ph ^= 1u; }
                    if ((u & 1u) != me) continue;     // the other producer's use
                    if (!mbar_wait(&empty[cs], cph ^ 1u, a.status, DEV_TIMEOUT_PRODUCER_EMPTY, abort_flag,
                                   a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[cs], wbytes + xbytes);
                    uint8_t* dW = sW + static_cast<size_t>(cs) * a.wslot;
                    uint8_t* dX = sX + static_cast<size_t>(cs) * a.xslot;
                    const int kx = kb * kBK;
                    if (t.swap) {
                        // weights (M side): one contiguous 16 KB tile, streamed once
                        bulk_load(dW, weight_rows(pa, wg, t.n0, kb), 16384u, &full[cs], pol_first);
                        for (int j = 0; j < nb; ++j)
                            tma_load_2d(&maps.tokB[t.phase], dX + j * 4096, &full[cs], kx,
                                        static_cast<int32_t>(t.row0 + 32 * j), pol_last);
                    } else {
                        // tokens (M side): 128 rows, kept in L2 for the group's other
                        // weight tiles; weights: BN rows, marked first to leave L2
                        // once the group's row tiles (running together) have read them
                        tma_load_2d(&maps.tokA[t.phase], dX, &full[cs], kx, static_cast<int32_t>(t.row0), pol_last);
                        if (pa.BN >= 128) {
                            for (int j = 0; j < pa.BN / 128; ++j)
                                bulk_load(dW + j * 16384, weight_rows(pa, wg, t.n0 + 128 * j, kb), 16384u, &full[cs],
                                          pol_first);
                        } else {
                            bulk_load(dW, weight_rows(pa, wg, t.n0, kb), wbytes, &full[cs], pol_first);
                        }
                    }
                    issued_mask |= 1u << cs;
                    issued_ph = (issued_ph & ~(1u << cs)) | (cph << cs);
                }
            }
            // Leaving without the end marker means a wait failed and raised the
            // abort flag, which every consumer's wait watches, so none needs it.
            // Drain: every copy this producer issued has landed before the CTA
            // may exit.  A stage is armed and its copies issued together, and
            // only this producer uses its stages (the ring depth is even), so
            // each of them completes its last armed phase once those land.
            for (int i = 0; i < S; ++i)
                if (issued_mask & (1u << i)) mbar_drain(&full[i], (issued_ph >> i) & 1u, a.status, DEV_TIMEOUT_DRAIN, a.wait_limit);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            uint32_t s = 0, ph = 0, r = 0, rph = 0;
            int it = 0;
            bool ok = true;
            while (ok) {
                if (!mbar_wait(&rfull[r], rph, a.status, DEV_TIMEOUT_MMA_FULL, abort_flag, a.wait_limit)) break;
                const int tile = ring[r];
                mbar_arrive(&rempty[r]);
                if (++r == kRing) { r = 0; rph ^= 1u; }
                if (tile < 0) break;
                const Tile t = decode_tile(a, tile, tstart, off);
                const int buf = it & 1;
                const uint32_t use = static_cast<uint32_t>(it >> 1);
                ++it;
                if (!mbar_wait(&tempty[buf], (use & 1u) ^ 1u, a.status, DEV_TIMEOUT_MMA_TEMPTY, abort_flag, a.wait_limit))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf) * 256u;
                const uint32_t n_mma = t.swap ? static_cast<uint32_t>((t.rows + 31) / 32) * 32u
                                              : static_cast<uint32_t>(a.ph[t.phase].BN);
                const uint32_t idesc = umma_idesc_bf16(128, n_mma);
                for (int kb = t.kb0; kb < t.kb1; ++kb) {
                    if (!mbar_wait(&full[s], ph, a.status, DEV_TIMEOUT_MMA_FULL, abort_flag, a.wait_limit)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t w_base = smem_u32(sW + static_cast<size_t>(s) * a.wslot);
                    const uint32_t x_base = smem_u32(sX + static_cast<size_t>(s) * a.xslot);
                    const uint32_t a_base = t.swap ? w_base : x_base;  // M side: weights or tokens
                    const uint32_t b_base = t.swap ? x_base : w_base;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        umma_bf16(d_tmem, umma_desc_sw128(a_base + kk * 32), umma_desc_sw128(b_base + kk * 32),
                                  idesc, (kb > t.kb0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[s]);
                    if (++s == static_cast<uint32_t>(S)) { s = 0; ph ^= 1u; }
                }
                if (ok) umma_commit(&tfull[buf]);
            }
            // All issued MMAs complete before TMEM is released.
            umma_commit(drain);
            mbar_drain(drain, 0, a.status, DEV_TIMEOUT_DRAIN, a.wait_limit);
        }
    } else if (warp != kProducer1Warp) {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        uint32_t r = 0, rph = 0;
        int it = 0;
        uint32_t nst = 0;  // staged tile stores this warp issued
        for (;;) {
            if (!mbar_wait(&rfull[r], rph, a.status, DEV_TIMEOUT_EPI_TFULL, abort_flag, a.wait_limit)) break;
            const int tile = ring[r];
            __syncwarp();
            if (lane == 0) mbar_arrive(&rempty[r]);
            if (++r == kRing) { r = 0; rph ^= 1u; }
            if (tile < 0) break;
            const Tile t = decode_tile(a, tile, tstart, off);
            const PhaseArgs& pa = a.ph[t.phase];
            const int buf = it & 1;
            const uint32_t use = static_cast<uint32_t>(it >> 1);
            ++it;
            if (!mbar_wait(&tfull[buf], use & 1u, a.status, DEV_TIMEOUT_EPI_TFULL, abort_flag, a.wait_limit)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + static_cast<uint32_t>(buf) * 256u +
                                   (static_cast<uint32_t>(q * 32) << 16);
            float v[32];
            if (!t.swap) {
                const int rr = q * 32 + lane;
                const bool valid = rr < t.rows;
                const int64_t grow = t.row0 + rr;
                const int nchunks = pa.BN / 32;
                // fp32 output of a slab whose 32 rows all belong to the group: staged
                // in shared memory and written by one TMA tile store per chunk
                const bool staged = pa.tma_out && a.stg_bufs > 0 && q * 32 + 32 <= t.rows;
                // H of such a slab: four chunks (64 columns of H) fill one staging
                // buffer, written by one TMA tile store
                const bool staged_h = pa.tma_h && a.stg_bufs > 0 && q * 32 + 32 <= t.rows;
                for (int c = 0; c < nchunks; ++c) {
                    tmem_ld32(taddr + static_cast<uint32_t>(c * 32), v);
                    if (staged_h) {
                        const int sub = c & 3;
                        uint8_t* stg = sStg + static_cast<size_t>(q * a.stg_bufs + static_cast<int>(nst % a.stg_bufs)) * 4096;
                        if (sub == 0) {
                            if (lane == 0) {
                                if (a.stg_bufs > 1) bulk_wait_read<1>(); else bulk_wait_read<0>();
                            }
                            __syncwarp();
                        }
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            pk[i] = pack_bf16x2(silu_f(v[2 * i]) * v[16 + 2 * i],
                                                silu_f(v[2 * i + 1]) * v[16 + 2 * i + 1]);
                        uint8_t* row = stg + lane * 128;
                        *reinterpret_cast<uint4*>(row + (((2 * sub) ^ (lane & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        *reinterpret_cast<uint4*>(row + (((2 * sub + 1) ^ (lane & 7)) << 4)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                        if (sub == 3) {
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) {
                                tma_store_2d(&maps.out[t.phase], stg, t.n0 / 2 + (c >> 2) * 64,
                                             static_cast<int32_t>(t.row0 + q * 32));
                                bulk_commit();
                            }
                            ++nst;
                        }
                        continue;
                    }
                    if (staged) {
                        uint8_t* stg = sStg + static_cast<size_t>(q * a.stg_bufs + static_cast<int>(nst % a.stg_bufs)) * 4096;
                        if (lane == 0) {
                            // the store that last used this buffer has read it
                            if (a.stg_bufs > 1) bulk_wait_read<1>(); else bulk_wait_read<0>();
                        }
                        __syncwarp();
                        stage_row_f32_sw128(stg, lane, v);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&maps.out[t.phase], stg, t.n0 + c * 32,
                                         static_cast<int32_t>(t.split * pa.split_rows + t.row0 + q * 32));
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
                            pk[i] = pack_bf16x2(silu_f(v[2 * i]) * v[16 + 2 * i],
                                                silu_f(v[2 * i + 1]) * v[16 + 2 * i + 1]);
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<bf16*>(pa.out) + grow * pa.ldo +
                                                              (t.n0 / 2 + c * 16));
                        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    } else {
                        const int col0 = t.n0 + c * 32;
                        float* Y = static_cast<float*>(pa.out) + static_cast<int64_t>(t.split) * pa.split_stride +
                                   grow * pa.ldo + col0;
                        if (col0 + 32 <= pa.N_store && (pa.ldo & 3) == 0) {  // float4 rows need 16 B alignment
                            float4* dst = reinterpret_cast<float4*>(Y);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (col0 + i < pa.N_store) Y[i] = v[i];
                        }
                    }
                }
            } else {
                const int nb = (t.rows + 31) / 32;
                for (int c = 0; c < nb; ++c) {
                    tmem_ld32(taddr + static_cast<uint32_t>(c * 32), v);
                    if (pa.epi == EPI_SWIGLU_BF16) {
                        // lane l < 16 holds gate row f0 + l and lane l + 16 the up
                        // row of the same f, each for 32 tokens.  The half-warps
                        // split the tokens: lane l finishes token j, lane l + 16
                        // token j + 16, after one exchange per token pair, so each
                        // lane computes 16 SiLUs and every store writes for both.
                        const bool hi = lane >= 16;
                        const int f = t.n0 / 2 + q * 16 + (lane & 15);
                        const int tok0 = c * 32 + (hi ? 16 : 0);
                        bf16* H = static_cast<bf16*>(pa.out) + (t.row0 + tok0) * pa.ldo + f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float other = __shfl_xor_sync(0xffffffffu, hi ? v[j] : v[j + 16], 16);
                            const float g = hi ? other : v[j];
                            const float u = hi ? v[j + 16] : other;
                            if (tok0 + j < t.rows) H[static_cast<int64_t>(j) * pa.ldo] = __float2bfloat16_rn(silu_f(g) * u);
                        }
                    } else {
                        float* Y = static_cast<float*>(pa.out) + static_cast<int64_t>(t.split) * pa.split_stride;
                        const int col = t.n0 + q * 32 + lane;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int tok = c * 32 + j;
                            if (tok < t.rows && col < pa.N_store) Y[(t.row0 + tok) * pa.ldo + col] = v[j];
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&tempty[buf]);
                if (t.phase == 0 && a.dep) {
                    // publish this warp's rows of H to the phase-1 tiles of group g
                    // (rows written by TMA tile stores must have landed first)
                    if (pa.tma_h) bulk_wait_all();
                    fence_proxy_async_global();
                    __threadfence();
                    atomicAdd(&a.sched[1 + t.g], 1);
                }
            }
        }
    }

    // staged output stores complete (and stop reading shared memory) before the CTA exits
    if (warp >= 2 && warp != kProducer1Warp && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ----------------------------------------------------------------- host

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// 2D bf16 map over [rows, cols] (cols contiguous) with box {64, box_rows} and
// the 128-byte swizzle that the UMMA descriptors expect.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows < 1 ? 1 : rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

// 2D output map over [rows, cols] (cols contiguous, row stride ld elements)
// with a box of 32 rows x 128 bytes (32 fp32 or 64 bf16 columns) and the
// 128-byte swizzle of the staged output tiles.
bool make_out_map(CUtensorMap* m, void* base, uint64_t rows, uint64_t cols, uint64_t ld, bool bf16_out) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows < 1 ? 1 : rows};
    cuuint64_t strides[1] = {ld * (bf16_out ? 2 : 4)};
    cuuint32_t box[2] = {bf16_out ? 64u : 32u, 32u};  // 128 bytes of a row
    cuuint32_t es[2] = {1, 1};
    return enc(m, bf16_out ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims,
               strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Whether a phase's fp32 output can take staged TMA tile stores: full-width
// rows (no clipped columns), 16-byte aligned rows and base, partial slices a
// whole number of rows apart.
bool out_map_ok(const GemmPhase& g) {
    return g.epi == EPI_F32 && g.out != nullptr && g.N_store == g.N && g.N % 32 == 0 && g.ldo % 4 == 0 &&
           g.ldo >= g.N && (reinterpret_cast<uintptr_t>(g.out) & 15u) == 0 &&
           (g.ksplit <= 1 || g.split_stride % g.ldo == 0);
}

// Whether a SwiGLU phase's bf16 H can take staged TMA tile stores (token-major
// tiles of BN = 128 or 256, so four chunks make whole 64-column boxes).
bool h_map_ok(const GemmPhase& g) {
    return g.epi == EPI_SWIGLU_BF16 && g.out != nullptr && g.ksplit <= 1 && g.ldo % 8 == 0 && g.N % 128 == 0 &&
           (reinterpret_cast<uintptr_t>(g.out) & 15u) == 0;
}

// Rows of the output map of a phase that out_map_ok accepts (every partial slice).
uint64_t out_map_rows(const GemmPhase& g, int ksplit) {
    const int64_t split_rows = ksplit > 1 ? g.split_stride / g.ldo : 0;
    return static_cast<uint64_t>(static_cast<int64_t>(ksplit - 1) * split_rows + g.tok_rows);
}

int num_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    static int cached[64] = {0};
    if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    if (dev >= 0 && dev < 64) cached[dev] = n;
    return n;
}

// Scheduler words: a tile counter, one readiness counter per group, and the
// CTA-pair kernel's second (weight-major) tile counter.
size_t gemm_sched_bytes(int G) { return static_cast<size_t>(G + 2) * sizeof(int); }

// Returns 0 on success, -2 for an unsupported shape, -3 for a CUDA failure.
// L.sched must point at gemm_sched_bytes(G) bytes that are zero when the
// kernel starts.
int launch_grouped_gemm(const GemmLaunch& L, cudaStream_t st) {
    if (L.G < 1 || L.G > kMaxGroups || L.nphase < 1 || L.nphase > 2 || !L.sched) return -2;
    DevArgs a{};
    a.group_off = L.group_off;
    a.G = L.G;
    a.dense_rows = L.dense_rows;
    a.nphase = L.nphase;
    a.dep = (L.nphase == 2) ? 1 : 0;
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
    bool any_swap_possible = false;
    uint32_t wslot = 0, xslot = kTileABytes;
    for (int p = 0; p < L.nphase; ++p) {
        const GemmPhase& g = L.ph[p];
        if (g.Kdim < 16 || g.Kdim % 8 != 0 || g.N < 32) return -2;
        PhaseArgs& ph = a.ph[p];
        ph.w = g.w;
        ph.w_group_elems = static_cast<int64_t>((g.N + 127) / 128) * ((g.Kdim + kBK - 1) / kBK) * 8192;
        if ((reinterpret_cast<uintptr_t>(g.w) & 15u) != 0) return -2;
        ph.N = g.N;
        ph.N_store = g.N_store;
        ph.k_blocks = (g.Kdim + kBK - 1) / kBK;
        ph.epi = g.epi;
        ph.out = g.out;
        ph.ldo = g.ldo;
        ph.split_stride = g.split_stride;
        // Token-major tiles take the widest BN that divides N.  When groups
        // are expected to be small (mean below 128 rows) BN is capped at 128,
        // so a weight slot is the same 16 KB a weight-major tile needs and
        // the operand ring stays deep.
        int bn_cap = L.small_groups ? 128 : 256;
        if (L.bn_max > 0 && L.bn_max < bn_cap) bn_cap = L.bn_max;
        int bn = 0;
        for (int c : {256, 128, 64, 32})
            if (c <= bn_cap && g.N % c == 0) { bn = c; break; }
        if (bn == 0) return -2;
        if (g.epi == EPI_SWIGLU_BF16 && (g.N % 32 != 0 || g.ksplit > 1)) return -2;
        ph.BN = bn;
        int ks = g.ksplit < 1 ? 1 : g.ksplit;
        if (ks > ph.k_blocks) ks = ph.k_blocks;
        ph.kb_per_split = (ph.k_blocks + ks - 1) / ks;
        ph.ksplit = (ph.k_blocks + ph.kb_per_split - 1) / ph.kb_per_split;
        wslot = wslot > static_cast<uint32_t>(bn) * 128u ? wslot : static_cast<uint32_t>(bn) * 128u;
        if (g.N % 128 == 0 && a.swap_max_rows > 0) any_swap_possible = true;
    }
    if (any_swap_possible) {
        if (wslot < kTileABytes) wslot = kTileABytes;
        const uint32_t xs = static_cast<uint32_t>(a.BNs) * 128u;
        if (xs > xslot) xslot = xs;
    }
    a.wslot = wslot;
    a.xslot = xslot;
    const size_t fixed = 1024 + static_cast<size_t>(2 * 16 + 4 + 2 * kRing + 1) * 8 + kRing * 4 + 16 +
                         static_cast<size_t>(L.G + 1) * (8 + 2 * 4) + 64;
    const size_t budget = 227 * 1024 - fixed;
    // even: each of the two producers owns the stages of one parity
    auto ring_stages = [&](size_t bytes) { return std::min(static_cast<int>(bytes / (wslot + xslot)), 16) & ~1; };
    const int stages = ring_stages(budget);
    if (stages < 2) return -2;
    a.stages = stages;
    // Output staging for fp32 token-major tiles (4 epilogue warps x 4 KB per
    // buffer): two buffers per warp, else one, where the ring keeps its depth.
    bool want_stg = false;
    for (int p = 0; p < L.nphase; ++p) want_stg = want_stg || out_map_ok(L.ph[p]) || h_map_ok(L.ph[p]);
    a.stg_bufs = 0;
    for (int nb = 2; want_stg && nb >= 1 && a.stg_bufs == 0; --nb) {
        const size_t stg = static_cast<size_t>(nb) * 4 * 4096;
        if (budget > stg && ring_stages(budget - stg) == stages) a.stg_bufs = nb;
    }
    const size_t smem = fixed + static_cast<size_t>(stages) * (wslot + xslot) + static_cast<size_t>(a.stg_bufs) * 4 * 4096;

    Maps maps;
    std::memset(&maps, 0, sizeof(maps));
    for (int p = 0; p < L.nphase; ++p) {
        const GemmPhase& g = L.ph[p];
        const uint64_t tok_rows = static_cast<uint64_t>(g.tok_rows < 1 ? 1 : g.tok_rows);
        if (!make_map(&maps.tokA[p], g.tok, tok_rows, g.Kdim, 128u)) return -3;
        if (!make_map(&maps.tokB[p], g.tok, tok_rows, g.Kdim, 32u)) return -3;
        PhaseArgs& ph = a.ph[p];
        ph.tma_out = (a.stg_bufs > 0 && out_map_ok(g)) ? 1 : 0;
        ph.tma_h = (a.stg_bufs > 0 && h_map_ok(g) && ph.BN % 128 == 0) ? 1 : 0;
        ph.split_rows = ph.tma_out && ph.ksplit > 1 ? g.split_stride / g.ldo : 0;
        if (ph.tma_out && !make_out_map(&maps.out[p], g.out, out_map_rows(g, ph.ksplit), g.N, g.ldo, false)) return -3;
        if (ph.tma_h && !make_out_map(&maps.out[p], g.out, static_cast<uint64_t>(g.tok_rows), g.N / 2, g.ldo, true))
            return -3;
    }

    static std::atomic<unsigned long long> attr_done{0};
    if (smem_attr_once(reinterpret_cast<const void*>(grouped_gemm_kernel), 227 * 1024, attr_done) != 0) return -3;
    const int sms = num_sms();
    if (sms <= 0) return -3;
    // Upper bound on the tile count, to avoid idle CTAs on tiny problems.
    int64_t bound = 0;
    for (int p = 0; p < L.nphase; ++p) {
        const GemmPhase& g = L.ph[p];
        const int64_t rows_total = L.group_off ? g.tok_rows : L.dense_rows;
        const int64_t tm = ((rows_total + 127) / 128 + L.G) * (g.N / a.ph[p].BN) * a.ph[p].ksplit;
        const int64_t sw =
            (g.N % 128 == 0) ? ((rows_total + a.BNs - 1) / a.BNs + L.G) * (g.N / 128) * a.ph[p].ksplit : 0;
        bound += tm > sw ? tm : sw;
    }
    const int grid = static_cast<int>(bound < sms ? (bound < 1 ? 1 : bound) : sms);
    if (launch_pdl(grouped_gemm_kernel, dim3(grid), dim3(kThreads), smem, st, maps, a) != cudaSuccess) return -3;
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace moe
