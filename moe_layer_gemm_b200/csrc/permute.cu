// Dispatch: group the (token, slot) assignments by expert, in token order,
// with an optional per-expert capacity.
//
// "MoE computation notes" (cf-1.com/news/5905749), section 2.1: permute the
// tokens so those going to one expert are adjacent, using sort and cumsum
// offsets; section 3.1: an expert keeps at most C = CF * T * K / E
// assignments and the overflow is dropped.
//
// The rank of (t, k) on expert e is the number of assignments (t', k')
// before it in token-major order that chose e: the earlier tokens that chose
// e, plus the earlier slots of the same token if it lists e more than once
// (the router never does; such a token is treated as separate assignments).
// It is assembled from exact integer counts, never from the order in which
// atomics happen to land:
//   base of the block (earlier blocks)  + earlier warps of the block
//   + earlier lanes of the warp (one __match_any_sync per slot)
//   + earlier slots of the same token.
// Kept iff rank < C; row = offsets[e] + rank.
//
// An index outside [0, E) is never used as an address: the slot is skipped
// (not counted, inv = -1) and DEV_BAD_INDEX is recorded in the status word
// when the caller passed one.
//
// Batches of at most kSmallT tokens take one fused single-CTA kernel
// (count, scan, rank); larger ones take hist -> scan -> rank over many CTAs.
// A gather kernel then copies each token row once per kept slot with
// 16-byte loads, all of a lane's loads issued before its stores.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kTokPerBlock = 256;  // one token per thread in hist/rank
constexpr int kMaxE = 256;
constexpr int kMaxK = 16;
constexpr int kSmallThreads = 1024;
constexpr int kSmallT = 1024;

// Per-warp table used to count, for each of this lane's experts, the earlier
// lanes of the warp that chose the same expert in any slot.
struct WarpTable {
    unsigned* mask;  // [E]
    int* tag;        // [E]
};

// Expert of slot (t, k), or -1 (and the status recorded) when the caller's
// index lies outside [0, E).
__device__ __forceinline__ int checked_expert(const int32_t* idx, int64_t i, int E, int* status) {
    const int e = idx[i];
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) return e;
    if (status) atomicCAS(status, 0, DEV_BAD_INDEX);
    return -1;
}

// pre[k] = slots of earlier lanes of the warp, and earlier slots of this
// lane, that chose my[k] (slots with my[k] < 0 are ignored).
__device__ __forceinline__ void warp_prefix(const int (&my)[kMaxK], int K, int lane, WarpTable tab, int gen,
                                            int (&pre)[kMaxK]) {
    const unsigned lt = (1u << lane) - 1u;
    for (int k = 0; k < K; ++k) {
        pre[k] = 0;
        for (int k2 = 0; k2 < k; ++k2) pre[k] += (my[k2] == my[k]) ? 1 : 0;
    }
    for (int k2 = 0; k2 < K; ++k2) {
        const int v = my[k2];
        const unsigned m = __match_any_sync(0xffffffffu, v);
        if (v >= 0) {  // lanes with the same v write the same mask
            tab.mask[v] = m;
            tab.tag[v] = gen + k2;
        }
        __syncwarp();
        for (int k = 0; k < K; ++k) {
            const int e = my[k];
            if (e >= 0 && tab.tag[e] == gen + k2) pre[k] += __popc(tab.mask[e] & lt);
        }
        __syncwarp();
    }
}

__global__ void __launch_bounds__(kTokPerBlock)
hist_kernel(const int32_t* __restrict__ idx, int64_t T, int E, int K, int32_t* __restrict__ block_hist,
            int* __restrict__ status) {
    __shared__ int32_t h[kMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kTokPerBlock + threadIdx.x;
    if (t < T)
        for (int k = 0; k < K; ++k) {
            const int e = checked_expert(idx, t * K + k, E, status);
            if (e >= 0) atomicAdd(&h[e], 1);  // integer counts: order-free
        }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) block_hist[static_cast<int64_t>(blockIdx.x) * E + e] = h[e];
}

// One block of 1024 threads.  block_hist is rewritten in place with each
// block's rank base: per expert, an exclusive scan over the blocks.  Warp w
// takes experts w, w + 32, .. (up to 8 at once); its lanes take 32 blocks at
// a time, all loads issued before the warp scans, so a column of blocks costs
// one round of memory latency per 32 blocks instead of one per block.
constexpr int kScanExpertsPerWarp = kMaxE / 32;

__global__ void __launch_bounds__(1024)
scan_kernel(int32_t* __restrict__ block_hist, int nblocks, int E, int64_t C, int32_t* __restrict__ counts,
            int32_t* __restrict__ kept, int32_t* __restrict__ offsets, int32_t* __restrict__ n_dropped,
            int32_t* __restrict__ zero_out, int zero_count) {
    for (int i = threadIdx.x; i < zero_count; i += blockDim.x) zero_out[i] = 0;  // next kernel's scheduler words
    __shared__ int32_t sk[kMaxE];
    __shared__ int32_t sdrop[kMaxE];
    {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
        int carry[kScanExpertsPerWarp];
#pragma unroll
        for (int i = 0; i < kScanExpertsPerWarp; ++i) carry[i] = 0;
        for (int b0 = 0; b0 < nblocks; b0 += 32) {
            const int b = b0 + lane;
            int v[kScanExpertsPerWarp];
#pragma unroll
            for (int i = 0; i < kScanExpertsPerWarp; ++i) {
                const int e = warp + nw * i;
                v[i] = (e < E && b < nblocks) ? block_hist[static_cast<int64_t>(b) * E + e] : 0;
            }
#pragma unroll
            for (int i = 0; i < kScanExpertsPerWarp; ++i) {
                const int e = warp + nw * i;
                int incl = v[i];
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += u;
                }
                if (e < E && b < nblocks) block_hist[static_cast<int64_t>(b) * E + e] = carry[i] + incl - v[i];
                carry[i] += __shfl_sync(0xffffffffu, incl, 31);
            }
        }
        if (lane == 0)
#pragma unroll
            for (int i = 0; i < kScanExpertsPerWarp; ++i) {
                const int e = warp + nw * i;
                if (e >= E) continue;
                const int32_t run = carry[i];
                const int32_t kp = (C >= 0 && run > C) ? static_cast<int32_t>(C) : run;
                counts[e] = run;
                kept[e] = kp;
                sk[e] = kp;
                sdrop[e] = run - kp;
            }
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // warp-level exclusive scan over E <= 256 (8 per lane)
        const int lane = threadIdx.x;
        const int per = (E + 31) / 32;
        int s = 0, dsum = 0;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) { s += sk[e]; dsum += sdrop[e]; }
        }
        int incl = s;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - s;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) { offsets[e] = run; run += sk[e]; }
        }
        for (int o = 16; o >= 1; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
        if (lane == 31) offsets[E] = incl;
        if (lane == 0 && n_dropped) *n_dropped = dsum;
    }
}

__global__ void __launch_bounds__(kTokPerBlock)
rank_kernel(const int32_t* __restrict__ idx, int64_t T, int E, int K, int64_t C,
            const int32_t* __restrict__ block_base, const int32_t* __restrict__ offsets,
            int32_t* __restrict__ inv, int32_t* __restrict__ src, int* __restrict__ status) {
    constexpr int W = kTokPerBlock / 32;
    __shared__ int32_t wh[W][kMaxE];
    __shared__ unsigned tmask[W][kMaxE];
    __shared__ int tag[W][kMaxE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kTokPerBlock + threadIdx.x;
    const bool live = t < T;
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) {
        wh[i / E][i % E] = 0;
        tag[i / E][i % E] = 0;
    }
    __syncthreads();
    int my[kMaxK];
    for (int k = 0; k < K; ++k) {
        my[k] = live ? checked_expert(idx, t * K + k, E, status) : -1;
        if (my[k] >= 0) atomicAdd(&wh[warp][my[k]], 1);
    }
    int pre[kMaxK];
    warp_prefix(my, K, lane, WarpTable{tmask[warp], tag[warp]}, 1, pre);
    __syncthreads();
    if (!live) return;
    for (int k = 0; k < K; ++k) {
        const int e = my[k];
        if (e < 0) {
            inv[t * K + k] = -1;
            continue;
        }
        int32_t r = block_base[static_cast<int64_t>(blockIdx.x) * E + e] + pre[k];
        for (int w2 = 0; w2 < warp; ++w2) r += wh[w2][e];
        if (C < 0 || r < C) {
            const int32_t row = offsets[e] + r;
            inv[t * K + k] = row;
            src[row] = static_cast<int32_t>(t);
        } else {
            inv[t * K + k] = -1;
        }
    }
}

// Whole dispatch of a batch of T <= kSmallT tokens in one CTA.
__global__ void __launch_bounds__(kSmallThreads)
dispatch_small_kernel(const int32_t* __restrict__ idx, int T, int E, int K, int64_t C,
                      int32_t* __restrict__ counts, int32_t* __restrict__ kept, int32_t* __restrict__ offsets,
                      int32_t* __restrict__ inv, int32_t* __restrict__ src, int32_t* __restrict__ n_dropped,
                      int32_t* __restrict__ zero_out, int zero_count, int* __restrict__ status) {
    constexpr int W = kSmallThreads / 32;
    for (int i = threadIdx.x; i < zero_count; i += blockDim.x) zero_out[i] = 0;  // next kernel's scheduler words
    extern __shared__ int32_t sm[];
    int32_t* wh = sm;                                              // [W][E]
    unsigned* tmask = reinterpret_cast<unsigned*>(wh + W * E);     // [W][E]
    int* tag = reinterpret_cast<int*>(tmask + W * E);              // [W][E]
    int32_t* soff = tag + W * E;                                   // [E+1]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = threadIdx.x;
    const bool live = t < T;
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) {
        wh[i] = 0;
        tag[i] = 0;
    }
    __syncthreads();
    int my[kMaxK];
    for (int k = 0; k < K; ++k) {
        my[k] = live ? checked_expert(idx, static_cast<int64_t>(t) * K + k, E, status) : -1;
        if (my[k] >= 0) atomicAdd(&wh[warp * E + my[k]], 1);
    }
    int pre[kMaxK];
    warp_prefix(my, K, lane, WarpTable{tmask + warp * E, tag + warp * E}, 1, pre);
    __syncthreads();
    if (warp == 0) {
        // totals, capacity, exclusive scan of kept counts, drops
        const int per = (E + 31) / 32;
        int s = 0, dsum = 0;
        int kp_local[8];
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            int kp = 0;
            if (e < E) {
                int c = 0;
                for (int w2 = 0; w2 < W; ++w2) c += wh[w2 * E + e];
                kp = (C >= 0 && c > C) ? static_cast<int>(C) : c;
                counts[e] = c;
                kept[e] = kp;
                dsum += c - kp;
            }
            kp_local[i] = kp;
            s += kp;
        }
        int incl = s;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - s;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) {
                soff[e] = run;
                offsets[e] = run;
            }
            run += kp_local[i];
        }
        for (int o = 16; o >= 1; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
        if (lane == 31) offsets[E] = incl;
        if (lane == 0 && n_dropped) *n_dropped = dsum;
    }
    __syncthreads();
    if (!live) return;
    for (int k = 0; k < K; ++k) {
        const int e = my[k];
        if (e < 0) {
            inv[t * K + k] = -1;
            continue;
        }
        int r = pre[k];
        for (int w2 = 0; w2 < warp; ++w2) r += wh[w2 * E + e];
        if (C < 0 || r < C) {
            const int row = soff[e] + r;
            inv[t * K + k] = row;
            src[row] = t;
        } else {
            inv[t * K + k] = -1;
        }
    }
}

constexpr int kGatherBatch = 8;

__global__ void __launch_bounds__(256)
gather_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ inv, int64_t T, int d, int K,
              int parts, __nv_bfloat16* __restrict__ x_perm) {
    // `parts` warps share one token row, each copying a contiguous slice
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
    const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int nvec = d / 8;
    const int slice = (nvec + parts - 1) / parts;
    for (int64_t job = gw; job < T * parts; job += nw) {
        const int64_t t = job / parts;
        const int p = static_cast<int>(job - t * parts);
        int32_t rows[kMaxK];
        int nr = 0;
        for (int k = 0; k < K; ++k) {
            const int32_t r = inv[t * K + k];
            if (r >= 0) rows[nr++] = r;
        }
        if (nr == 0) continue;
        const uint4* s = reinterpret_cast<const uint4*>(x + t * d);
        const int c_end = min(nvec, (p + 1) * slice);
        for (int c0 = p * slice + lane; c0 < c_end; c0 += 32 * kGatherBatch) {
            uint4 v[kGatherBatch];
#pragma unroll
            for (int b = 0; b < kGatherBatch; ++b) {
                const int c = c0 + 32 * b;
                if (c < c_end) v[b] = __ldg(s + c);
            }
            for (int i = 0; i < nr; ++i) {
                uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(rows[i]) * d);
#pragma unroll
                for (int b = 0; b < kGatherBatch; ++b) {
                    const int c = c0 + 32 * b;
                    if (c < c_end) dst[c] = v[b];
                }
            }
        }
    }
}

// Dispatch and row gather of a batch of T <= kSmallT tokens in one launch
// (the layer's path; moe_permute keeps the two-kernel form).  Every CTA
// computes the whole dispatch in shared memory, exactly as
// dispatch_small_kernel does (same counts, ranks and rows); CTA 0 also
// writes the results out.  Each CTA then copies its share of (token, slice)
// jobs straight from its shared copy of the rows, so the gather needs no
// second launch and no global read of inv.
__global__ void __launch_bounds__(kSmallThreads)
dispatch_gather_small_kernel(const int32_t* __restrict__ idx, const __nv_bfloat16* __restrict__ x, int T, int d,
                             int E, int K, int64_t C, int parts, int32_t* __restrict__ counts,
                             int32_t* __restrict__ kept, int32_t* __restrict__ offsets, int32_t* __restrict__ inv,
                             int32_t* __restrict__ src, int32_t* __restrict__ n_dropped,
                             __nv_bfloat16* __restrict__ x_perm, int32_t* __restrict__ zero_out, int zero_count,
                             int* __restrict__ status) {
    pdl_trigger();
    pdl_wait();
    constexpr int W = kSmallThreads / 32;
    const bool writer = blockIdx.x == 0;
    if (writer)
        for (int i = threadIdx.x; i < zero_count; i += blockDim.x) zero_out[i] = 0;  // next kernel's scheduler words
    extern __shared__ int32_t sm[];
    int32_t* wh = sm;                                              // [W][E]
    unsigned* tmask = reinterpret_cast<unsigned*>(wh + W * E);     // [W][E]
    int* tag = reinterpret_cast<int*>(tmask + W * E);              // [W][E]
    int32_t* soff = tag + W * E;                                   // [E+1]
    int32_t* srow = soff + E + 1;                                  // [T][K] row of (t, k), or -1
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = threadIdx.x;
    const bool live = t < T;
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) {
        wh[i] = 0;
        tag[i] = 0;
    }
    __syncthreads();
    int my[kMaxK];
    for (int k = 0; k < K; ++k) {
        my[k] = live ? checked_expert(idx, static_cast<int64_t>(t) * K + k, E, status) : -1;
        if (my[k] >= 0) atomicAdd(&wh[warp * E + my[k]], 1);
    }
    int pre[kMaxK];
    warp_prefix(my, K, lane, WarpTable{tmask + warp * E, tag + warp * E}, 1, pre);
    __syncthreads();
    if (warp == 0) {
        // totals, capacity, exclusive scan of kept counts, drops
        const int per = (E + 31) / 32;
        int s = 0, dsum = 0;
        int kp_local[8];
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            int kp = 0;
            if (e < E) {
                int c = 0;
                for (int w2 = 0; w2 < W; ++w2) c += wh[w2 * E + e];
                kp = (C >= 0 && c > C) ? static_cast<int>(C) : c;
                if (writer) {
                    counts[e] = c;
                    kept[e] = kp;
                }
                dsum += c - kp;
            }
            kp_local[i] = kp;
            s += kp;
        }
        int incl = s;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - s;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) {
                soff[e] = run;
                if (writer) offsets[e] = run;
            }
            run += kp_local[i];
        }
        for (int o = 16; o >= 1; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
        if (writer && lane == 31) offsets[E] = incl;
        if (writer && lane == 0 && n_dropped) *n_dropped = dsum;
    }
    __syncthreads();
    if (live) {
        for (int k = 0; k < K; ++k) {
            const int e = my[k];
            int r = pre[k];
            if (e >= 0)
                for (int w2 = 0; w2 < warp; ++w2) r += wh[w2 * E + e];
            const int row = (e >= 0 && (C < 0 || r < C)) ? soff[e] + r : -1;
            srow[t * K + k] = row;
            if (writer) {
                inv[t * K + k] = row;
                if (row >= 0) src[row] = t;
            }
        }
    }
    __syncthreads();
    // gather: job (token, slice) j = blockIdx.x + gridDim.x * (warp + W * i)
    const int nvec = d / 8;
    const int slice = (nvec + parts - 1) / parts;
    const int jobs = T * parts;
    for (int job = blockIdx.x + gridDim.x * warp; job < jobs; job += gridDim.x * W) {
        const int tt = job / parts;
        const int p = job - tt * parts;
        const uint4* sx = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(tt) * d);
        const int c_end = min(nvec, (p + 1) * slice);
        for (int c0 = p * slice + lane; c0 < c_end; c0 += 32 * kGatherBatch) {
            uint4 v[kGatherBatch];
#pragma unroll
            for (int b = 0; b < kGatherBatch; ++b) {
                const int c = c0 + 32 * b;
                if (c < c_end) v[b] = __ldg(sx + c);
            }
            for (int k = 0; k < K; ++k) {
                const int row = srow[tt * K + k];
                if (row < 0) continue;
                uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(row) * d);
#pragma unroll
                for (int b = 0; b < kGatherBatch; ++b) {
                    const int c = c0 + 32 * b;
                    if (c < c_end) dst[c] = v[b];
                }
            }
        }
    }
}

}  // namespace

int permute_blocks(int64_t T) { return static_cast<int>((T + kTokPerBlock - 1) / kTokPerBlock); }

int launch_permute(const int32_t* idx, const bf16* x, int64_t T, int d, int E, int K, int64_t C,
                   int32_t* block_hist, int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* inv,
                   int32_t* src, bf16* x_perm, int32_t* n_dropped, int32_t* zero_out, int zero_count,
                   int* status, cudaStream_t st) {
    if (E > kMaxE || K > kMaxK) return -2;
    if (T <= kSmallT) {
        const size_t smem = static_cast<size_t>(3 * (kSmallThreads / 32) * E + E + 1) * 4;
        static std::atomic<unsigned long long> attr_done{0};
        if (smem_attr_once(reinterpret_cast<const void*>(dispatch_small_kernel),
                           (3 * (kSmallThreads / 32) * kMaxE + kMaxE + 1) * 4, attr_done) != 0)
            return -3;
        dispatch_small_kernel<<<1, kSmallThreads, smem, st>>>(idx, static_cast<int>(T), E, K, C, counts, kept,
                                                              offsets, inv, src, n_dropped, zero_out, zero_count,
                                                              status);
    } else {
        const int nb = permute_blocks(T);
        hist_kernel<<<nb, kTokPerBlock, 0, st>>>(idx, T, E, K, block_hist, status);
        scan_kernel<<<1, 1024, 0, st>>>(block_hist, nb, E, C, counts, kept, offsets, n_dropped, zero_out,
                                        zero_count);
        rank_kernel<<<nb, kTokPerBlock, 0, st>>>(idx, T, E, K, C, block_hist, offsets, inv, src, status);
    }
    if (x != nullptr && x_perm != nullptr) {
        const int sms = num_sms() > 0 ? num_sms() : 148;
        // enough warps to cover the machine a few times over
        int parts = 1;
        while (parts < 16 && T * parts < static_cast<int64_t>(sms) * 32 && (d / 8) / (parts * 2) >= 32) parts *= 2;
        const int64_t jobs = T * parts;
        const int64_t need = (jobs + 7) / 8;
        const int grid = static_cast<int>(need < sms * 16 ? need : sms * 16);
        gather_kernel<<<grid, 256, 0, st>>>(x, inv, T, d, K, parts, x_perm);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

int launch_count(int64_t T) { return T <= kSmallT ? 1 : 3; }

bool dispatch_gather_fused_supported(int64_t T, int E, int K) { return T <= kSmallT && E <= kMaxE && K <= kMaxK; }

int launch_dispatch_gather_small(const int32_t* idx, const bf16* x, int64_t T, int d, int E, int K, int64_t C,
                                 int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* inv, int32_t* src,
                                 bf16* x_perm, int32_t* n_dropped, int32_t* zero_out, int zero_count,
                                 int* status, cudaStream_t st) {
    if (!dispatch_gather_fused_supported(T, E, K) || !x || !x_perm || d % 8 != 0) return -2;
    const size_t smem = static_cast<size_t>(3 * (kSmallThreads / 32) * E + E + 1 + T * K) * 4;
    static std::atomic<unsigned long long> attr_done{0};
    if (smem_attr_once(reinterpret_cast<const void*>(dispatch_gather_small_kernel),
                       (3 * (kSmallThreads / 32) * kMaxE + kMaxE + 1 + kSmallT * kMaxK) * 4, attr_done) != 0)
        return -3;
    const int sms = num_sms() > 0 ? num_sms() : 148;
    // (token, slice) jobs: enough for every warp of the grid
    int parts = 1;
    while (parts < 16 && T * parts < static_cast<int64_t>(sms) * 32 && (d / 8) / (parts * 2) >= 32) parts *= 2;
    const int64_t jobs = T * parts;
    const int64_t need = (jobs + (kSmallThreads / 32) - 1) / (kSmallThreads / 32);
    const int grid = static_cast<int>(need < sms ? (need < 1 ? 1 : need) : sms);
    (void)launch_pdl(dispatch_gather_small_kernel, dim3(grid), dim3(kSmallThreads), smem, st, idx, x,
                     static_cast<int>(T), d, E, K, C, parts, counts, kept, offsets, inv, src, n_dropped, x_perm,
                     zero_out, zero_count, status);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

// ------------------------------------------------------------------------
// Dispatch without a caller-provided workspace.
//
// The only scratch the dispatch kernels need is the per-block histogram /
// rank-base table (ceil(T/256) x E int32).  Here it lives in a file-scope
// device array that every GPU loading this library holds until the process
// exits.  All calls share it: each call writes every element it reads
// before reading it, so nothing has to be cleared between calls, but two
// calls whose kernels overlap on the same GPU (different streams) race on
// it.  Host code cannot use the array's name as a device address; its
// address is looked up once per device with cudaGetSymbolAddress.
namespace {

constexpr int64_t kStaticHistInts = int64_t(1) << 16;  // 256 KB
static __device__ __align__(256) int32_t g_dispatch_scratch[kStaticHistInts];

std::mutex g_scratch_mutex;
void* g_scratch_addr[64] = {nullptr};

// Device address of g_dispatch_scratch on the current device, looked up on
// first use; nullptr if the lookup fails.
int32_t* dispatch_scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return static_cast<int32_t*>(g_scratch_addr[dev]);
}

}  // namespace

int64_t permute_static_max_hist() { return kStaticHistInts; }

// -2: the batch needs more scratch than the static array holds; -3: CUDA failure.
int launch_permute_static(const int32_t* idx, const bf16* x, int64_t T, int d, int E, int K, int64_t C,
                          int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* inv, int32_t* src,
                          bf16* x_perm, int32_t* n_dropped, cudaStream_t st) {
    if (static_cast<int64_t>(permute_blocks(T)) * E > kStaticHistInts) return -2;
    int32_t* scratch = dispatch_scratch_address();
    if (scratch == nullptr) return -3;
    return launch_permute(idx, x, T, d, E, K, C, scratch, counts, kept, offsets, inv, src, x_perm, n_dropped,
                          nullptr, 0, nullptr, st);
}

}  // namespace moe
