// Dispatch: group the (token, slot) assignments by expert, in token order,
// with an optional per-expert capacity.
//
// "MoE computation notes" (cf-1.com/news/5905749), section 2.1: permute the
// tokens so those going to one expert are adjacent, using sort and cumsum
// offsets; section 3.1: an expert keeps at most C = CF * T * K / E
// assignments and the overflow is dropped.
//
// Four launches, no atomics in any ordering decision:
//   1. hist:   block b counts its tokens' selections per expert
//   2. scan:   per expert, exclusive scan over blocks (rank base of block b),
//              totals = counts, kept = min(counts, C), offsets = exclusive
//              cumsum of kept, n_dropped
//   3. rank:   each (t, k) gets rank = (# earlier tokens choosing the same
//              expert): block base + earlier warps of the block + earlier
//              lanes of the warp.  Kept iff rank < C; row = offsets[e] + rank
//   4. gather: one warp per token reads x[t] once with 16-byte loads and
//              writes it to each of its kept rows
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "internal.h"

namespace moe {

namespace {

constexpr int kTokPerBlock = 256;  // one token per thread in hist/rank
constexpr int kMaxE = 1024;

__global__ void __launch_bounds__(kTokPerBlock)
hist_kernel(const int32_t* __restrict__ idx, int64_t T, int E, int K, int32_t* __restrict__ block_hist) {
    __shared__ int32_t h[kMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kTokPerBlock + threadIdx.x;
    if (t < T)
        for (int k = 0; k < K; ++k) atomicAdd(&h[idx[t * K + k]], 1);  // integer counts: order-free
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) block_hist[static_cast<int64_t>(blockIdx.x) * E + e] = h[e];
}

// One block of 1024 threads.  block_hist is rewritten in place with each
// block's rank base.
__global__ void __launch_bounds__(1024)
scan_kernel(int32_t* __restrict__ block_hist, int nblocks, int E, int64_t C, int32_t* __restrict__ counts,
            int32_t* __restrict__ kept, int32_t* __restrict__ offsets, int32_t* __restrict__ n_dropped) {
    __shared__ int32_t sk[kMaxE];
    __shared__ int32_t sdrop[kMaxE];
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t run = 0;
        for (int b = 0; b < nblocks; ++b) {
            const int64_t i = static_cast<int64_t>(b) * E + e;
            const int32_t c = block_hist[i];
            block_hist[i] = run;
            run += c;
        }
        const int32_t kp = (C >= 0 && run > C) ? static_cast<int32_t>(C) : run;
        counts[e] = run;
        kept[e] = kp;
        sk[e] = kp;
        sdrop[e] = run - kp;
    }
    __syncthreads();
    if (threadIdx.x == 0) {  // E <= 1024: a serial exclusive scan is a few microseconds at most
        int32_t run = 0, dr = 0;
        for (int e = 0; e < E; ++e) {
            offsets[e] = run;
            run += sk[e];
            dr += sdrop[e];
        }
        offsets[E] = run;
        if (n_dropped) *n_dropped = dr;
    }
}

__global__ void __launch_bounds__(kTokPerBlock)
rank_kernel(const int32_t* __restrict__ idx, int64_t T, int E, int K, int64_t C,
            const int32_t* __restrict__ block_base, const int32_t* __restrict__ offsets,
            int32_t* __restrict__ inv, int32_t* __restrict__ src) {
    constexpr int W = kTokPerBlock / 32;
    constexpr int kMaxK = 16;
    __shared__ int32_t wh[W][kMaxE / 4];  // per-warp histograms for E <= 256
    __shared__ int32_t ids[W][32][kMaxK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kTokPerBlock + threadIdx.x;
    const bool live = t < T;
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) wh[i / E][i % E] = 0;
    __syncthreads();
    int my[kMaxK];
    for (int k = 0; k < K; ++k) {
        my[k] = live ? idx[t * K + k] : -1;
        ids[warp][lane][k] = my[k];
        if (live) atomicAdd(&wh[warp][my[k]], 1);
    }
    __syncthreads();
    if (!live) return;
    for (int k = 0; k < K; ++k) {
        const int e = my[k];
        int32_t r = block_base[static_cast<int64_t>(blockIdx.x) * E + e];
        for (int w2 = 0; w2 < warp; ++w2) r += wh[w2][e];
        for (int j = 0; j < lane; ++j)
            for (int k2 = 0; k2 < K; ++k2) r += (ids[warp][j][k2] == e) ? 1 : 0;
        if (C < 0 || r < C) {
            const int32_t row = offsets[e] + r;
            inv[t * K + k] = row;
            src[row] = static_cast<int32_t>(t);
        } else {
            inv[t * K + k] = -1;
        }
    }
}

__global__ void __launch_bounds__(256)
gather_kernel(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ inv, int64_t T, int d, int K,
              __nv_bfloat16* __restrict__ x_perm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nw = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int nvec = d / 8;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp; t < T; t += nw) {
        int32_t rows[16];
        int nr = 0;
        for (int k = 0; k < K; ++k) {
            const int32_t r = inv[t * K + k];
            if (r >= 0) rows[nr++] = r;
        }
        if (nr == 0) continue;
        const uint4* s = reinterpret_cast<const uint4*>(x + t * d);
        for (int c = lane; c < nvec; c += 32) {
            const uint4 v = __ldg(s + c);
            for (int i = 0; i < nr; ++i)
                reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(rows[i]) * d)[c] = v;
        }
    }
}

}  // namespace

int permute_blocks(int64_t T) { return static_cast<int>((T + kTokPerBlock - 1) / kTokPerBlock); }

int launch_permute(const int32_t* idx, const bf16* x, int64_t T, int d, int E, int K, int64_t C,
                   int32_t* block_hist, int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* inv,
                   int32_t* src, bf16* x_perm, int32_t* n_dropped, cudaStream_t st) {
    if (E > 256 || K > 16) return -2;
    const int nb = permute_blocks(T);
    hist_kernel<<<nb, kTokPerBlock, 0, st>>>(idx, T, E, K, block_hist);
    scan_kernel<<<1, 1024, 0, st>>>(block_hist, nb, E, C, counts, kept, offsets, n_dropped);
    rank_kernel<<<nb, kTokPerBlock, 0, st>>>(idx, T, E, K, C, block_hist, offsets, inv, src);
    if (x != nullptr && x_perm != nullptr) {
        const int sms = num_sms() > 0 ? num_sms() : 148;
        int64_t need = (T + 7) / 8;
        int grid = static_cast<int>(need < sms * 8 ? need : sms * 8);
        gather_kernel<<<grid, 256, 0, st>>>(x, inv, T, d, K, x_perm);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace moe
