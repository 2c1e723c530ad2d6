// Expert parallelism: the receiving rank's regroup of token rows.
//
// "MoE computation notes" (cf-1.com/news/5905749), section 4.2, and "MoE
// inference engineering in practice" (ybb.press/quantum-computing/18594),
// section 2.2: with the experts spread over G GPUs, each GPU routes its own
// tokens, sends every token row to the GPU that holds its expert (an
// all-to-all), runs its local experts, and sends the results back.
//
// A source rank sends its dispatched rows expert-major, so the rows one rank
// receives arrive source-major: source 0's rows for local expert 0, 1, ..,
// E_l - 1, then source 1's, and so on.  The expert GEMMs need one contiguous
// group per local expert.  This kernel moves received row r of block
// (source s, local expert e) to
//     row_of[r] = offsets[e] + (rows of e from sources before s) + (r - start of the block)
// so each expert's rows are grouped by source, and within a source in the
// order it sent them; offsets is the exclusive prefix of the per-expert row
// totals.  row_of is kept to send the results back in the received order.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kRegroupThreads = 1024;
constexpr int kMaxBlocks = 2048;  // G * E_l (e.g. 8 ranks x 256 local experts)

// Exclusive scan of v over the CTA's threads (one value per thread), in a
// fixed order; returns the exclusive prefix and writes the total to *total.
__device__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? warp_tot[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += u;
        }
        if (lane < nw) warp_tot[lane] = wi - w;  // exclusive prefix of the warps
        if (lane == 31) *total = wi;
    }
    __syncthreads();
    const int r = warp_tot[warp] + incl - v;
    __syncthreads();  // warp_tot is reused by the next scan
    return r;
}

// Every CTA builds the block tables in shared memory, CTA 0 writes the
// offsets, then all CTAs move rows (grid-stride over rows, one warp per row).
__global__ void __launch_bounds__(kRegroupThreads)
ep_regroup_kernel(const int32_t* __restrict__ counts, int G, int El, int64_t n, const __nv_bfloat16* __restrict__ in,
                  int d, __nv_bfloat16* __restrict__ out, int32_t* __restrict__ offsets, int32_t* __restrict__ row_of) {
    __shared__ int src_start[kMaxBlocks + 1];  // flat block b = s * El + e, in received (source-major) order
    __shared__ int dst_start[kMaxBlocks];
    __shared__ int col[kMaxBlocks];            // exclusive prefix over sources within expert e, at s * El + e
    __shared__ int warp_tot[32];
    __shared__ int total;
    const int nb = G * El;
    const int per = (nb + blockDim.x - 1) / blockDim.x;  // consecutive blocks per thread
    // 1. source-major exclusive prefix of the counts: where each block starts in `in`
    {
        const int b0 = threadIdx.x * per;
        int s = 0;
        for (int i = 0; i < per; ++i)
            if (b0 + i < nb) s += counts[b0 + i];
        int run = block_exclusive_scan(s, warp_tot, &total);
        for (int i = 0; i < per; ++i)
            if (b0 + i < nb) {
                src_start[b0 + i] = run;
                run += counts[b0 + i];
            }
        if (threadIdx.x == 0) src_start[nb] = total;
    }
    // 2. per expert: prefix over sources, and the expert's total
    int etot = 0;
    const int e_per = (El + blockDim.x - 1) / blockDim.x;
    for (int i = 0; i < e_per; ++i) {
        const int e = threadIdx.x * e_per + i;
        if (e < El) {
            int run = 0;
            for (int s = 0; s < G; ++s) {
                col[s * El + e] = run;
                run += counts[s * El + e];
            }
            etot += run;
        }
    }
    // 3. exclusive prefix of the expert totals: each expert's first output row
    {
        int run = block_exclusive_scan(etot, warp_tot, &total);
        for (int i = 0; i < e_per; ++i) {
            const int e = threadIdx.x * e_per + i;
            if (e < El) {
                int te = 0;
                for (int s = 0; s < G; ++s) te += counts[s * El + e];
                if (blockIdx.x == 0) offsets[e] = run;
                for (int s = 0; s < G; ++s) dst_start[s * El + e] = run + col[s * El + e];
                run += te;
            }
        }
        if (blockIdx.x == 0 && threadIdx.x == 0) offsets[El] = total;
    }
    __syncthreads();
    // 4. rows: warp per row; find the row's block by binary search
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    const int64_t lim = n < static_cast<int64_t>(src_start[nb]) ? n : static_cast<int64_t>(src_start[nb]);
    const int nvec = d / 8;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp; r < lim; r += nwarps) {
        int lo = 0, hi = nb;  // src_start[lo] <= r < src_start[hi]; empty blocks are skipped by the search
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (src_start[mid] <= r) lo = mid; else hi = mid;
        }
        const int64_t dst = dst_start[lo] + (r - src_start[lo]);
        if (lane == 0) row_of[r] = static_cast<int32_t>(dst);
        const uint4* s4 = reinterpret_cast<const uint4*>(in + r * d);
        uint4* d4 = reinterpret_cast<uint4*>(out + dst * d);
        for (int c = lane; c < nvec; c += 32) d4[c] = __ldg(s4 + c);
    }
}

}  // namespace

int ep_regroup_max_blocks() { return kMaxBlocks; }

int launch_ep_regroup(const int32_t* counts, int G, int El, int64_t n, const bf16* in, int d, bf16* out,
                      int32_t* offsets, int32_t* row_of, cudaStream_t st) {
    if (G < 1 || El < 1 || static_cast<int64_t>(G) * El > kMaxBlocks || d % 8 != 0 || n < 0) return -2;
    const int sms = num_sms() > 0 ? num_sms() : 148;
    const int64_t need = (n + 31) / 32;
    const int grid = static_cast<int>(need < sms ? (need < 1 ? 1 : need) : sms);
    ep_regroup_kernel<<<grid, kRegroupThreads, 0, st>>>(counts, G, El, n, in, d, out, offsets, row_of);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace moe
