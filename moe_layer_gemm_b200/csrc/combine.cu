// Combine, load statistics and the aux-free bias update.
//
// Combine: "MoE computation notes" (cf-1.com/news/5905749), section 2 step 4
// and section 2.3: the output is the weighted sum of the K experts' outputs,
// put back in token order; section 2.2: unselected experts add nothing.  A
// deterministic gather: one CTA per token reads its K rows (skipping
// dropped slots) and sums them in slot order in fp32; no atomics.  When the
// expert GEMM split its reduction, the partial slices are summed here first,
// in slice order.
//
// Statistics: same notes, section 1.2: aux = N * sum_i f_i * P_i.
// Bias: "MoE inference engineering in practice"
// (ybb.press/quantum-computing/18594), section 1.2: overloaded experts get
// bias -= alpha, underloaded bias += alpha.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kMaxK = 16;

constexpr int kMaxSplit = 8;

__device__ __forceinline__ float warp_sum_fixed(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// The statistics tail (one CTA of any multiple of 32 threads): warp w
// reduces experts w, w + nw, ...: lane l adds router blocks l, l + 32, ...
// in order, then a fixed butterfly; P_i = sum / T, f_i = counts_i / (T K),
// P~_i (top-K weights) likewise; aux = E * sum_i f_i P_i and aux_topk =
// E * sum_i f_i P~_i summed per warp in expert order, then over warps in
// warp order; z_loss = (sum of the blocks' squared log-sum-exp sums: lane l
// adds blocks l, l + 32, ..., then the fixed butterfly) / T.  Then the bias update, one expert per thread.  Every sum
// has a fixed order, so results are reproducible.
// Column `col` of the router statistics rows summed over the blocks: lane l
// adds blocks l, l + 32, ... in order, then the fixed butterfly.
__device__ __forceinline__ float sum_column(const float* part, int64_t row, int col, int nblocks, int lane) {
    float v = 0.f;
    for (int b = lane; b < nblocks; b += 32) v += part[b * row + col];
    return warp_sum_fixed(v);
}

__device__ void stats_tail(const StatsTail& s, int64_t T, int K) {
    __shared__ float red[2][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    const int E = s.E;
    const int64_t row = 2 * static_cast<int64_t>(E) + 1;
    if (s.part) {
        const float invT = 1.0f / static_cast<float>(T);
        const float invA = 1.0f / static_cast<float>(T * K);
        // P_i, f_i and their products (one pass), then P~_i (a second pass)
        float acc = 0.f;
        for (int e = warp; e < E; e += nw) {
            const float pe = sum_column(s.part, row, e, s.nblocks, lane) * invT;
            const float fe = static_cast<float>(s.counts[e]) * invA;
            if (lane == 0) {
                s.P[e] = pe;
                if (s.f) s.f[e] = fe;
                acc += fe * pe;
            }
        }
        float acc_t = 0.f;
        if (s.P_topk || s.aux_topk)
            for (int e = warp; e < E; e += nw) {
                const float pte = sum_column(s.part, row, E + e, s.nblocks, lane) * invT;
                if (lane == 0) {
                    if (s.P_topk) s.P_topk[e] = pte;
                    acc_t += static_cast<float>(s.counts[e]) * invA * pte;
                }
            }
        if (lane == 0) {
            red[0][warp] = acc;
            red[1][warp] = acc_t;
        }
        __syncthreads();
        if (warp == 0) {
            const float z = s.z_loss ? sum_column(s.part, row, 2 * E, s.nblocks, lane) : 0.f;
            if (lane == 0) {
                float a = 0.f, at = 0.f;
                for (int i = 0; i < nw; ++i) {
                    a += red[0][i];
                    at += red[1][i];
                }
                if (s.aux) *s.aux = static_cast<float>(E) * a;
                if (s.aux_topk) *s.aux_topk = static_cast<float>(E) * at;
                if (s.z_loss) *s.z_loss = z * invT;
            }
        }
    }
    if (s.bias && s.alpha != 0.0f) {
        const int64_t TK = T * K;
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            const int64_t lhs = static_cast<int64_t>(s.counts[e]) * E;
            float b = s.bias[e];
            if (lhs > TK) b = __fsub_rn(b, s.alpha);
            else if (lhs < TK) b = __fadd_rn(b, s.alpha);
            s.bias[e] = b;
        }
    }
}

// Store 4 consecutive outputs: fp32, or each rounded to bf16 (nearest even)
// from the same fp32 sum, so a bf16 output is exactly RNE of the fp32 one.
__device__ __forceinline__ void store4(float* y, int64_t i4, float4 v) { reinterpret_cast<float4*>(y)[i4] = v; }
__device__ __forceinline__ void store4(__nv_bfloat16* y, int64_t i4, float4 v) {
    const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t*>(&lo);
    u.y = *reinterpret_cast<const uint32_t*>(&hi);
    reinterpret_cast<uint2*>(y)[i4] = u;
}

// S >= nsplit slots for partial slices (S == nsplit except the 8-slot
// fallback, which reads only the nsplit slices that exist).  Slots are
// handled in groups of G, whose G x S loads are all in flight at once; G
// shrinks as slices grow so the registers, and with them the resident
// CTAs, stay put (more loads per thread measured slower at K = 4).
template <int S, typename OutT>
__global__ void __launch_bounds__(256, S == 1 ? 8 : (S >= 8 ? 2 : 4))  // one slice: 32 registers, 8 CTAs per SM
combine_kernel(const float* __restrict__ yp, int nsplit, int64_t split_stride, const int32_t* __restrict__ inv,
               const float* __restrict__ w, int64_t T, int d, int K, OutT* __restrict__ y, const StatsTail tail) {
    pdl_trigger();
    pdl_wait();
    // with a statistics tail the last CTA does only that
    const int ntok_blocks = static_cast<int>(gridDim.x) - (tail.counts ? 1 : 0);
    if (tail.counts && static_cast<int>(blockIdx.x) == ntok_blocks) {
        stats_tail(tail, tail.T > 0 ? tail.T : T, K);
        return;
    }
    const int nvec = d / 4;
    const int64_t svec = split_stride / 4;
    // the token's rows and weights, read once per CTA
    __shared__ int32_t rows[kMaxK];
    __shared__ float ws[kMaxK];
    for (int64_t t = blockIdx.x; t < T; t += ntok_blocks) {
        if (static_cast<int>(threadIdx.x) < K) {
            rows[threadIdx.x] = inv[t * K + threadIdx.x];
            ws[threadIdx.x] = w[t * K + threadIdx.x];
        }
        __syncthreads();
        for (int c = threadIdx.x; c < nvec; c += blockDim.x) {
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            // slots in groups of G: a group's loads are all issued before its
            // arithmetic; slices are summed in slice order and slots
            // accumulated in slot order
            constexpr int G = S >= 4 ? 2 : 4;
            for (int k0 = 0; k0 < K; k0 += G) {
                float4 v[G][S];
#pragma unroll
                for (int j = 0; j < G; ++j) {
                    const int k = k0 + j;
                    const bool live = k < K && rows[k] >= 0;
                    const float4* base =
                        reinterpret_cast<const float4*>(yp + static_cast<int64_t>(live ? rows[k] : 0) * d) + c;
#pragma unroll
                    for (int sl = 0; sl < S; ++sl)
                        v[j][sl] = (live && sl < nsplit) ? __ldg(base + sl * svec) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int j = 0; j < G; ++j) {
                    const int k = k0 + j;
                    if (k < K && rows[k] >= 0) {
                        float4 u = v[j][0];
#pragma unroll
                        for (int sl = 1; sl < S; ++sl)
                            if (sl < nsplit) {
                                u.x += v[j][sl].x; u.y += v[j][sl].y; u.z += v[j][sl].z; u.w += v[j][sl].w;
                            }
                        acc.x = fmaf(ws[k], u.x, acc.x);
                        acc.y = fmaf(ws[k], u.y, acc.y);
                        acc.z = fmaf(ws[k], u.z, acc.z);
                        acc.w = fmaf(ws[k], u.w, acc.w);
                    }
                }
            }
            store4(y + t * d, c, acc);
        }
        __syncthreads();  // rows / ws are rewritten for the next token
    }
}

// One reduction slice (no split): a warp per token, no block barriers.  Lane
// k < K reads the slot's row and weight, shuffled to all lanes; each lane
// then sums columns lane, lane + 32, ... of the K rows, two 16-byte columns
// at a time with all their loads issued together, slots in slot order, as
// combine_kernel does (the same fp32 operations in the same order, so the
// output is bit-identical).  With a statistics tail the last CTA does only that.
template <typename OutT>
__global__ void __launch_bounds__(256, 4)
combine_warp_kernel(const float* __restrict__ yp, const int32_t* __restrict__ inv, const float* __restrict__ w,
                    int64_t T, int d, int K, OutT* __restrict__ y, const StatsTail tail) {
    pdl_trigger();
    pdl_wait();
    const int ntok_blocks = static_cast<int>(gridDim.x) - (tail.counts ? 1 : 0);
    if (tail.counts && static_cast<int>(blockIdx.x) == ntok_blocks) {
        stats_tail(tail, tail.T > 0 ? tail.T : T, K);
        return;
    }
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(ntok_blocks) * (blockDim.x >> 5);
    const int nvec = d / 4;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps) {
        const int32_t my_row = lane < K ? inv[t * K + lane] : -1;
        const float my_w = lane < K ? w[t * K + lane] : 0.f;
        for (int c0 = lane; c0 < nvec; c0 += 64) {
            const int c1 = c0 + 32;
            const bool two = c1 < nvec;
            float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
            // slots in groups of 4: both columns' loads of a group in flight together
            for (int k0 = 0; k0 < K; k0 += 4) {
                float4 v0[4], v1[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int k = k0 + j;
                    const int r = __shfl_sync(0xffffffffu, my_row, k < K ? k : 0);
                    const bool live = k < K && r >= 0;
                    const float4* base = reinterpret_cast<const float4*>(yp + static_cast<int64_t>(live ? r : 0) * d);
                    v0[j] = live ? __ldg(base + c0) : make_float4(0.f, 0.f, 0.f, 0.f);
                    v1[j] = (live && two) ? __ldg(base + c1) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int k = k0 + j;
                    const int r = __shfl_sync(0xffffffffu, my_row, k < K ? k : 0);
                    const float wk = __shfl_sync(0xffffffffu, my_w, k < K ? k : 0);
                    if (k < K && r >= 0) {
                        a0.x = fmaf(wk, v0[j].x, a0.x);
                        a0.y = fmaf(wk, v0[j].y, a0.y);
                        a0.z = fmaf(wk, v0[j].z, a0.z);
                        a0.w = fmaf(wk, v0[j].w, a0.w);
                        a1.x = fmaf(wk, v1[j].x, a1.x);
                        a1.y = fmaf(wk, v1[j].y, a1.y);
                        a1.z = fmaf(wk, v1[j].z, a1.z);
                        a1.w = fmaf(wk, v1[j].w, a1.w);
                    }
                }
            }
            store4(y + t * d, c0, a0);
            if (two) store4(y + t * d, c1, a1);
        }
    }
}

// y_perm[r] = sum over slices s of part[s][r], rows r < offsets[E].
__global__ void __launch_bounds__(256)
reduce_splits_kernel(const float* __restrict__ part, int nsplit, int64_t split_stride,
                     const int32_t* __restrict__ offsets, int E, int d, float* __restrict__ out) {
    pdl_trigger();
    pdl_wait();
    const int64_t n = static_cast<int64_t>(offsets[E]) * (d / 4);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float4 v = reinterpret_cast<const float4*>(part)[i];
        for (int s = 1; s < nsplit; ++s) {
            const float4 u = reinterpret_cast<const float4*>(part + s * split_stride)[i];
            v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
        }
        reinterpret_cast<float4*>(out)[i] = v;
    }
}

// One block: f_i = counts_i / (T K); aux = E * sum_i f_i P_i (fixed-order tree).
__global__ void __launch_bounds__(256)
stats_kernel(const int32_t* __restrict__ counts, const float* __restrict__ P, int64_t T, int E, int K,
             float* __restrict__ f, float* __restrict__ aux) {
    pdl_trigger();
    pdl_wait();
    __shared__ float red[256];
    const float inv = 1.0f / static_cast<float>(T * K);
    float part = 0.f;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const float fe = static_cast<float>(counts[e]) * inv;
        if (f) f[e] = fe;
        if (P) part += fe * P[e];
    }
    red[threadIdx.x] = part;
    __syncthreads();
    for (int s = blockDim.x / 2; s > 0; s >>= 1) {
        if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
        __syncthreads();
    }
    if (threadIdx.x == 0 && aux) *aux = static_cast<float>(E) * red[0];
}


__global__ void bias_update_kernel(const int32_t* __restrict__ counts, int64_t TK, int E, float alpha,
                                   float* __restrict__ bias) {
    pdl_trigger();
    pdl_wait();
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= E) return;
    const int64_t lhs = static_cast<int64_t>(counts[e]) * E;
    float b = bias[e];
    if (lhs > TK) b = __fsub_rn(b, alpha);
    else if (lhs < TK) b = __fadd_rn(b, alpha);
    bias[e] = b;
}

__global__ void accumulate_counts_kernel(int32_t* __restrict__ dst, const int32_t* __restrict__ src, int E,
                                         int first) {
    pdl_trigger();
    pdl_wait();
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < E) dst[e] = (first ? 0 : dst[e]) + src[e];
}

// W13p[e][32b + j][k] = (j < 16 ? W1 : W3)[e][k][16b + (j & 15)];  W2p[e][n][k] = W2[e][k][n].
// Both are [rows][cols] <- transpose of a [cols][rows]-shaped source, by
// 32 x 32 tiles through shared memory.
__global__ void pack_w13_kernel(const __nv_bfloat16* __restrict__ W1, const __nv_bfloat16* __restrict__ W3,
                                int d, int f, __nv_bfloat16* __restrict__ W13p) {
    __shared__ __nv_bfloat16 tile[32][33];
    const int e = blockIdx.z;
    const int k0 = blockIdx.x * 32;  // d index
    const int r0 = blockIdx.y * 32;  // packed row index (2f rows), one 32-row block = 16 gate + 16 up
    const int b = r0 / 32;
    const __nv_bfloat16* s1 = W1 + static_cast<int64_t>(e) * d * f;
    const __nv_bfloat16* s3 = W3 + static_cast<int64_t>(e) * d * f;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int k = k0 + i;
        const int j = threadIdx.x;
        const int col = 16 * b + (j & 15);
        __nv_bfloat16 v = __float2bfloat16_rn(0.f);
        if (k < d) v = (j < 16 ? s1 : s3)[static_cast<int64_t>(k) * f + col];
        tile[i][j] = v;
    }
    __syncthreads();
    const int64_t kb = (d + 63) / 64;
    __nv_bfloat16* dst = W13p + static_cast<int64_t>(e) * ((2 * f + 127) / 128) * kb * 8192;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int r = r0 + i, k = k0 + threadIdx.x;
        if (k < d) dst[tiled_offset(r, k, kb)] = tile[threadIdx.x][i];
    }
}

__global__ void pack_w2_kernel(const __nv_bfloat16* __restrict__ W2, int d, int f, __nv_bfloat16* __restrict__ W2p) {
    __shared__ __nv_bfloat16 tile[32][33];
    const int e = blockIdx.z;
    const int k0 = blockIdx.x * 32;  // f index (reduction of the down projection)
    const int n0 = blockIdx.y * 32;  // d index (output rows of W2p)
    const __nv_bfloat16* s = W2 + static_cast<int64_t>(e) * f * d;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int k = k0 + i, n = n0 + threadIdx.x;
        tile[i][threadIdx.x] = (k < f && n < d) ? s[static_cast<int64_t>(k) * d + n] : __float2bfloat16_rn(0.f);
    }
    __syncthreads();
    const int64_t kb = (f + 63) / 64;
    __nv_bfloat16* dst = W2p + static_cast<int64_t>(e) * ((d + 127) / 128) * kb * 8192;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int n = n0 + i, k = k0 + threadIdx.x;
        if (n < d && k < f) dst[tiled_offset(n, k, kb)] = tile[threadIdx.x][i];
    }
}

}  // namespace

template <typename OutT>
void launch_combine_t(int g, int threads, cudaStream_t st, const float* y_perm, int nsplit, int64_t split_stride,
                      const int32_t* inv, const float* w, int64_t T, int d, int K, OutT* y, const StatsTail& tail) {
    switch (nsplit) {
        case 1: (void)launch_pdl(combine_kernel<1, OutT>, dim3(g), dim3(threads), 0, st, y_perm, nsplit, split_stride, inv, w, T, d, K, y, tail); break;
        case 2: (void)launch_pdl(combine_kernel<2, OutT>, dim3(g), dim3(threads), 0, st, y_perm, nsplit, split_stride, inv, w, T, d, K, y, tail); break;
        case 3: (void)launch_pdl(combine_kernel<3, OutT>, dim3(g), dim3(threads), 0, st, y_perm, nsplit, split_stride, inv, w, T, d, K, y, tail); break;
        case 4: (void)launch_pdl(combine_kernel<4, OutT>, dim3(g), dim3(threads), 0, st, y_perm, nsplit, split_stride, inv, w, T, d, K, y, tail); break;
        default: (void)launch_pdl(combine_kernel<8, OutT>, dim3(g), dim3(threads), 0, st, y_perm, nsplit, split_stride, inv, w, T, d, K, y, tail); break;
    }
}

int launch_combine(const float* y_perm, int nsplit, int64_t split_stride, const int32_t* inv, const float* w,
                   int64_t T, int d, int K, void* y, bool y_bf16, cudaStream_t st, const StatsTail* tail_in) {
    if (K > kMaxK || d % 4 != 0 || nsplit < 1 || nsplit > kMaxSplit) return -2;
    const int sms = num_sms() > 0 ? num_sms() : 148;
    int64_t grid = T < static_cast<int64_t>(sms) * 16 ? T : static_cast<int64_t>(sms) * 16;
    if (grid < 1) grid = 1;
    const int threads = d / 4 >= 256 ? 256 : ((d / 4 + 31) / 32) * 32;
    StatsTail tail{};
    if (tail_in && tail_in->counts) {
        tail = *tail_in;
        if (tail.part && !tail.P) return -2;
        ++grid;  // one extra CTA for the tail
    }
    if (nsplit == 1 && K <= 32 && d >= 128) {
        // a warp per token: 8 tokens per CTA, the grid (with the statistics
        // CTA) capped at 4 CTAs per SM, one resident wave; a statistics CTA
        // beyond the wave would start only once a token CTA had finished
        int64_t gw = (T + 7) / 8;
        const int64_t cap = static_cast<int64_t>(sms) * 4 - (tail.counts ? 1 : 0);
        if (gw > cap) gw = cap;
        if (gw < 1) gw = 1;
        if (tail.counts) ++gw;
        if (y_bf16)
            (void)launch_pdl(combine_warp_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(gw)), dim3(256), 0, st, y_perm,
                             inv, w, T, d, K, static_cast<__nv_bfloat16*>(y), tail);
        else
            (void)launch_pdl(combine_warp_kernel<float>, dim3(static_cast<unsigned>(gw)), dim3(256), 0, st, y_perm, inv, w,
                             T, d, K, static_cast<float*>(y), tail);
        return cudaGetLastError() == cudaSuccess ? 0 : -3;
    }
    const int g = static_cast<int>(grid);
    if (y_bf16)
        launch_combine_t(g, threads, st, y_perm, nsplit, split_stride, inv, w, T, d, K, static_cast<__nv_bfloat16*>(y),
                         tail);
    else
        launch_combine_t(g, threads, st, y_perm, nsplit, split_stride, inv, w, T, d, K, static_cast<float*>(y), tail);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

int launch_reduce_splits(const float* part, int nsplit, int64_t split_stride, const int32_t* offsets, int E, int d,
                         float* y_perm, cudaStream_t st) {
    const int sms = num_sms() > 0 ? num_sms() : 148;
    (void)launch_pdl(reduce_splits_kernel, dim3(sms * 4), dim3(256), 0, st, part, nsplit, split_stride, offsets, E, d, y_perm);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

int launch_stats(const int32_t* counts, const float* prob_mean, int64_t T, int E, int K, float* f, float* aux,
                 const float*, cudaStream_t st) {
    (void)launch_pdl(stats_kernel, dim3(1), dim3(256), 0, st, counts, prob_mean, T, E, K, f, aux);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}


int launch_accumulate_counts(int32_t* dst, const int32_t* src, int E, bool first, cudaStream_t st) {
    (void)launch_pdl(accumulate_counts_kernel, dim3((E + 255) / 256), dim3(256), 0, st, dst, src, E, first ? 1 : 0);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

int launch_bias_update(const int32_t* counts, int64_t T, int E, int K, float alpha, float* bias, cudaStream_t st) {
    (void)launch_pdl(bias_update_kernel, dim3((E + 255) / 256), dim3(256), 0, st, counts, T * K, E, alpha, bias);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

size_t packed_w13_bytes(int E, int d, int f) {
    return static_cast<size_t>(E) * ((2 * f + 127) / 128) * ((d + 63) / 64) * 16384;
}
size_t packed_w2_bytes(int E, int d, int f) {
    return static_cast<size_t>(E) * ((d + 127) / 128) * ((f + 63) / 64) * 16384;
}

int launch_pack(const bf16* W1, const bf16* W3, const bf16* W2, int E, int d, int f, bf16* W13p, bf16* W2p,
                cudaStream_t st) {
    // padding of partial tiles stays zero
    if (cudaMemsetAsync(W13p, 0, packed_w13_bytes(E, d, f), st) != cudaSuccess) return -3;
    if (cudaMemsetAsync(W2p, 0, packed_w2_bytes(E, d, f), st) != cudaSuccess) return -3;
    dim3 block(32, 8);
    dim3 g13((d + 31) / 32, (2 * f) / 32, E);
    pack_w13_kernel<<<g13, block, 0, st>>>(W1, W3, d, f, W13p);
    dim3 g2((f + 31) / 32, (d + 31) / 32, E);
    pack_w2_kernel<<<g2, block, 0, st>>>(W2, d, f, W2p);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace moe
