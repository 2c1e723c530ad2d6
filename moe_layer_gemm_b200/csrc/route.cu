// Router: logits = x . W_r (+ bias), top-K selection and renormalisation.
//
// "MoE computation notes" (cf-1.com/news/5905749), section 1.2: the router
// is one linear map from the hidden state to one score per expert;
// section 2 steps 2-3 and section 2.1: keep the K best experts and weight
// them by a softmax over the K kept scores.  "MoE inference engineering in
// practice" (ybb.press/quantum-computing/18594), section 1: top-k on the
// logits then softmax; section 1.2: route on gate(x) + bias.
//
// Small E (<= 32) with W_r fitting in shared memory: one warp per token.
// Lanes stream the token's row with 16-byte loads, each lane keeps E partial
// dot products, a butterfly reduction leaves all E logits in every lane, and
// the top-K and the softmax over the kept logits run in registers.  Nothing
// but the K indices and weights (and optionally the logits) is written.
//
// Large E: the logits come from the tensor-core GEMM (gemm.cu) and a
// warp-per-token kernel selects from them (lane j owns experts j, j+32, ..).
//
// Ties: equal fp32 values rank the lower expert index first (-0.0 == +0.0).
// The per-token full softmax of the unbiased logits is summed per block in a
// fixed order for P_i; blocks' partial sums are added in block order later,
// so the statistics are deterministic.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cfloat>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kRouteWarps = 8;
constexpr int64_t kSplitRouteMaxT = 512;  // batches up to this size take one CTA per token

// Warp-wide top-K over values v[j] of expert (lane + 32 j), j < J.
// Returns, in lane r < K, the r-th selected (value, expert); other lanes get
// (-inf, -1).  `valid[j]` marks real experts.
template <int J>
__device__ __forceinline__ void warp_topk(const float (&v)[J], const bool (&valid)[J], int K, int lane,
                                          float& out_v, int& out_e) {
    bool taken[J];
#pragma unroll
    for (int j = 0; j < J; ++j) taken[j] = !valid[j];
    out_v = -FLT_MAX;
    out_e = -1;
    for (int r = 0; r < K; ++r) {
        float bv = -FLT_MAX;
        int be = 0x7fffffff;
        bool have = false;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int e = lane + 32 * j;
            if (!taken[j] && (!have || v[j] > bv)) {  // ascending j: ties keep the lower index
                bv = v[j];
                be = e;
                have = true;
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const bool ohave = __shfl_xor_sync(0xffffffffu, static_cast<int>(have), o) != 0;
            if (ohave && (!have || ov > bv || (ov == bv && oe < be))) {
                bv = ov;
                be = oe;
                have = true;
            }
        }
        // every lane now holds the same winner
#pragma unroll
        for (int j = 0; j < J; ++j)
            if (lane + 32 * j == be) taken[j] = true;
        if (lane == r) {
            out_v = bv;
            out_e = be;
        }
    }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// Selection, weights and statistics for one token whose unbiased logits are
// l[j] (expert lane + 32 j).  With want_prob, psum[j] accumulates the full
// softmax probability of expert lane + 32 j, tsum[j] its renormalised top-K
// weight when selected, and lane 0's zsum the squared log-sum-exp of the
// unbiased logits (the router z-loss term).
template <int J>
__device__ __forceinline__ void finish_token(const float (&l)[J], const bool (&valid)[J], const float* bias,
                                             int64_t t, int K, int lane, int32_t* idx, float* w,
                                             float (&psum)[J], float (&tsum)[J], float& zsum, bool want_prob) {
    if (want_prob) {
        float m = -FLT_MAX;
#pragma unroll
        for (int j = 0; j < J; ++j)
            if (valid[j]) m = fmaxf(m, l[j]);
        m = warp_max(m);
        float p[J];
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            p[j] = valid[j] ? expf(l[j] - m) : 0.f;
            s += p[j];
        }
        s = warp_sum(s);
        const float inv = 1.0f / s;
#pragma unroll
        for (int j = 0; j < J; ++j) psum[j] += p[j] * inv;
        if (lane == 0) {
            const float lse = m + logf(s);
            zsum += lse * lse;
        }
    }
    float lb[J];
#pragma unroll
    for (int j = 0; j < J; ++j) lb[j] = (bias != nullptr && valid[j]) ? l[j] + bias[lane + 32 * j] : l[j];
    float sv;
    int se;
    warp_topk<J>(lb, valid, K, lane, sv, se);
    const float vmax = __shfl_sync(0xffffffffu, sv, 0);
    const float ex = (lane < K) ? expf(sv - vmax) : 0.f;
    const float den = warp_sum(ex);
    const float wk = ex / den;
    if (lane < K) {
        idx[t * K + lane] = se;
        w[t * K + lane] = wk;
    }
    if (want_prob)
        for (int r = 0; r < K; ++r) {  // slot r's weight goes to the lane that owns its expert
            const int er = __shfl_sync(0xffffffffu, se, r);
            const float wr = __shfl_sync(0xffffffffu, wk, r);
#pragma unroll
            for (int j = 0; j < J; ++j)
                if (er == lane + 32 * j) tsum[j] += wr;
        }
}

// One row of 2 E + 1 floats per CTA: [probability sums | top-K weight sums |
// squared log-sum-exp sum], each summed over the CTA's warps in warp order.
template <int J>
__device__ __forceinline__ void write_prob_partials(const float (&psum)[J], const float (&tsum)[J], float zsum,
                                                    int E, float* prob_part) {
    __shared__ float sp[kRouteWarps][J * 32];
    __shared__ float st[kRouteWarps][J * 32];
    __shared__ float sz[kRouteWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int j = 0; j < J; ++j) {
        sp[warp][lane + 32 * j] = psum[j];
        st[warp][lane + 32 * j] = tsum[j];
    }
    if (lane == 0) sz[warp] = zsum;
    __syncthreads();
    float* row = prob_part + static_cast<int64_t>(blockIdx.x) * (2 * E + 1);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float s = 0.f, u = 0.f;
        for (int wi = 0; wi < kRouteWarps; ++wi) {
            s += sp[wi][e];
            u += st[wi][e];
        }
        row[e] = s;
        row[E + e] = u;
    }
    if (threadIdx.x == 0) {
        float z = 0.f;
        for (int wi = 0; wi < kRouteWarps; ++wi) z += sz[wi];
        row[2 * E] = z;
    }
}

// Fused router for E <= 32.  W_r is staged in shared memory as [d][8*EV]
// bf16 rows (zero-padded), EV = 16-byte vectors per row.  Each lane loads
// all of its 16-byte chunks of the token row before any arithmetic, so a
// warp keeps up to kXBatch loads in flight instead of one.
constexpr int kXBatch = 8;

template <int EV>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_fused_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ Wr,
                   const float* __restrict__ bias, int64_t T, int d, int E, int K,
                   float* __restrict__ logits, int32_t* __restrict__ idx, float* __restrict__ w,
                   float* __restrict__ prob_part) {
    pdl_trigger();
    pdl_wait();
    constexpr int EP = EV * 8;  // padded experts per row
    extern __shared__ uint4 swr_raw[];
    // 16-byte slot s of chunk c (8 rows = 8*EV slots) lives at s ^ (c & 7):
    // the lanes of a quarter-warp read the same row of consecutive chunks,
    // which would otherwise all fall in the same four banks.
    if (E == EP) {
        const uint4* src = reinterpret_cast<const uint4*>(Wr);
        for (int i = threadIdx.x; i < d * EV; i += blockDim.x) swr_raw[i ^ ((i / (8 * EV)) & 7)] = __ldg(src + i);
    } else {
        for (int i = threadIdx.x; i < d * EV; i += blockDim.x) {
            const int r = i / EV, vv = i - r * EV;
            uint4 pk;
            __nv_bfloat16* pe = reinterpret_cast<__nv_bfloat16*>(&pk);
#pragma unroll
            for (int h = 0; h < 8; ++h) {
                const int e = vv * 8 + h;
                pe[h] = e < E ? Wr[static_cast<int64_t>(r) * E + e] : __float2bfloat16_rn(0.f);
            }
            swr_raw[i ^ ((i / (8 * EV)) & 7)] = pk;
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kRouteWarps;
    float psum[1] = {0.f}, tsum[1] = {0.f}, zsum = 0.f;
    const bool want_prob = prob_part != nullptr;
    const int nvec = d / 8;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteWarps + warp; t < T; t += nwarps) {
        float acc[EP];
#pragma unroll
        for (int e = 0; e < EP; ++e) acc[e] = 0.f;
        const uint4* xr = reinterpret_cast<const uint4*>(x + t * d);
        for (int c0 = lane; c0 < nvec; c0 += 32 * kXBatch) {
            uint4 xv[kXBatch];
#pragma unroll
            for (int b = 0; b < kXBatch; ++b) {
                const int c = c0 + 32 * b;
                xv[b] = c < nvec ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int b = 0; b < kXBatch; ++b) {
                const int c = c0 + 32 * b;
                if (c >= nvec) break;
                const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&xv[b]);
#pragma unroll
                for (int i2 = 0; i2 < 4; ++i2) {
                    const float2 xf = __bfloat1622float2(xp[i2]);
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const float xs = half ? xf.y : xf.x;
                        const int slot0 = (c * 8 + 2 * i2 + half) * EV;
#pragma unroll
                        for (int vv = 0; vv < EV; ++vv) {
                            const uint4 wv = swr_raw[(slot0 + vv) ^ (c & 7)];
                            const __nv_bfloat162* wp = reinterpret_cast<const __nv_bfloat162*>(&wv);
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const float2 w2 = __bfloat1622float2(wp[h]);
                                acc[vv * 8 + 2 * h] = fmaf(xs, w2.x, acc[vv * 8 + 2 * h]);
                                acc[vv * 8 + 2 * h + 1] = fmaf(xs, w2.y, acc[vv * 8 + 2 * h + 1]);
                            }
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < EP; ++e) acc[e] = warp_sum(acc[e]);
        float l[1] = {-FLT_MAX};
#pragma unroll
        for (int e = 0; e < EP; ++e)
            if (e == lane) l[0] = acc[e];
        bool valid[1] = {lane < E};
        if (logits != nullptr && valid[0]) logits[t * E + lane] = l[0];
        finish_token<1>(l, valid, bias, t, K, lane, idx, w, psum, tsum, zsum, want_prob);
    }
    if (want_prob) write_prob_partials<1>(psum, tsum, zsum, E, prob_part);
}

// Small batches (decode): one CTA per token, its hidden dimension split
// across the 8 warps so the whole machine shares the latency chain.  W_r is
// read through L1 (each warp touches only its slice of rows).  Per-warp
// partial logits are summed in warp order in shared memory, then warp 0
// selects.  prob_part gets one row per CTA (= per token).
template <int EV>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_split_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ Wr,
                   const float* __restrict__ bias, int64_t T, int d, int E, int K, float* __restrict__ logits,
                   int32_t* __restrict__ idx, float* __restrict__ w, float* __restrict__ prob_part) {
    pdl_trigger();
    pdl_wait();
    constexpr int EP = EV * 8;
    __shared__ float part[kRouteWarps][EP];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nvec = d / 8;
    const int per_warp = (nvec + kRouteWarps - 1) / kRouteWarps;
    const int c_beg = warp * per_warp, c_end = min(nvec, c_beg + per_warp);
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        float acc[EP];
#pragma unroll
        for (int e = 0; e < EP; ++e) acc[e] = 0.f;
        const uint4* xr = reinterpret_cast<const uint4*>(x + t * d);
        if (E == EP) {
            // A W_r row is EV 16-byte vectors, so the 8 rows of one x vector
            // are 8 EV contiguous vectors.  Every load of a batch is issued
            // before any arithmetic: one round of L2 latency per batch.
            constexpr int VB = EV == 1 ? 2 : 1;  // x vectors per lane per batch
            const uint4* wr4 = reinterpret_cast<const uint4*>(Wr);
            for (int c0 = c_beg + lane; c0 < c_end; c0 += 32 * VB) {
                uint4 xv[VB];
                uint4 wv[VB][8 * EV];
#pragma unroll
                for (int b = 0; b < VB; ++b) {
                    const int c = c0 + 32 * b;
                    const bool ok = c < c_end;
                    xv[b] = ok ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int j = 0; j < 8 * EV; ++j)
                        wv[b][j] = ok ? __ldg(wr4 + static_cast<int64_t>(c) * 8 * EV + j) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int b = 0; b < VB; ++b) {
                    const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&xv[b]);
#pragma unroll
                    for (int i2 = 0; i2 < 4; ++i2) {
                        const float2 xf = __bfloat1622float2(xp[i2]);
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const float xs = half ? xf.y : xf.x;
#pragma unroll
                            for (int vv = 0; vv < EV; ++vv) {
                                const __nv_bfloat162* wp =
                                    reinterpret_cast<const __nv_bfloat162*>(&wv[b][(2 * i2 + half) * EV + vv]);
#pragma unroll
                                for (int h = 0; h < 4; ++h) {
                                    const float2 w2 = __bfloat1622float2(wp[h]);
                                    acc[vv * 8 + 2 * h] = fmaf(xs, w2.x, acc[vv * 8 + 2 * h]);
                                    acc[vv * 8 + 2 * h + 1] = fmaf(xs, w2.y, acc[vv * 8 + 2 * h + 1]);
                                }
                            }
                        }
                    }
                }
            }
        } else {
            for (int c0 = c_beg + lane; c0 < c_end; c0 += 32 * kXBatch) {
                uint4 xv[kXBatch];
#pragma unroll
                for (int b = 0; b < kXBatch; ++b) {
                    const int c = c0 + 32 * b;
                    xv[b] = c < c_end ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int b = 0; b < kXBatch; ++b) {
                    const int c = c0 + 32 * b;
                    if (c >= c_end) break;
                    const __nv_bfloat162* xp = reinterpret_cast<const __nv_bfloat162*>(&xv[b]);
#pragma unroll
                    for (int i2 = 0; i2 < 4; ++i2) {
                        const float2 xf = __bfloat1622float2(xp[i2]);
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const float xs = half ? xf.y : xf.x;
                            const int row = c * 8 + 2 * i2 + half;
#pragma unroll
                            for (int e = 0; e < EP; ++e) {
                                const float wv =
                                    e < E ? __bfloat162float(__ldg(Wr + static_cast<int64_t>(row) * E + e)) : 0.f;
                                acc[e] = fmaf(xs, wv, acc[e]);
                            }
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int e = 0; e < EP; ++e) acc[e] = warp_sum(acc[e]);
        if (lane == 0) {
#pragma unroll
            for (int e = 0; e < EP; ++e) part[warp][e] = acc[e];
        }
        __syncthreads();
        if (warp == 0) {
            float l[1] = {-FLT_MAX};
            if (lane < E) {
                float sum = 0.f;
                for (int w2 = 0; w2 < kRouteWarps; ++w2) sum += part[w2][lane];
                l[0] = sum;
            }
            bool valid[1] = {lane < E};
            if (logits != nullptr && valid[0]) logits[t * E + lane] = l[0];
            float psum[1] = {0.f};
            float tsum[1] = {0.f}, zsum = 0.f;
            finish_token<1>(l, valid, bias, t, K, lane, idx, w, psum, tsum, zsum, prob_part != nullptr);
            if (prob_part != nullptr) {  // one statistics row per token (see write_prob_partials)
                float* row = prob_part + t * (2 * E + 1);
                if (lane < E) {
                    row[lane] = psum[0];
                    row[E + lane] = tsum[0];
                }
                if (lane == 0) row[2 * E] = zsum;
            }
        }
        __syncthreads();
    }
}

// The logits are the sum of nsplit partial slices (a split reduction of the
// logits GEMM), added in slice order; with logits_out the sums are stored.
template <int J>
__global__ void __launch_bounds__(kRouteWarps * 32)
topk_from_logits_kernel(const float* __restrict__ logits, int nsplit, int64_t split_stride,
                        float* __restrict__ logits_out, const float* __restrict__ bias, int64_t T, int E,
                        int K, int32_t* __restrict__ idx, float* __restrict__ w, float* __restrict__ prob_part) {
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kRouteWarps;
    float psum[J], tsum[J], zsum = 0.f;
#pragma unroll
    for (int j = 0; j < J; ++j) psum[j] = tsum[j] = 0.f;
    const bool want_prob = prob_part != nullptr;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kRouteWarps + warp; t < T; t += nwarps) {
        float l[J];
        bool valid[J];
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int e = lane + 32 * j;
            valid[j] = e < E;
            l[j] = valid[j] ? logits[t * E + e] : -FLT_MAX;
        }
        // slice by slice, so the J loads of a slice are in flight together
        for (int sp = 1; sp < nsplit; ++sp) {
            const float* ls = logits + sp * split_stride + t * E;
            float u[J];
#pragma unroll
            for (int j = 0; j < J; ++j) u[j] = valid[j] ? ls[lane + 32 * j] : 0.f;
#pragma unroll
            for (int j = 0; j < J; ++j) l[j] += u[j];
        }
        if (logits_out != nullptr)
#pragma unroll
            for (int j = 0; j < J; ++j)
                if (valid[j]) logits_out[t * E + lane + 32 * j] = l[j];
        finish_token<J>(l, valid, bias, t, K, lane, idx, w, psum, tsum, zsum, want_prob);
    }
    if (want_prob) write_prob_partials<J>(psum, tsum, zsum, E, prob_part);
}

// P_i: warp w reduces experts w, w+32, ...: lane l adds router blocks l,
// l+32, ... in order, then a fixed butterfly (reproducible).  Block rows are
// 2 E + 1 floats wide (write_prob_partials); P's sums are the first E.
__global__ void __launch_bounds__(1024)
prob_finalize_kernel(const float* __restrict__ part, int nblocks, int E, float invT, float* __restrict__ out) {
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int e = warp; e < E; e += nw) {
        float s = 0.f;
        for (int b = lane; b < nblocks; b += 32) s += part[static_cast<int64_t>(b) * (2 * E + 1) + e];
        s = warp_sum(s);
        if (lane == 0) out[e] = s * invT;
    }
}

// WrT[e][k] = Wr[k][e] for e < E, 0 for E <= e < E_pad.
__global__ void transpose_router_kernel(const __nv_bfloat16* __restrict__ Wr, int d, int E, int E_pad,
                                        __nv_bfloat16* __restrict__ WrT) {
    pdl_trigger();
    pdl_wait();
    __shared__ __nv_bfloat16 tile[32][33];
    const int k0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int k = k0 + i, e = e0 + threadIdx.x;
        tile[i][threadIdx.x] = (k < d && e < E) ? Wr[static_cast<int64_t>(k) * E + e] : __float2bfloat16_rn(0.f);
    }
    __syncthreads();
    const int64_t kb = (d + 63) / 64;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int e = e0 + i, k = k0 + threadIdx.x;
        if (e < E_pad && k < kb * 64) WrT[tiled_offset(e, k, kb)] = tile[threadIdx.x][i];  // zero past d and E
    }
}

}  // namespace

int route_blocks(int64_t T) {
    if (T <= kSplitRouteMaxT) return static_cast<int>(T);  // the small-batch router: one CTA per token
    const int sms = num_sms() > 0 ? num_sms() : 148;
    int64_t need = (T + kRouteWarps - 1) / kRouteWarps;
    int64_t cap = static_cast<int64_t>(sms) * 4;
    return static_cast<int>(need < cap ? (need < 1 ? 1 : need) : cap);
}

int route_fused_supported(int d, int E) {
    if (E > 32 || d % 8 != 0) return 0;
    const int EP = E <= 8 ? 8 : (E <= 16 ? 16 : 32);
    return static_cast<size_t>(d) * EP * 2 <= 96 * 1024 ? 1 : 0;
}

template <int EV>
int launch_fused_ev(const bf16* x, const bf16* Wr, const float* bias, int64_t T, int d, int E, int K, float* logits,
                    int32_t* idx, float* w, float* prob_part, int nblocks, cudaStream_t st) {
    static std::atomic<unsigned long long> attr_done{0};
    if (smem_attr_once(reinterpret_cast<const void*>(route_fused_kernel<EV>), 96 * 1024, attr_done) != 0) return -3;
    const size_t smem = static_cast<size_t>(d) * EV * 8 * 2;
    (void)launch_pdl(route_fused_kernel<EV>, dim3(nblocks), dim3(kRouteWarps * 32), smem, st, x, Wr, bias, T, d, E, K, logits, idx, w, prob_part);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

int launch_route_fused(const bf16* x, const bf16* Wr, const float* bias, int64_t T, int d, int E, int K,
                       float* logits, int32_t* idx, float* w, float* prob_part, int nblocks, cudaStream_t st) {
    if (T <= kSplitRouteMaxT) {
        // nblocks == T here (route_blocks): one CTA per token
        const int th = kRouteWarps * 32;
        if (E <= 8)
            (void)launch_pdl(route_split_kernel<1>, dim3(static_cast<unsigned>(T)), dim3(th), 0, st, x, Wr, bias, T, d, E, K, logits,
                             idx, w, prob_part);
        else if (E <= 16)
            (void)launch_pdl(route_split_kernel<2>, dim3(static_cast<unsigned>(T)), dim3(th), 0, st, x, Wr, bias, T, d, E, K, logits,
                             idx, w, prob_part);
        else
            (void)launch_pdl(route_split_kernel<4>, dim3(static_cast<unsigned>(T)), dim3(th), 0, st, x, Wr, bias, T, d, E, K, logits,
                             idx, w, prob_part);
        return cudaGetLastError() == cudaSuccess ? 0 : -3;
    }
    if (E <= 8) return launch_fused_ev<1>(x, Wr, bias, T, d, E, K, logits, idx, w, prob_part, nblocks, st);
    if (E <= 16) return launch_fused_ev<2>(x, Wr, bias, T, d, E, K, logits, idx, w, prob_part, nblocks, st);
    return launch_fused_ev<4>(x, Wr, bias, T, d, E, K, logits, idx, w, prob_part, nblocks, st);
}

int launch_topk_from_logits(const float* logits, int nsplit, int64_t split_stride, float* logits_out,
                            const float* bias, int64_t T, int E, int K, int32_t* idx, float* w, float* prob_part,
                            int nblocks, cudaStream_t st) {
    const int th = kRouteWarps * 32;
    if (nsplit < 1) return -2;
    if (E <= 32)
        (void)launch_pdl(topk_from_logits_kernel<1>, dim3(nblocks), dim3(th), 0, st, logits, nsplit, split_stride,
                         logits_out, bias, T, E, K, idx, w, prob_part);
    else if (E <= 64)
        (void)launch_pdl(topk_from_logits_kernel<2>, dim3(nblocks), dim3(th), 0, st, logits, nsplit, split_stride,
                         logits_out, bias, T, E, K, idx, w, prob_part);
    else if (E <= 128)
        (void)launch_pdl(topk_from_logits_kernel<4>, dim3(nblocks), dim3(th), 0, st, logits, nsplit, split_stride,
                         logits_out, bias, T, E, K, idx, w, prob_part);
    else if (E <= 256)
        (void)launch_pdl(topk_from_logits_kernel<8>, dim3(nblocks), dim3(th), 0, st, logits, nsplit, split_stride,
                         logits_out, bias, T, E, K, idx, w, prob_part);
    else
        return -2;
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

int launch_prob_finalize(const float* prob_part, int nblocks, int E, int64_t T, float* prob_mean, cudaStream_t st) {
    (void)launch_pdl(prob_finalize_kernel, dim3(1), dim3(1024), 0, st, prob_part, nblocks, E, 1.0f / static_cast<float>(T), prob_mean);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

int launch_transpose_router(const bf16* Wr, int d, int E, int E_pad, bf16* WrT, cudaStream_t st) {
    dim3 grid(((d + 63) / 64) * 2, (E_pad + 31) / 32), block(32, 8);  // columns up to the tile padding
    (void)launch_pdl(transpose_router_kernel, dim3(grid), dim3(block), 0, st, Wr, d, E, E_pad, WrT);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace moe
