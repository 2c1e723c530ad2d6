// Offloaded experts: group-wise INT4 storage and its unpacking into an
// on-device expert cache.
//
// "MoE inference engineering in practice" (ybb.press/quantum-computing/18594),
// section 3.2: when the experts do not all fit in GPU memory, some live in
// host memory, quantized group-wise to INT4 to cut the transfer volume; an
// LRU cache in GPU memory keeps the frequently used ones.
//
// Codes follow the packed weight layout (moe_pack_weights): for every
// 128-row x 64-column tile of an expert's packed matrix there are 4096 bytes
// of 4-bit codes (element i of the tile, in the tile's own swizzled order, in
// the low nibble of byte i / 2 for even i, the high nibble for odd i; two's
// complement) and 128 fp32 scales, one per tile row.  A tile row's 64
// elements are one quantization group: 64 consecutive reduction-axis weights
// of one output column.  Per group, in fp32: s = amax / 7 (correctly rounded
// division), q = clamp(round-half-even(w / s), -8, 7); an all-zero group has
// s = 0 and q = 0.  Unpacking writes bf16(q * s) (the fp32 product rounded
// to nearest even) into the same tile positions of a cache slot, so the
// expert GEMMs read a slot exactly like packed weights.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kTileElems = 128 * 64;
constexpr int kTileCodeBytes = kTileElems / 2;
constexpr int kUnpackJobsMax = 64;  // (expert, slot) pairs per launch, passed by value

__host__ __device__ __forceinline__ int64_t tiles_w13(int d, int f) {
    return static_cast<int64_t>((2 * f + 127) / 128) * ((d + 63) / 64);
}
__host__ __device__ __forceinline__ int64_t tiles_w2(int d, int f) {
    return static_cast<int64_t>((d + 127) / 128) * ((f + 63) / 64);
}

// Position of element (row r, column c) of a 128 x 64 tile: the 128-byte
// swizzle of the packed layout.
__device__ __forceinline__ int tile_pos(int r, int c) { return r * 64 + ((((c >> 3) ^ (r & 7)) << 3) | (c & 7)); }

// One CTA per tile (expert, row block, column block) of one matrix.  The
// 128 x 64 block is staged in shared memory as fp32; thread r (< 128) then
// quantizes row r.  `gate_up` selects the W13 row interleave (rows 32 b ..
// 32 b + 15 from W1 columns 16 b.., rows 32 b + 16 .. from W3), otherwise
// the transposed W2 (packed row n = column n of W2).
__global__ void __launch_bounds__(256)
int4_pack_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B, int Kred, int Ncols,
                 int rows_packed, int gate_up, uint8_t* __restrict__ q, float* __restrict__ s) {
    __shared__ float tile[128][65];
    const int kbn = (Kred + 63) / 64;
    const int64_t ntile = static_cast<int64_t>((rows_packed + 127) / 128) * kbn;
    const int e = blockIdx.y;
    const int64_t t = blockIdx.x;
    if (t >= ntile) return;
    const int rb = static_cast<int>(t / kbn), kb = static_cast<int>(t % kbn);
    const __nv_bfloat16* a = A + static_cast<int64_t>(e) * Kred * Ncols;
    const __nv_bfloat16* b = gate_up ? B + static_cast<int64_t>(e) * Kred * Ncols : nullptr;
    // stage: element (r, c) = packed row 128 rb + r, reduction index 64 kb + c
    for (int i = threadIdx.x; i < 128 * 64; i += blockDim.x) {
        const int c = i / 128, r = i % 128;  // consecutive threads: consecutive rows (source columns)
        const int n = 128 * rb + r, k = 64 * kb + c;
        float v = 0.f;
        if (n < rows_packed && k < Kred) {
            if (gate_up) {
                const int blk = n / 32, j = n % 32;
                const int col = 16 * blk + (j & 15);
                v = __bfloat162float((j < 16 ? a : b)[static_cast<int64_t>(k) * Ncols + col]);
            } else {
                v = __bfloat162float(a[static_cast<int64_t>(k) * Ncols + n]);
            }
        }
        tile[r][c] = v;
    }
    __syncthreads();
    const int r = threadIdx.x;
    if (r >= 128) return;
    float amax = 0.f;
    for (int c = 0; c < 64; ++c) amax = fmaxf(amax, fabsf(tile[r][c]));
    const float sc = __fdiv_rn(amax, 7.0f);
    uint8_t* qt = q + (static_cast<int64_t>(e) * ntile + t) * kTileCodeBytes;
    for (int c = 0; c < 64; c += 2) {  // columns c and c + 1 share one byte of the swizzled order
        uint32_t nib[2];
        for (int h = 0; h < 2; ++h) {
            int code = 0;
            if (sc > 0.f) {
                const float x = rintf(__fdiv_rn(tile[r][c + h], sc));
                code = static_cast<int>(fminf(7.f, fmaxf(-8.f, x)));
            }
            nib[h] = static_cast<uint32_t>(code) & 0xFu;
        }
        const int i = tile_pos(r, c);  // even: the pair (c, c + 1) maps to (i, i + 1)
        qt[i >> 1] = static_cast<uint8_t>(nib[0] | (nib[1] << 4));
    }
    s[(static_cast<int64_t>(e) * ntile + t) * 128 + r] = sc;
}

struct UnpackJobs {
    int n;
    int expert[kUnpackJobsMax];
    int slot[kUnpackJobsMax];
};

// Grid-stride over (job, tile) pairs, one tile per CTA step: 256 threads,
// each 16 bytes of codes = 32 elements of half a tile row.
__global__ void __launch_bounds__(256)
int4_unpack_kernel(UnpackJobs jobs, const uint8_t* __restrict__ q, const float* __restrict__ s, int64_t ntile,
                   __nv_bfloat16* __restrict__ W) {
    pdl_trigger();
    pdl_wait();
    const int64_t total = static_cast<int64_t>(jobs.n) * ntile;
    for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
        const int j = static_cast<int>(u / ntile);
        const int64_t t = u - static_cast<int64_t>(j) * ntile;
        const int64_t src = static_cast<int64_t>(jobs.expert[j]) * ntile + t;
        const int64_t dst = static_cast<int64_t>(jobs.slot[j]) * ntile + t;
        const uint4 cw = reinterpret_cast<const uint4*>(q + src * kTileCodeBytes)[threadIdx.x];
        const int i0 = threadIdx.x * 32;  // first element; 32 elements lie in row i0 / 64
        const float sc = s[src * 128 + (i0 >> 6)];
        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
        uint32_t outw[16];
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int h = 0; h < 8; h += 2) {
                const int lo = static_cast<int>(static_cast<int32_t>(words[w] << (28 - 4 * h)) >> 28);
                const int hi = static_cast<int>(static_cast<int32_t>(words[w] << (24 - 4 * h)) >> 28);
                const __nv_bfloat162 p = __floats2bfloat162_rn(__fmul_rn(static_cast<float>(lo), sc),
                                                               __fmul_rn(static_cast<float>(hi), sc));
                outw[w * 4 + h / 2] = *reinterpret_cast<const uint32_t*>(&p);
            }
        uint4* o = reinterpret_cast<uint4*>(W + dst * kTileElems + i0);
#pragma unroll
        for (int v = 0; v < 4; ++v) o[v] = make_uint4(outw[4 * v], outw[4 * v + 1], outw[4 * v + 2], outw[4 * v + 3]);
    }
}

}  // namespace

void int4_sizes(int E, int d, int f, size_t* q13, size_t* s13, size_t* q2, size_t* s2) {
    *q13 = static_cast<size_t>(E) * tiles_w13(d, f) * kTileCodeBytes;
    *s13 = static_cast<size_t>(E) * tiles_w13(d, f) * 128 * sizeof(float);
    *q2 = static_cast<size_t>(E) * tiles_w2(d, f) * kTileCodeBytes;
    *s2 = static_cast<size_t>(E) * tiles_w2(d, f) * 128 * sizeof(float);
}

int launch_int4_pack(const bf16* W1, const bf16* W3, const bf16* W2, int E, int d, int f, uint8_t* q13, float* s13,
                     uint8_t* q2, float* s2, cudaStream_t st) {
    if (E < 1 || E > 65535) return -2;
    const int64_t t13 = tiles_w13(d, f), t2 = tiles_w2(d, f);
    int4_pack_kernel<<<dim3(static_cast<unsigned>(t13), E), 256, 0, st>>>(W1, W3, d, f, 2 * f, 1, q13, s13);
    int4_pack_kernel<<<dim3(static_cast<unsigned>(t2), E), 256, 0, st>>>(W2, nullptr, f, d, d, 0, q2, s2);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

int launch_int4_unpack(int n_jobs, const int32_t* job_expert, const int32_t* job_slot, int d, int f,
                       const uint8_t* q13, const float* s13, const uint8_t* q2, const float* s2, bf16* W13c,
                       bf16* W2c, cudaStream_t st) {
    const int64_t t13 = tiles_w13(d, f), t2 = tiles_w2(d, f);
    const int sms = num_sms() > 0 ? num_sms() : 148;
    for (int j0 = 0; j0 < n_jobs; j0 += kUnpackJobsMax) {
        UnpackJobs jb{};
        jb.n = n_jobs - j0 < kUnpackJobsMax ? n_jobs - j0 : kUnpackJobsMax;
        for (int j = 0; j < jb.n; ++j) {
            jb.expert[j] = job_expert[j0 + j];
            jb.slot[j] = job_slot[j0 + j];
        }
        const int64_t w13 = jb.n * t13, w2 = jb.n * t2;
        const int g13 = static_cast<int>(w13 < 4LL * sms ? w13 : 4LL * sms);
        const int g2 = static_cast<int>(w2 < 4LL * sms ? w2 : 4LL * sms);
        (void)launch_pdl(int4_unpack_kernel, dim3(g13), dim3(256), 0, st, jb, q13, s13, t13, W13c);
        (void)launch_pdl(int4_unpack_kernel, dim3(g2), dim3(256), 0, st, jb, q2, s2, t2, W2c);
        if (cudaGetLastError() != cudaSuccess) return -3;
    }
    return 0;
}

}  // namespace moe
