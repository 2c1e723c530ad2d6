// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), fed by
// TMA, for the expert FFN of an MoE layer: each expert g multiplies its own
// contiguous group of token rows by its own weight matrix ("MoE computation
// notes", cf-1.com/news/5905749, section 2.1: permute tokens so each expert
// gets one contiguous batch and run one matrix product per group).
//
// One persistent CTA per SM walks a device-built list of output tiles, so
// the ragged group sizes never travel to the host.  Roles per CTA (192
// threads):
//   warp 0        TMA producer (one elected thread), multi-stage smem ring
//   warp 1        TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2..5    epilogue: TMEM -> registers -> SwiGLU / fp32 -> global
// The accumulator is double-buffered in TMEM (2 x 256 fp32 columns), so the
// epilogue of tile i overlaps the main loop of tile i+1.
//
// Two tile orientations:
//   token-major (swap = 0):  D[128 tokens x BN weight rows]; used when groups
//                            hold many tokens (prefill).
//   weight-major (swap = 1): D[128 weight rows x n tokens] (n <= 128, a
//                            multiple of 32); used when groups are small
//                            (decode), so no tensor-core rows are wasted on
//                            padding and the weight stream dominates.  The
//                            reduction can be split (deterministic partial
//                            slices, summed later in a fixed order).
// No TMA multicast is used anywhere.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kBK = 64;                 // reduction elements per stage (one 128 B swizzle row)
constexpr int kThreads = 192;
constexpr uint32_t kTileABytes = 128u * 128u;  // 128 rows x 64 bf16
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxGroups = 1024;

struct DevArgs {
    const int32_t* group_off;
    int G;
    int64_t dense_rows;
    int N;
    int N_store;
    int k_blocks;
    int ksplit;
    int kb_per_split;
    int swap;
    int BN;  // token-major: weight rows per tile; weight-major: max tokens per tile
    int epi;
    int stages;
    uint32_t stage_b_bytes;
    void* out;
    int64_t ldo;
    int64_t split_stride;
    int* status;
};

struct Tile {
    int g;
    int64_t row0;  // first token row of the tile
    int rows;      // valid token rows (<= 128 or <= BN)
    int n0;        // first weight row within the group
    int kb0, kb1;  // reduction blocks [kb0, kb1)
    int split;
};

__device__ __forceinline__ int64_t grp_off(const int64_t* off, int g) { return off[g]; }

__device__ __forceinline__ int tiles_of_group(const DevArgs& a, int64_t rows) {
    if (rows <= 0) return 0;
    if (!a.swap) {
        int64_t mt = (rows + 127) / 128;
        return static_cast<int>(mt * (a.N / a.BN));
    }
    int64_t nch = (rows + a.BN - 1) / a.BN;
    return static_cast<int>(nch * (a.N / 128) * a.ksplit);
}

__device__ __forceinline__ Tile decode_tile(const DevArgs& a, int tile, const int* tstart,
                                            const int64_t* off) {
    int lo = 0, hi = a.G;  // tstart[lo] <= tile < tstart[hi]
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (tstart[mid] <= tile) lo = mid; else hi = mid;
    }
    Tile t;
    t.g = lo;
    int local = tile - tstart[lo];
    int64_t base = off[lo];
    int64_t rows_g = off[lo + 1] - base;
    if (!a.swap) {
        int mt = static_cast<int>((rows_g + 127) / 128);
        int n = local / mt, m = local - n * mt;
        t.row0 = base + static_cast<int64_t>(m) * 128;
        t.rows = static_cast<int>(rows_g - static_cast<int64_t>(m) * 128 < 128 ? rows_g - static_cast<int64_t>(m) * 128 : 128);
        t.n0 = n * a.BN;
        t.kb0 = 0;
        t.kb1 = a.k_blocks;
        t.split = 0;
    } else {
        int nch = static_cast<int>((rows_g + a.BN - 1) / a.BN);
        int s = local % a.ksplit;
        int rest = local / a.ksplit;
        int c = rest % nch;
        int w = rest / nch;
        t.row0 = base + static_cast<int64_t>(c) * a.BN;
        t.rows = static_cast<int>(rows_g - static_cast<int64_t>(c) * a.BN < a.BN ? rows_g - static_cast<int64_t>(c) * a.BN : a.BN);
        t.n0 = w * 128;
        t.kb0 = s * a.kb_per_split;
        t.kb1 = min(a.k_blocks, t.kb0 + a.kb_per_split);
        t.split = s;
    }
    return t;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_tok,
                    const __grid_constant__ CUtensorMap tm_w, const DevArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int S = a.stages;
    uint8_t* sA = smem;
    uint8_t* sB = smem + static_cast<size_t>(S) * kTileABytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(sB + static_cast<size_t>(S) * a.stage_b_bytes);
    uint64_t* empty = full + S;
    uint64_t* tfull = empty + S;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int64_t* off = reinterpret_cast<int64_t*>(tmem_slot + 4);  // [G+1]
    int* tstart = reinterpret_cast<int*>(off + a.G + 1);        // [G+1]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_tok);
        tma_prefetch_desc(&tm_w);
    }
    if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
    for (int g = threadIdx.x; g <= a.G; g += blockDim.x)
        off[g] = a.group_off ? static_cast<int64_t>(a.group_off[g]) : (g == 0 ? 0 : a.dense_rows);
    __syncthreads();
    if (warp == 0) {
        // tile prefix over groups: each lane scans a contiguous span
        const int span = (a.G + 31) / 32;
        const int g0 = min(a.G, lane * span), g1 = min(a.G, g0 + span);
        int sum = 0;
        for (int g = g0; g < g1; ++g) sum += tiles_of_group(a, off[g + 1] - off[g]);
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
        for (int g = g0; g < g1; ++g) {
            tstart[g] = run;
            run += tiles_of_group(a, off[g + 1] - off[g]);
        }
        if (lane == 31) tstart[a.G] = incl;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = tstart[a.G];

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            const uint64_t pol_w = policy_evict_first();
            const uint64_t pol_t = policy_evict_last();
            uint32_t s = 0, ph = 0;
            uint32_t issued_mask = 0, issued_ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
                const Tile t = decode_tile(a, tile, tstart, off);
                const int nb = a.swap ? (t.rows + 31) / 32 : 0;
                const uint32_t bytes = a.swap ? kTileABytes + static_cast<uint32_t>(nb) * 4096u
                                              : kTileABytes + static_cast<uint32_t>(a.BN) * 128u;
                const int wrow = t.g * a.N + t.n0;
                for (int kb = t.kb0; kb < t.kb1; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, a.status, DEV_TIMEOUT_PRODUCER_EMPTY, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[s], bytes);
                    uint8_t* dA = sA + static_cast<size_t>(s) * kTileABytes;
                    uint8_t* dB = sB + static_cast<size_t>(s) * a.stage_b_bytes;
                    const int kx = kb * kBK;
                    if (!a.swap) {
                        tma_load_2d(&tm_tok, dA, &full[s], kx, static_cast<int32_t>(t.row0), pol_t);
                        tma_load_2d(&tm_w, dB, &full[s], kx, wrow, pol_w);
                    } else {
                        tma_load_2d(&tm_w, dA, &full[s], kx, wrow, pol_w);
                        for (int j = 0; j < nb; ++j)
                            tma_load_2d(&tm_tok, dB + j * 4096, &full[s], kx,
                                        static_cast<int32_t>(t.row0 + 32 * j), pol_t);
                    }
                    issued_mask |= 1u << s;
                    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                    if (++s == static_cast<uint32_t>(S)) { s = 0; ph ^= 1u; }
                }
            }
            // Drain: every issued load has landed before the CTA may exit.
            for (int i = 0; i < S; ++i)
                if (issued_mask & (1u << i)) {
                    uint32_t p = (issued_ph >> i) & 1u;
                    for (uint32_t it = 0; it < kWaitLimit; ++it)
                        if (mbar_try_wait(&full[i], p)) break;
                }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            uint32_t s = 0, ph = 0;
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
                const Tile t = decode_tile(a, tile, tstart, off);
                const int buf = it & 1;
                const uint32_t use = static_cast<uint32_t>(it >> 1);
                if (!mbar_wait(&tempty[buf], (use & 1u) ^ 1u, a.status, DEV_TIMEOUT_MMA_TEMPTY, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf) * 256u;
                const uint32_t n_mma = a.swap ? static_cast<uint32_t>((t.rows + 31) / 32) * 32u
                                              : static_cast<uint32_t>(a.BN);
                const uint32_t idesc = umma_idesc_bf16(128, n_mma);
                for (int kb = t.kb0; kb < t.kb1; ++kb) {
                    if (!mbar_wait(&full[s], ph, a.status, DEV_TIMEOUT_MMA_FULL, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + static_cast<size_t>(s) * kTileABytes);
                    const uint32_t b_base = smem_u32(sB + static_cast<size_t>(s) * a.stage_b_bytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        umma_bf16(d_tmem, umma_desc_sw128(a_base + kk * 32), umma_desc_sw128(b_base + kk * 32),
                                  idesc, (kb > t.kb0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);
                    if (++s == static_cast<uint32_t>(S)) { s = 0; ph ^= 1u; }
                }
                if (ok) umma_commit(&tfull[buf]);
            }
            // All issued MMAs complete before TMEM is released.
            umma_commit(drain);
            for (uint32_t i = 0; i < kWaitLimit; ++i)
                if (mbar_try_wait(drain, 0)) break;
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        int it = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
            const Tile t = decode_tile(a, tile, tstart, off);
            const int buf = it & 1;
            const uint32_t use = static_cast<uint32_t>(it >> 1);
            if (!mbar_wait(&tfull[buf], use & 1u, a.status, DEV_TIMEOUT_EPI_TFULL, abort_flag)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + static_cast<uint32_t>(buf) * 256u +
                                   (static_cast<uint32_t>(q * 32) << 16);
            float v[32];
            if (!a.swap) {
                const int r = q * 32 + lane;
                const bool valid = r < t.rows;
                const int64_t grow = t.row0 + r;
                const int nchunks = a.BN / 32;
                for (int c = 0; c < nchunks; ++c) {
                    tmem_ld32(taddr + static_cast<uint32_t>(c * 32), v);
                    if (!valid) continue;
                    if (a.epi == EPI_SWIGLU_BF16) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            pk[i] = pack_bf16x2(silu_f(v[2 * i]) * v[16 + 2 * i],
                                                silu_f(v[2 * i + 1]) * v[16 + 2 * i + 1]);
                        bf16* H = static_cast<bf16*>(a.out) + grow * a.ldo + (t.n0 / 2 + c * 16);
                        uint4* dst = reinterpret_cast<uint4*>(H);
                        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    } else {
                        const int col0 = t.n0 + c * 32;
                        float* Y = static_cast<float*>(a.out) + grow * a.ldo + col0;
                        if (col0 + 32 <= a.N_store && (a.ldo & 3) == 0) {  // float4 rows need 16 B alignment
                            float4* dst = reinterpret_cast<float4*>(Y);
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                        } else {
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (col0 + i < a.N_store) Y[i] = v[i];
                        }
                    }
                }
            } else {
                const int nb = (t.rows + 31) / 32;
                for (int c = 0; c < nb; ++c) {
                    tmem_ld32(taddr + static_cast<uint32_t>(c * 32), v);
                    if (a.epi == EPI_SWIGLU_BF16) {
                        const int f = t.n0 / 2 + q * 16 + (lane & 15);
                        bf16* H = static_cast<bf16*>(a.out);
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float u = __shfl_xor_sync(0xffffffffu, v[j], 16);
                            const int tok = c * 32 + j;
                            if (lane < 16 && tok < t.rows)
                                H[(t.row0 + tok) * a.ldo + f] = __float2bfloat16_rn(silu_f(v[j]) * u);
                        }
                    } else {
                        float* Y = static_cast<float*>(a.out) + static_cast<int64_t>(t.split) * a.split_stride;
                        const int col = t.n0 + q * 32 + lane;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int tok = c * 32 + j;
                            if (tok < t.rows && col < a.N_store) Y[(t.row0 + tok) * a.ldo + col] = v[j];
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
        }
    }

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
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

int num_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    static int cached[64] = {0};
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    if (dev < 64) cached[dev] = n;
    return n;
}

// Returns 0 on success, -2 for an unsupported shape, -3 for a CUDA failure.
int launch_grouped_gemm(const GemmLaunch& L, cudaStream_t st) {
    if (L.G < 1 || L.G > kMaxGroups || L.Kdim < 16 || L.Kdim % 8 != 0 || L.N < 16) return -2;
    DevArgs a{};
    a.group_off = L.group_off;
    a.G = L.G;
    a.dense_rows = L.dense_rows;
    a.N = L.N;
    a.N_store = L.N_store;
    a.k_blocks = (L.Kdim + kBK - 1) / kBK;
    a.swap = L.swap;
    a.epi = L.epi;
    a.out = L.out;
    a.ldo = L.ldo;
    a.split_stride = L.split_stride;
    a.status = L.status;
    if (!L.swap) {
        int bn = 0;
        for (int c : {256, 128, 64, 32})
            if (L.N % c == 0) { bn = c; break; }
        if (bn == 0) return -2;
        a.BN = bn;
        a.ksplit = 1;
        a.kb_per_split = a.k_blocks;
    } else {
        if (L.N % 128 != 0) return -2;
        int64_t mx = L.max_group_rows < 1 ? 1 : L.max_group_rows;
        a.BN = static_cast<int>(mx >= 128 ? 128 : ((mx + 31) / 32) * 32);
        int ks = L.ksplit < 1 ? 1 : L.ksplit;
        if (ks > a.k_blocks) ks = a.k_blocks;
        a.kb_per_split = (a.k_blocks + ks - 1) / ks;
        a.ksplit = (a.k_blocks + a.kb_per_split - 1) / a.kb_per_split;
    }
    if (L.epi == EPI_SWIGLU_BF16 && (L.N % 32 != 0)) return -2;
    a.stage_b_bytes = static_cast<uint32_t>(a.BN) * 128u;
    const uint32_t stage = kTileABytes + a.stage_b_bytes;
    const size_t fixed = 1024 + (2 * 8 + 5) * 8 + 16 + static_cast<size_t>(L.G + 1) * 12 + 64;
    const size_t budget = 227 * 1024 - fixed;
    int stages = static_cast<int>(budget / stage);
    if (stages > 8) stages = 8;
    if (stages < 2) return -2;
    a.stages = stages;
    const size_t smem = fixed + static_cast<size_t>(stages) * stage;

    CUtensorMap tm_tok, tm_w;
    const uint64_t tok_rows = static_cast<uint64_t>(L.tok_rows < 1 ? 1 : L.tok_rows);
    if (!make_map(&tm_tok, L.tok, tok_rows, static_cast<uint64_t>(L.Kdim),
                  L.swap ? 32u : 128u))
        return -3;
    if (!make_map(&tm_w, L.w, static_cast<uint64_t>(L.G) * L.N, static_cast<uint64_t>(L.Kdim),
                  L.swap ? 128u : static_cast<uint32_t>(a.BN)))
        return -3;

    static bool attr_set = false;
    if (!attr_set) {
        if (cudaFuncSetAttribute(grouped_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 227 * 1024) != cudaSuccess)
            return -3;
        attr_set = true;
    }
    int sms = num_sms();
    if (sms <= 0) return -3;
    // Upper bound on the tile count, to avoid idle CTAs on tiny problems.
    int64_t rows_total = L.group_off ? L.tok_rows : L.dense_rows;
    int64_t bound;
    if (!L.swap) {
        bound = ((rows_total + 127) / 128 + L.G) * (L.N / a.BN);
    } else {
        bound = ((rows_total + a.BN - 1) / a.BN + L.G) * (L.N / 128) * a.ksplit;
    }
    int grid = static_cast<int>(bound < sms ? (bound < 1 ? 1 : bound) : sms);
    grouped_gemm_kernel<<<grid, kThreads, smem, st>>>(tm_tok, tm_w, a);
    return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // namespace moe
