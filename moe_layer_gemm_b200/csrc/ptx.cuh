// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA tile loads, tcgen05
// (TMEM allocation, UMMA issue/commit, TMEM loads).  Every wait is bounded: a
// wait that runs out records a code in the caller's status word and returns
// false instead of spinning forever.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace moe {

// Device status codes written to the workspace flag (0 = fine).
enum : int {
    DEV_OK = 0,
    DEV_TIMEOUT_PRODUCER_EMPTY = 1,
    DEV_TIMEOUT_MMA_FULL = 2,
    DEV_TIMEOUT_MMA_TEMPTY = 3,
    DEV_TIMEOUT_EPI_TFULL = 4,
    DEV_TIMEOUT_DRAIN = 5,
    DEV_TIMEOUT_DEPENDENCY = 6,
    DEV_BAD_INDEX = 7,  // a dispatch input named an expert outside [0, E); the slot was skipped
    DEV_BAD_SLOT = 8,   // an expert with rows had no valid cache slot; slot 0 was read instead
};

// Weight matrix of group g: g itself, or its cache slot from `slot_of`
// (nullptr: none).  A slot outside [0, n_slots) is never used as an address:
// the status records DEV_BAD_SLOT and slot 0 is read instead.
// Slot value that leaves group g out of a launch (its tiles are not counted).
constexpr int32_t kSlotSkip = -2;
__device__ __forceinline__ bool group_skipped(const int32_t* slot_of, int g) {
    return slot_of != nullptr && slot_of[g] == kSlotSkip;
}

__device__ __forceinline__ int weight_slot(const int32_t* slot_of, int n_slots, int g, int* status) {
    if (slot_of == nullptr) return g;
    const int s = slot_of[g];
    if (static_cast<unsigned>(s) < static_cast<unsigned>(n_slots)) return s;
    atomicCAS(status, 0, DEV_BAD_SLOT);
    return 0;
}

// Default poll limit of a bounded wait: about a few seconds on a B200
// before it gives up.  Launches pass their limit to the kernels (a test can
// ask for a much shorter one).
constexpr uint32_t kWaitLimit = 1u << 26;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Programmatic dependent launch.  pdl_wait blocks until the grids this one
// depends on (the previous kernel on the stream, when this one was launched
// with programmatic stream serialization) have completed and their memory is
// visible; without that launch attribute it returns at once.  Every kernel
// launched that way calls it, unconditionally and before touching any
// buffer another kernel writes or reads, so completion stays transitive
// along the stream.  pdl_trigger lets the next such kernel start launching
// once every CTA of this grid has called it or exited.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
                 ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Non-blocking probe: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity has completed.  Gives up after
// `limit` polls: records `code` in *status (first writer wins), raises
// *abort_flag and returns false.  `abort_flag` (shared) lets other roles stop
// early after a failure: once it is set the wait returns false without
// recording anything.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status, int code,
                                          volatile int* abort_flag, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 1023u) == 1023u) {
            if (*abort_flag) return false;
            if (i > 65536u) __nanosleep(64);
        }
    }
    atomicCAS(status, 0, code);
    *abort_flag = 1;
    return false;
}

// Drain wait: the phase with the given parity must complete (copies or MMAs
// in flight finish before the CTA exits), whatever the abort flag says.
// Gives up after `limit` polls, recording `code`, and returns false.
__device__ __forceinline__ bool mbar_drain(uint64_t* bar, uint32_t parity, int* status, int code, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 1023u) == 1023u && i > 65536u) __nanosleep(64);
    }
    atomicCAS(status, 0, code);
    return false;
}

// Complete `bytes` of the barrier's current phase's expected transaction
// count without a copy (stands in for bytes that will never arrive).
__device__ __forceinline__ void mbar_complete_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2D tiled load: box at (x = inner coordinate, y = row) into shared memory,
// completing `bytes` on `bar`.  x must be a multiple of 8 bf16 elements
// (16 bytes); every caller passes multiples of 64.
__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, void* smem_dst, uint64_t* bar,
                                            int32_t x, int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
          "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Untiled bulk copy global -> shared of `bytes` (multiple of 16; both
// addresses 16-byte aligned), completing on `bar`.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* src, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar)),
          "l"(policy)
        : "memory");
}

// ------------------------------------------------ staged fp32 tile stores
// An epilogue warp holds 32 rows x 32 fp32 columns of an output tile, one
// row per lane.  Stored directly, each 16-byte store instruction touches 32
// rows; instead the warp writes them into a 4 KB staging buffer (1024-byte
// aligned) in the 128-byte-swizzled layout of a TMA box {32 columns, 32 rows}
// (16-byte chunk j of row r at chunk j ^ (r mod 8): each quarter-warp's
// stores cover all 32 banks), and one lane stores the box with a TMA tile
// store.  Column x must be a multiple of 4 (16 bytes); a store is clipped at
// the tensor map's extent, never at a group boundary, so only fully valid
// 32-row slabs go this way.
__device__ __forceinline__ void stage_row_f32_sw128(uint8_t* stg, int lane, const float* v) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}
// Make this thread's shared-memory writes visible to the async proxy (TMA).
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// 2D tiled store shared -> global of the box at (x, y), in this thread's
// bulk async-group (commit with bulk_commit).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(smem_src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Until at most N of this thread's committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Until all of this thread's committed bulk groups are complete (writes done).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Element offset of (row n, column k) of a K-major bf16 matrix stored as
// 128-row x 64-column tiles (row-block-major, then column-block) with the
// 128-byte swizzle inside each 16 KB tile: the 16-byte chunk c of row r sits
// at chunk c ^ (r mod 8), as a 128-byte-swizzled TMA load would place it.
__host__ __device__ __forceinline__ int64_t tiled_offset(int64_t n, int64_t k, int64_t k_blocks) {
    const int64_t blk = (n >> 7) * k_blocks + (k >> 6);
    const int r = static_cast<int>(n & 127), c = static_cast<int>(k & 63);
    return blk * 8192 + r * 64 + ((((c >> 3) ^ (r & 7)) << 3) | (c & 7));
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---------------------------------------------------------------- tcgen05
// Allocate `ncols` TMEM columns (power of two >= 32); the base address is
// written to shared memory.  Must be executed by one whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(smem_slot)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored with the
// 128-byte swizzle as TMA writes it: rows of 64 bf16 (128 B), 8-row groups of
// 1024 B.  Leading offset 16 B (unused for this layout), stride offset
// 1024 B, descriptor version 1, layout code 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, both operands K-major, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(uint32_t M, uint32_t N) {
    return (1u << 4)            // D format f32
         | (1u << 7)            // A format bf16
         | (1u << 10)           // B format bf16
         | ((N >> 3) << 17)
         | ((M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, one 128 x N x 16 step.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05.mma of this thread
// have completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}

// Load 32 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t elect_lane0() {
    return (threadIdx.x & 31u) == 0u;
}

}  // namespace moe
