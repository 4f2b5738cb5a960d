// Thin wrappers over the sm_100a PTX instructions the tensor-core kernels use:
// mbarriers (with bounded waits), TMA tile loads, and tcgen05 (TMEM
// allocation, MMA issue/commit, TMEM loads and stores). Every wrapper is one
// documented PTX instruction; no library code is involved.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace ba {

// A wait that has not completed after this long gives up and reports
// BA_ERR_TIMEOUT instead of hanging the GPU.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------- mbarrier ---

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}\n"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}

// One lane's wait for the phase of `bar` with the given parity to complete.
// Returns false (after setting *abort) if the wait ran past limit_ns or
// another thread of the CTA already gave up.
__device__ __forceinline__ bool mbar_wait_lane(uint64_t *bar, uint32_t parity, volatile int *abort,
                                               uint64_t limit_ns = kWaitLimitNs)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (global_timer_ns() - t0 > limit_ns) {
            *abort = 1;
            return false;
        }
    }
}

// Waits for the phase of `bar` with the given parity to complete. Called by
// all 32 lanes of a warp: every lane waits and the result is made uniform, so
// that after a timeout no lane is left behind at a warp-collective
// instruction (elect.sync, tcgen05.ld, shuffles) that the others never reach.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                          uint64_t limit_ns = kWaitLimitNs)
{
    return __all_sync(0xffffffffu, mbar_wait_lane(bar, parity, abort, limit_ns));
}

// Barrier over a group of threads, on an mbarrier initialised with the group's
// thread count: every thread arrives, then waits (bounded) for the phase to
// complete, so a thread that has given up cannot leave the others waiting
// forever. `phase` is the caller's parity, flipped on each use. Arrival and
// wait order the group's shared-memory writes before its later reads.
__device__ __forceinline__ bool group_sync(uint64_t *bar, uint32_t &phase, volatile int *abort)
{
    mbar_arrive(bar);
    const bool ok = mbar_wait(bar, phase, abort);
    phase ^= 1;
    return ok;
}

// ------------------------------------------------------------------ TMA ---

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 2-D tiled load of one box into shared memory, completing on `bar`.
// x (innermost, elements) must be a multiple of 16 bytes; y may be anything,
// rows past the tensor's end are filled with zeros.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t x, int32_t y)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
                 "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
                 : "memory");
}

// Brings one box of a 2-D tensor into L2 ahead of its load (no shared memory
// is written and no barrier is involved).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int32_t x, int32_t y)
{
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
                 : "memory");
}

// 2-D tiled store of one box from shared memory to global memory, tracked by
// the issuing thread's bulk async-groups. x (innermost, elements) must be a
// multiple of 16 bytes and neither coordinate may be negative; rows past the
// tensor's end are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t x, int32_t y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Waits until at most N of this thread's bulk groups are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait_group()
{
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// 4-byte asynchronous copy global -> shared (no register staging).
__device__ __forceinline__ void cp_async_4(void *dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Arrives on `bar` once all of this thread's earlier cp.async copies have
// landed; the arrival is counted in the barrier's expected count.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Makes generic-proxy shared-memory writes visible to the async proxy
// (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// A 128-row tile whose first `valid` rows (valid < 128) belong to the current
// example holds the next example's rows after them, which a masked product
// would still multiply by a zero probability (and 0 x inf is NaN). Such a
// tile is loaded by load_tail_tile: the TMA (CHUNKS boxes of 128 rows x 64
// columns, each a 16 KB 128B-swizzled chunk at dst + c * 16 KB) completes on
// the producer warp's private barrier `tail`; the warp waits for it, clears
// rows [valid, 128) of every chunk (the swizzle permutes 16-byte units only
// within a row's own 128 bytes, so a row is the same 128 bytes swizzled or
// not), makes the clears visible to the tensor core's operand reads and then
// arrives on `full` (one plain arrival in place of the expect_tx one). Both
// functions are out of line, so that the kernels' hot loops (whose code sits
// at the edge of the instruction cache) carry only the common full-tile load.
// Called by all 32 lanes of the producer warp; false after a timed-out wait.
static __device__ __noinline__ bool finish_tail_tile(uint8_t *dst, int chunks, uint64_t *full, uint64_t *tail,
                                                     uint32_t tail_phase, int valid, volatile int *abort)
{
    constexpr uint32_t kChunkBytes = 128 * 128;
    const int lane = threadIdx.x & 31;
    if (!mbar_wait(tail, tail_phase, abort)) return false;
    const int v = valid < 0 ? 0 : valid;
    const int units = (128 - v) * 8; // 16-byte units from row v to the end of a chunk
    for (int c = 0; c < chunks; ++c) {
        uint4 *z = reinterpret_cast<uint4 *>(dst + c * kChunkBytes + v * 128);
        for (int u = lane; u < units; u += 32) z[u] = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(full);
    __syncwarp();
    return true;
}

static __device__ __noinline__ bool load_tail_tile(uint8_t *dst, int chunks, const CUtensorMap *map, uint64_t *full,
                                                   uint64_t *tail, uint32_t tail_phase, int32_t x, int32_t y,
                                                   int valid, volatile int *abort)
{
    constexpr uint32_t kChunkBytes = 128 * 128;
    if ((threadIdx.x & 31) == 0) {
        mbar_arrive_expect_tx(tail, chunks * kChunkBytes);
        for (int c = 0; c < chunks; ++c) tma_load_2d(dst + c * kChunkBytes, map, tail, x + 64 * c, y);
    }
    __syncwarp();
    return finish_tail_tile(dst, chunks, full, tail, tail_phase, valid, abort);
}

// -------------------------------------------------------------- tcgen05 ---

// Whole warp: allocate `ncols` TMEM columns; the base address lands in *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
// Called by all 32 lanes of the issuing warp; the elected lane (the lowest
// active one, the same lane that issues the MMAs below) commits, so the
// barrier tracks that lane's MMAs.
__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}\n" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T   (bf16 in, fp32 accumulate). Called by all 32
// lanes of one warp with the same operands; one elected lane issues. Issuing from
// a converged warp keeps the operands in uniform registers, which makes the
// issue several times faster than from a single-lane branch.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T   (A K-major in TMEM, two bf16 per column).
// Warp-collective like mma_ss.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
                 "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// D[tmem] (+)= (A[smem] * B[smem]^T) with MX block scaling: A, B E4M3 (K = 32
// per instruction), each row of A and of B scaled by the E8M0 factor held in
// TMEM at sfa / sfb (the byte given by the address's top two bits, which the
// instruction descriptor repeats). Warp-collective like mma_ss.
__device__ __forceinline__ void mma_mx_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p, e;\n\t"
                 "elect.sync _|e, 0xffffffff;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "@e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
                     d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
                 : "memory");
}

// Instruction descriptor of the block-scaled kind::mxf8f6f4 MMA with E4M3 A
// and B (K-major) and E8M0 scale factors; fp32 accumulator. Bits: [4,6) B
// scale-factor byte, [7,10) A format (0 = E4M3), [10,13) B format, [17,23)
// N >> 3, 23 scale format (1 = E8M0), [24,29) M >> 4, [29,31) A scale-factor
// byte; K = 32.
__host__ __device__ constexpr uint32_t idesc_mx_e4m3(int M, int N, uint32_t sfa_byte, uint32_t sfb_byte)
{
    return (sfb_byte << 4) | (uint32_t(N >> 3) << 17) | (1u << 23) | (uint32_t(M >> 4) << 24) | (sfa_byte << 29);
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulator.
// Bits: [4,6) D format (1 = f32), [7,10) A format (1 = bf16), [10,13) B
// format, 15 A major (1 = MN), 16 B major, [17,23) N >> 3, [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
           ((b_mn_major ? 1u : 0u) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
// Bits: [0,14) start >> 4, [16,30) leading byte offset >> 4, [32,46) stride
// byte offset >> 4, [46,48) version (1 on sm_100), [61,64) layout (2 = 128B
// swizzle). K-major: rows of 64 bf16 (128 B), 8-row groups `sbo` apart, lbo
// unused. MN-major: 64 contiguous MN elements per 128 B row, `lbo` between
// 64-element MN chunks, `sbo` between 8-row K groups.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
           (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

#define BA_R8(a, i) a[i], a[i + 1], a[i + 2], a[i + 3], a[i + 4], a[i + 5], a[i + 6], a[i + 7]

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// columns [col, col+32) of TMEM lane (warp's lane base + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]),
                   "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
                   "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}

// Waits for this thread's outstanding TMEM loads; the register barrier below
// keeps uses of the loaded registers after the wait.
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void reg_fence(uint32_t (&r)[N])
{
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i])::"memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t (&r)[4])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
                 "r"(r[14]), "r"(r[15])
                 : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
                 "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]),
                 "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),
                 "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]),
                 "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// --------------------------------------------------------------- scalar ---

// Per-warpgroup register budget (all four warps of the warpgroup execute it).
// The budgets of a CTA's warpgroups must add up to no more than it was
// launched with, or the increase waits for registers that never come free.
template <uint32_t N>
__device__ __forceinline__ void warpgroup_regs_inc()
{
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void warpgroup_regs_dec()
{
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Two fp32 lanes per instruction (sm_100 packed f32x2 arithmetic).
union F2Bits {
    float2 f;
    unsigned long long u;
};

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
    F2Bits A{a}, B{b}, C{c}, R;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(R.u) : "l"(A.u), "l"(B.u), "l"(C.u));
    return R.f;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b)
{
    F2Bits A{a}, B{b}, R;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(R.u) : "l"(A.u), "l"(B.u));
    return R.f;
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b)
{
    F2Bits A{a}, B{b}, R;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(R.u) : "l"(A.u), "l"(B.u));
    return R.f;
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 2^x on the FMA pipe for x <= 8 (values below 2^-125 come out as 2^-125 or
// smaller, far below what a bf16 P can hold next to the row maximum). Round x
// to the nearest integer n with the 1.5 * 2^23 trick, evaluate 2^(x-n) on
// [-0.5, 0.5] with a cubic fitted to 2^f (relative error < 8e-5, measured on a
// dense grid), and add n to the exponent field.
__device__ __forceinline__ float exp2_fma(float x)
{
    x = fmaxf(x, -125.f);
    const float t = x + 12582912.f;
    const float f = x - (t - 12582912.f);
    const float p = fmaf(fmaf(fmaf(0.055171654f, f, 0.24261115f), f, 0.69326097f), f, 0.99992806f);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// 32 bytes (eight words) to global memory in one instruction; dst must be
// 32-byte aligned. A warp storing one row per lane then writes whole 32-byte
// sectors with half the instructions of 16-byte stores.
__device__ __forceinline__ void st_global_32b(void *dst, const uint32_t *w)
{
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

} // namespace ba
