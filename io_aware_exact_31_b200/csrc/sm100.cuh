// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// attention kernels use: mbarriers with bounded waits, TMA tensor/bulk copies,
// and the 5th-generation tensor core (tcgen05: TMEM alloc, MMA, commit, ld/st).
//
// Every wait in this file is bounded: it polls until the barrier phase
// completes, the CTA-wide abort flag is raised, or a wall-clock limit passes;
// on the last two it records an error code and returns false so the caller
// can unwind instead of hanging the GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace fa {

// Error codes written to the device error word (first error wins).
enum : uint32_t {
    DEV_OK = 0,
    DEV_TIMEOUT_BASE = 0x100,  // + a site id: which wait gave up
};

// Wall-clock bound of one barrier wait.  A correct launch never waits longer
// than a few milliseconds at any barrier.
#ifndef FA_WAIT_TIMEOUT_NS
#define FA_WAIT_TIMEOUT_NS 2000000000ull
#endif

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }
__device__ __forceinline__ uint32_t warp_id() { return threadIdx.x >> 5; }

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Programmatic dependent launch: grid_dep_wait blocks the calling thread
// until the grids this launch depends on have completed and their writes are
// visible; grid_dep_launch lets the dependent launch start once every CTA of
// this grid has executed it (or exited).
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, P;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Per-CTA failure state: a shared abort flag (so one timed-out wait releases
// every other waiting role quickly) and a global error word for the host.
struct Guard {
    volatile int* abort_flag;  // shared memory
    uint32_t* err;             // global memory, may be null
};

__device__ __forceinline__ void guard_fail(const Guard& g, uint32_t code) {
    *g.abort_flag = 1;
    if (g.err) atomicCAS(g.err, 0u, code);
}

// Wait until the phase with the given parity has completed.  Returns false
// (after recording `site`) on timeout or when another role already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const Guard& g,
                                          uint32_t site,
                                          uint64_t timeout_ns = FA_WAIT_TIMEOUT_NS) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_test(bar, parity)) return true;
        if (*g.abort_flag) return false;
        if (globaltimer() - t0 > timeout_ns) {
            guard_fail(g, DEV_TIMEOUT_BASE + site);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag: used only to let copies that were
// already issued land before the CTA exits.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_test(bar, parity))
        if (globaltimer() - t0 > FA_WAIT_TIMEOUT_NS) return;
}

// Bounded wait until a global counter reaches `target` (acquire).  Gives up,
// returning false, when the CTA aborts, when another CTA has already recorded
// an error in the device error word (so that CTAs queued behind a failed one
// do not each wait out the full limit), or after the wall-clock limit.
__device__ __forceinline__ bool wait_counter(const int* cnt, int target, const Guard& g,
                                             uint32_t site) {
    const uint64_t t0 = globaltimer();
    while (true) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
        if (v >= target) return true;
        if (*g.abort_flag) return false;
        if (g.err && *reinterpret_cast<volatile uint32_t*>(g.err) != 0u) {
            *g.abort_flag = 1;
            return false;
        }
        if (globaltimer() - t0 > FA_WAIT_TIMEOUT_NS) {
            guard_fail(g, DEV_TIMEOUT_BASE + site);
            return false;
        }
        __nanosleep(64);
    }
}

// counter += 1 with release semantics at GPU scope.
__device__ __forceinline__ void counter_release_add(int* cnt) {
    asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(cnt) : "memory");
}

// Order this thread's generic-proxy and async-proxy (bulk copy) accesses to
// global memory with respect to each other.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Warp-collective wait: every lane polls (each acquires the barrier), then the
// outcome is made uniform and the warp reconverged, so the .sync.aligned
// tcgen05 instructions that follow are executed by all 32 lanes together.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, const Guard& g,
                                               uint32_t site) {
    const bool ok = mbar_wait(bar, parity, g, site);
    return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------
// Named barriers (subsets of warps)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ANDs a predicate over the participating threads.
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %3, 0;\n\t"
        "bar.red.and.pred q, %1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(id), "r"(nthreads), "r"(static_cast<uint32_t>(pred))
        : "memory");
    return r != 0;
}

// ---------------------------------------------------------------------------
// Register reallocation between warpgroups (all 4 warps of a warpgroup must
// execute the same instruction; the sum over warps must stay within the
// registers the CTA was launched with).
// ---------------------------------------------------------------------------
template <uint32_t N>
__device__ __forceinline__ void regs_increase() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_decrease() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------------------
// Proxy fences
// ---------------------------------------------------------------------------
// Make generic-proxy writes to shared memory visible to the async proxy
// (tensor core operand reads, bulk copies).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled load (no multicast) completing on `bar` with the box's byte count.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y, int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// Bring a 3-D tile into L2 ahead of its load (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* map, int32_t x, int32_t y,
                                                   int32_t z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}

// Same with an L2 eviction-priority hint (policy from createpolicy).
__device__ __forceinline__ void tma_load_3d_hint(void* smem_dst, const CUtensorMap* map,
                                                 uint64_t* bar, int32_t x, int32_t y, int32_t z,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z),
        "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 3-D tiled shared -> global store, tracked by the bulk async-group.  Rows and
// columns outside the tensor are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* smem_src, int32_t x,
                                             int32_t y, int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// 3-D tiled shared -> global add-reduction (tensor map element type decides
// the arithmetic, e.g. fp32 add), tracked by the bulk async-group.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* smem_src,
                                                  int32_t x, int32_t y, int32_t z) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group"
        " [%0, {%2, %3, %4}], [%1];" ::"l"(reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(smem_src)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// Contiguous global -> shared copy (16-byte aligned, size multiple of 16).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Contiguous shared -> global fp32 add-reduction (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_reduce_add_f32(float* gdst, const void* smem_src,
                                                    uint32_t bytes) {
    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                     reinterpret_cast<uint64_t>(gdst)),
                 "r"(smem_u32(smem_src)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until all committed bulk groups have finished READING shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Wait until all committed bulk groups have fully completed.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation tensor core
// ---------------------------------------------------------------------------
// TMEM address: bits [31:16] lane, bits [15:0] column (32-bit columns).
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
    return base + (lane << 16) + col;
}

// Executed by one full warp.  Writes the allocated base address to smem.
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_dst)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulator.
// a_mn / b_mn select MN-major (transposed) operands in shared memory.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N, bool a_mn, bool b_mn) {
    return (1u << 4)                        // D format: f32
           | (1u << 7)                      // A format: bf16
           | (1u << 10)                     // B format: bf16
           | ((a_mn ? 1u : 0u) << 15)       // A major
           | ((b_mn ? 1u : 0u) << 16)       // B major
           | ((N >> 3) << 17)               // N / 8
           | ((M >> 4) << 24);              // M / 16
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand tile.
//  K-major:  rows of 128 B (64 bf16 along K), 8-row groups `sbo` bytes apart.
//  MN-major: 64 bf16 along MN per 128-B row, K rows 128 B apart, 8-row K
//            groups `sbo` bytes apart, successive 64-wide MN chunks `lbo`
//            bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46)  // version
           | (2ull << 61);                                                       // SWIZZLE_128B
}

// Descriptor d advanced by k 16-byte units: added to the start-address field
// (bits 0-13) in the low word only, which cannot carry while the shared
// address stays below 2^18.
__device__ __forceinline__ uint64_t desc_off(uint64_t d, uint32_t k) {
    const uint32_t lo = static_cast<uint32_t>(d) + k;
    return (d & 0xFFFFFFFF00000000ull) | lo;
}

// Instruction descriptor, kind::f8f6f4 with E4M3 A/B and fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_e4m3(uint32_t M, uint32_t N, bool b_mn) {
    return (1u << 4)                        // D format: f32
           | (0u << 7) | (0u << 10)         // A, B format: E4M3
           | ((b_mn ? 1u : 0u) << 16)       // B major
           | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// MMA issue.  The whole warp, converged, executes the call; elect.sync inside
// the instruction block picks one lane (the same lane every time in a fully
// converged warp, so tc_commit_w tracks the MMAs that lane issued).  NSTEP
// K-steps of one accumulation go out from a single inline-PTX block with one
// elect.sync.  Step k > 0 reads the operands at the base descriptors advanced by
// a compile-time number of 16-byte units (added to the start-address field,
// which cannot carry below 256 KB of shared memory); the first step accumulates
// when `acc` is non-zero, the others always do.
//
// Issued this way one warp keeps the tensor core at its full rate: M = 128,
// N = 128, K = 16 bf16 MMAs complete every ~64 clocks whether A comes from
// shared memory or TMEM, also in the forward's sequence of two P.V halves and
// an S (with other warps streaming tcgen05.ld / st or exponentials meanwhile),
// and N = 64 ones every ~42-48.  One elect.sync block per MMA costs ~94 (SS) /
// ~104 (TS) clocks per instruction whatever N is up to 128, and a lane-0 branch
// of a diverged warp ~140 (microbenchmarks on B200, 148 SMs, one issuing warp
// per SM).
//
// Offset patterns (16-byte units at step k):
//   FA_STEP_KMAJOR (0): K-major 128-byte-swizzled tile, 32-byte K-steps inside
//                       128-byte rows, 64-element (bf16) row chunks 16 KB apart;
//   P > 0:              P units per step (MN-major tiles: K rows of 128 bytes).
#define FA_STEP_KMAJOR 0
template <int P>
__host__ __device__ constexpr uint32_t blk_off(int k) {
    return P == FA_STEP_KMAJOR ? static_cast<uint32_t>((k / 4) * 1024 + (k % 4) * 2)
                               : static_cast<uint32_t>(k * P);
}

#define FA_BLK_HEAD                                                                    \
    "{\n\t.reg .pred p, q, e;\n\t.reg .b64 a, b;\n\t.reg .b32 t;\n\t"                    \
    "elect.sync _|e, 0xffffffff;\n\t"                                                    \
    "setp.ne.b32 p, %4, 0;\n\t"                                                          \
    "setp.eq.b32 q, %4, %4;\n\t"
#define FA_SS0(K) "@e tcgen05.mma.cta_group::1.kind::" K " [%0], %1, %2, %3, p;\n\t"
#define FA_SSN(K, OA, OB)                                                              \
    "add.s64 a, %1, " OA ";\n\tadd.s64 b, %2, " OB ";\n\t"                             \
    "@e tcgen05.mma.cta_group::1.kind::" K " [%0], a, b, %3, q;\n\t"
#define FA_TS0(K) "@e tcgen05.mma.cta_group::1.kind::" K " [%0], [%1], %2, %3, p;\n\t"
#define FA_TSN(K, OA, OB)                                                              \
    "add.s32 t, %1, " OA ";\n\tadd.s64 b, %2, " OB ";\n\t"                             \
    "@e tcgen05.mma.cta_group::1.kind::" K " [%0], [t], b, %3, q;\n\t"

#define FA_IN5_SS "r"(d), "l"(a0), "l"(b0), "r"(id), "r"(acc)
#define FA_IN5_TS "r"(d), "r"(a0), "l"(b0), "r"(id), "r"(acc)
#define FA_OFF2(F, G) "n"(F(1)), "n"(G(1))
#define FA_OFF4(F, G) "n"(F(1)), "n"(F(2)), "n"(F(3)), "n"(G(1)), "n"(G(2)), "n"(G(3))
#define FA_OFF8(F, G)                                                                  \
    "n"(F(1)), "n"(F(2)), "n"(F(3)), "n"(F(4)), "n"(F(5)), "n"(F(6)), "n"(F(7)),       \
        "n"(G(1)), "n"(G(2)), "n"(G(3)), "n"(G(4)), "n"(G(5)), "n"(G(6)), "n"(G(7))

#define FA_DEFINE_BLK(NAME, KIND, ATYPE, S0, SN, IN5)                                          \
    template <int NSTEP, int PA, int PB>                                                  \
    __device__ __forceinline__ void NAME(uint32_t d, ATYPE a0, uint64_t b0, uint32_t id,  \
                                         uint32_t acc) {                                  \
        static_assert(NSTEP == 2 || NSTEP == 4 || NSTEP == 8, "NSTEP must be 2, 4 or 8"); \
        if constexpr (NSTEP == 2) {                                                       \
            asm volatile(FA_BLK_HEAD S0(KIND) SN(KIND, "%5", "%6") "}" ::IN5,          \
                         FA_OFF2(blk_off<PA>, blk_off<PB>));                              \
        } else if constexpr (NSTEP == 4) {                                                \
            asm volatile(FA_BLK_HEAD S0(KIND) SN(KIND, "%5", "%8") SN(KIND, "%6", "%9")  \
                             SN(KIND, "%7", "%10") "}" ::IN5,                          \
                         FA_OFF4(blk_off<PA>, blk_off<PB>));                              \
        } else {                                                                          \
            asm volatile(FA_BLK_HEAD S0(KIND) SN(KIND, "%5", "%12") SN(KIND, "%6", "%13") \
                             SN(KIND, "%7", "%14") SN(KIND, "%8", "%15")                  \
                                 SN(KIND, "%9", "%16") SN(KIND, "%10", "%17")             \
                                     SN(KIND, "%11", "%18") "}" ::IN5,                 \
                         FA_OFF8(blk_off<PA>, blk_off<PB>));                              \
        }                                                                                 \
    }

// D (+)= A[smem] B[smem]^T, NSTEP K-steps; PA / PB: offset patterns of A and B.
FA_DEFINE_BLK(mma_ss_blk, "f16", uint64_t, FA_SS0, FA_SSN, FA_IN5_SS)
FA_DEFINE_BLK(mma_ss_f8_blk, "f8f6f4", uint64_t, FA_SS0, FA_SSN, FA_IN5_SS)
// D (+)= A[tmem] B[smem]^T, NSTEP K-steps; A advances by PA columns per step.
FA_DEFINE_BLK(mma_ts_blk, "f16", uint32_t, FA_TS0, FA_TSN, FA_IN5_TS)
FA_DEFINE_BLK(mma_ts_f8_blk, "f8f6f4", uint32_t, FA_TS0, FA_TSN, FA_IN5_TS)

// Arrive once on `bar` when every tcgen05 op issued so far by the elected lane
// (the one that issued the MMAs) is done.  Warp-collective.
__device__ __forceinline__ void tc_commit_w(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Load 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// lane (lane_base + t).  The warp may only touch its own 32-lane quarter
// (warp_id % 4).  Results are valid only after tmem_ld_wait().
#define FA_R32(r)                                                                             \
    "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),       \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), \
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),           \
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),           \
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])

#define FA_W32(r)                                                                             \
    "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),   \
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),     \
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),   \
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),   \
        "r"(r[29]), "r"(r[30]), "r"(r[31])

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : FA_R32(r)
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        FA_W32(r)
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Tie registers written by tcgen05.ld to a point after tcgen05.wait::ld, so the
// compiler cannot hoist their uses above the wait.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t* r) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}

// ---------------------------------------------------------------------------
// Small math helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// acc.x += the low bf16 of w, acc.y += its high bf16: one mixed-precision add
// (bf16 operand, f32 accumulator, round to nearest) per half.  The result is
// bit-identical to widening each half to f32 and adding, without the two
// integer operations the widening costs.
__device__ __forceinline__ void add_bf16x2_f32(float2& acc, uint32_t w) {
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\t"
        "add.rn.f32.bf16 %1, hi, %1;\n\t}"
        : "+f"(acc.x), "+f"(acc.y)
        : "r"(w));
}

// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// The two bf16 halves of a packed pair, widened exactly to fp32.
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two fp32 -> two E4M3 (round to nearest, saturate to the finite range),
// lo in bits [7:0], hi in bits [15:8].
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Four E4M3 (bytes of w, lowest first) widened exactly to fp32, as two pairs.
__device__ __forceinline__ void unpack_e4m3x4(uint32_t w, float2& a, float2& b) {
    uint32_t h01, h23;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "mov.b32 {lo, hi}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
        : "=r"(h01), "=r"(h23)
        : "r"(w));
    a = __half22float2(*reinterpret_cast<const __half2*>(&h01));
    b = __half22float2(*reinterpret_cast<const __half2*>(&h23));
}

__device__ __forceinline__ void st_shared_v4(uint32_t saddr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ float4 ld_shared_v4f(uint32_t saddr) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(saddr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void st_global_v4(void* p, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

}  // namespace fa
