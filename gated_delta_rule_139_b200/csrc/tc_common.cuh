// tc_common.cuh -- Blackwell (sm_100a) building blocks written as inline PTX:
// tcgen05 MMAs with TMEM accumulators, shared-memory matrix descriptors for the
// 128-byte-swizzled canonical layouts, TMEM allocation / load / store, and
// mbarriers with bounded waits.
//
// Operand layouts (bf16, 128-byte swizzle; every tile base is 1024-byte aligned):
//
//  K-major tile, R rows x K elements (K a multiple of 64): stored as K/64
//  "K-blocks"; K-block kb holds columns [64kb, 64kb+64) of all R rows, one
//  128-byte line per row, 8-row groups 1024 bytes apart.  Inside a line the
//  16-byte chunk c of row r sits at chunk position c ^ (r % 8).
//
//  MN-major tile, K rows x MN elements (MN a multiple of 64): stored as MN/64
//  "MN-blocks"; MN-block mb holds elements [64mb, 64mb+64) of all K rows, one
//  128-byte line per K row, same 8-line swizzle atom.
//
// An MMA reads K = 16 bf16 per instruction: for K-major operands the
// descriptor start advances 32 bytes inside a line (and jumps to the next
// K-block every 4 steps); for MN-major operands it advances 2 swizzle atoms
// (2048 bytes).
#pragma once
#include <cuda_bf16.h>
#include <stdint.h>

namespace kda {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- layouts
// byte offset of element (r, k) in a K-major tile of R rows
__device__ __forceinline__ uint32_t kmajor_off(int r, int k, int R) {
    const int kb = k >> 6, kk = k & 63;
    const int chunk = (kk >> 3) ^ (r & 7);
    return (uint32_t)(kb * R * 128 + (r >> 3) * 1024 + (r & 7) * 128 + chunk * 16 + (kk & 7) * 2);
}
// byte offset of the 16-byte chunk holding elements (r, 8c..8c+7), K-major
__device__ __forceinline__ uint32_t kmajor_chunk_off(int r, int c8, int R) {
    const int kb = c8 >> 3, cc = c8 & 7;
    return (uint32_t)(kb * R * 128 + (r >> 3) * 1024 + (r & 7) * 128 + ((cc ^ (r & 7)) * 16));
}
// byte offset of element (k, mn) in an MN-major tile of K rows
__device__ __forceinline__ uint32_t mnmajor_off(int k, int mn, int K) {
    const int mb = mn >> 6, m = mn & 63;
    const int chunk = (m >> 3) ^ (k & 7);
    return (uint32_t)(mb * K * 128 + (k >> 3) * 1024 + (k & 7) * 128 + chunk * 16 + (m & 7) * 2);
}
// byte offset of the 16-byte chunk holding elements (k, 8c..8c+7), MN-major
__device__ __forceinline__ uint32_t mnmajor_chunk_off(int k, int c8, int K) {
    const int mb = c8 >> 3, cc = c8 & 7;
    return (uint32_t)(mb * K * 128 + (k >> 3) * 1024 + (k & 7) * 128 + ((cc ^ (k & 7)) * 16));
}

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor (sm_100 layout): start address >> 4 in bits
// [0,14), leading byte offset >> 4 in [16,30), stride byte offset >> 4 in
// [32,46), version 1 in [46,48), swizzle mode in [61,64) (2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// descriptor of k-step s (16 elements) of a K-major tile with R rows
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int R, int s) {
    return sdesc(base + (uint32_t)((s >> 2) * R * 128 + (s & 3) * 32), 16, 1024);
}
// descriptor of k-step s (16 K rows) of an MN-major tile with K rows
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t base, int K, int s) {
    return sdesc(base + (uint32_t)(s * 2048), (uint32_t)(K * 128), 1024);
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulate:
// D format bits [4,6) = 1 (f32); A, B formats [7,10), [10,13) = 1 (bf16);
// negate A bit 13; A major bit 15, B major bit 16 (1 = MN-major);
// N >> 3 in [17,23); M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn,
                                                  bool neg_a = false) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((neg_a ? 1u : 0u) << 13) |
           ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
// D (+)= A . B with A (M = 128 rows = TMEM lanes, bf16 pairs packed into 32-bit
// columns: element (m, k) at lane m, column k/2, low half for even k) read from
// TMEM at a_tmem, B from shared memory
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate));
}
// arrive on an mbarrier once every tcgen05 op issued so far by this thread is done
__device__ __forceinline__ void mma_commit(void* mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(mbar))
                 : "memory");
}
__device__ __forceinline__ void tmem_alloc(void* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
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
// make generic-proxy shared-memory writes visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// TMEM -> registers: this warp's 32 lanes, 16 consecutive 32-bit columns
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t* u = reinterpret_cast<uint32_t*>(v);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
        "%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
          "=r"(u[7]), "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]),
          "=r"(u[14]), "=r"(u[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    const uint32_t* u = reinterpret_cast<const uint32_t*>(v);
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16};" ::"r"(taddr),
        "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]),
        "r"(u[8]), "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]),
        "r"(u[15])
        : "memory");
}
// registers -> TMEM: this warp's 32 lanes, 8 consecutive 32-bit columns
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&u)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
        "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7])
        : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// wait for outstanding TMEM loads; the 16 destination registers are tied to the
// wait so that no use of them can be scheduled before it
__device__ __forceinline__ void tmem_wait16(float (&v)[16]) {
    uint32_t* u = reinterpret_cast<uint32_t*>(v);
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(u[0]), "+r"(u[1]), "+r"(u[2]), "+r"(u[3]), "+r"(u[4]), "+r"(u[5]),
                   "+r"(u[6]), "+r"(u[7]), "+r"(u[8]), "+r"(u[9]), "+r"(u[10]), "+r"(u[11]),
                   "+r"(u[12]), "+r"(u[13]), "+r"(u[14]), "+r"(u[15])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// TMEM address of (lane, column): lane in bits [16,32), column in [0,16)
__device__ __forceinline__ uint32_t taddr(uint32_t base, int lane, int col) {
    return base + ((uint32_t)lane << 16) + (uint32_t)col;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(void* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(void* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// The same test, but the thread may be suspended (issuing nothing) until the phase
// completes or about `hint_ns` nanoseconds pass, so waiting warps leave the issue
// slots to the warps that have work.
__device__ __forceinline__ bool mbar_try_wait_sleep(void* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait: gives up after `timeout_ns` nanoseconds of wall time, records
// `code` in *err (first error wins) and returns false.  Callers then stop
// issuing work, release their TMEM and return.
__device__ __forceinline__ bool mbar_wait(void* bar, uint32_t parity, int* err, int code,
                                          uint64_t timeout_ns = 1000000000ull) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 1000000u)) return true;
        if (globaltimer_ns() - t0 > timeout_ns) {
            if (err) atomicCAS(err, 0, code);
            return false;
        }
    }
}

// plain arrive (release) on an mbarrier
__device__ __forceinline__ void mbar_arrive(void* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- named barriers
// bar.sync on barrier `id` (1..15) among `n` threads (whole warps); id 0 is __syncthreads.
__device__ __forceinline__ void bar_named(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// the same barrier, returning whether any participating thread passed pred = true
__device__ __forceinline__ bool bar_named_or(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// ---------------------------------------------------------------- packing
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void st_shared_v4(uint32_t saddr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(saddr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

}  // namespace tc
}  // namespace kda
