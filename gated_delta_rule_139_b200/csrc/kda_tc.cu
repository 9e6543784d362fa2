// kda_tc.cu -- KDA chunked forward on the 5th-generation tensor cores (sm_100a).
//
// Source of the method: aiblin.ru, "Kimi K3 -- открытая модель, которая обошла
// закрытых лидеров рынка".  Section "Как хранить миллион токенов в памяти":
// the state S (d_k x d_v) is rewritten per token, erase-then-write with
// strength beta and per-channel forget gate alpha clamped to [e^-5, 1].
// Section "Как распараллелили последовательное обновление": (i) all tokens of a
// chunk are processed in parallel and the state is then passed from chunk to
// chunk; (ii) a long prefill is cut into segments whose state transitions are
// computed in parallel on different SMs of one GPU and reassembled exactly,
// each segment being described by a local state (its effect on a zero state)
// and a token-dependent transition matrix: S_out = M S_in + B.
//
// Kernels (one launch each, all on the caller's stream):
//   seg_setup          : segment table from cu_seqlens (or B x T) on the device.
//   chunk_kernel<TRANS_CACHE>: "pass 1" of kda_fwd's segmented plan, per (segment,
//                        head) the transition (B, M) of the segment -- the chunk loop
//                        applied to B from 0 and to M from I -- and every chunk's
//                        operand images bulk-stored to the chunk cache.
//   chunk_kernel<TRANS>: the transitions alone (kda_transition, kda_fwd_noalloc).
//   seg_scan           : S_in(j+1) = M_j S_in(j) + B_j, sequential over the
//                        segments of a sequence, parallel over (sequence, head,
//                        8-row block).
//   cached_kernel      : "pass 3" of the segmented plan, the state chain and the
//                        output from the true incoming state, each chunk's operands
//                        read back from the chunk cache.
//   chunk_kernel<FWD>  : "pass 3" without a cache (unsegmented plans, the
//                        no-allocation entry point): the whole chunk loop.
//   chunk_kernel<DUMP> : test aid: every chunk's operand images (W, U', K_dec,
//                        Q~, P, gamma) copied to global memory.
//   wait_probe, guard_check: the bounded-wait self-test, and (debug builds) the
//                        check of the workspace guard bands.
//
// Per chunk of C = 64 tokens (g = in-chunk inclusive cumsum of the clamped
// log-gates, per key channel), everything in the transposed orientation so
// that every tensor-core product has M = 128 rows:
//   A  = strict_lower(diag(beta) (K e^g)(K e^-g)^T),  P = lower_incl((Q e^g)(K e^-g)^T)
//   T  = (I + A)^-1                                      (fp32, CUDA cores)
//   W^T = (K e^g)^T (T diag(beta))^T,   U'^T = V^T (T diag(beta))^T
//   U^T = U'^T - S^T W^T
//   O^T = S^T (Q e^g)^T + U^T P^T
//   S^T <- S^T Diag(e^{g_last}) + U^T (K e^{g_last - g})
// Gate factors for A and P are referenced to the middle of each 32-token half
// (rho_a = g_15, rho_b = g_47) so every factor handed to the tensor core lies
// in [e^-80, e^80]; the cross-half block of A and P takes k_s e^{rho_b - g_s}
// (<= 1) for the first half's keys.  The state-side operands K e^g, Q e^g and
// K e^{g_last - g} are products of factors whose exact value is <= 1.
//
// Warp roles inside each CTA (one CTA per SM, 16 warps):
//   warps 0-7 ("prep"): the chunk-local work of chunk c+1 -- gates, operand images,
//     [A;P] product, inversion, W and U' products -- into a two-slot shared-memory
//     ring (Q~, K_dec, P, gamma; the v tile in the W piece) and the W and U
//     accumulators in tensor memory.  One prep thread (the copy thread) issues every
//     TMA load of the raw tiles (log alpha + beta, k, q, v, a chunk ahead) and every
//     bulk store to the chunk cache;
//   warps 8-15 ("chain"): the state chain of chunk c -- W from tensor memory into
//     the slot, bf16 copy of S, U -= S W, S += U K_dec, O = S Q~ + U P and the output
//     epilogue; for the transitions the same two products on B and then on M.
// The two groups meet only at mbarriers (slot full / empty, U and W columns free),
// so one chunk's chunk-local work overlaps the previous chunk's state products.
#include <cuda_bf16.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "kda_internal.h"
#include "tc_common.cuh"

namespace kda {
namespace {

__device__ int g_tc_status = 0;  // first device-side error code of this device (0 = none)

// Debug builds (-DKDA_DEBUG): an index the kernel derives from a device-built table
// is checked against the buffer it addresses before the first access through it.  A
// failed check records ERR_DEBUG_INDEX with the source line and the whole block
// returns; the condition is uniform over the block, and the checks sit before any
// barrier, TMEM allocation or asynchronous copy.  Release builds compile them out.
#ifdef KDA_DEBUG
#define KDA_DCHECK(cond)                                                                    \
    do {                                                                                    \
        if (!(cond)) {                                                                      \
            if (threadIdx.x == 0) atomicCAS(&g_tc_status, 0, ERR_DEBUG_INDEX | (__LINE__ << 8)); \
            return;                                                                         \
        }                                                                                   \
    } while (0)
#else
#define KDA_DCHECK(cond) \
    do {                 \
    } while (0)
#endif
#ifdef KDA_DEBUG
// The segment entry lies inside its sequence: n in [0, N), lo <= t_begin <= t_end <= hi
// with t_begin on a chunk boundary of the sequence.
__device__ bool seg_entry_ok(const TcArgs& a, const SegEntry& sg) {
    if (sg.n < 0 || sg.n >= a.N) return false;
    const int64_t lo = a.cu ? (int64_t)a.cu[sg.n] : (int64_t)sg.n * a.T;
    const int64_t hi = a.cu ? (int64_t)a.cu[sg.n + 1] : lo + a.T;
    return lo <= sg.t_begin && sg.t_begin <= sg.t_end && sg.t_end <= hi && (sg.t_begin - lo) % kChunk == 0;
}
#endif

// Phase trace (builds with -DKDA_PHASE_TRACE only): the SM clock at the phase
// boundaries of kTraceChunks chunks of CTA (0, 0) from chunk g_trace_c0 on, per warp
// group (0 prep, 1 chain), and per CTA of the transition pass its start and end
// (global timer, ns), SM, chunk count and start and end SM clock; read back by
// kda_trace_read / kda_trace_spans.
#ifdef KDA_PHASE_TRACE
__device__ __forceinline__ unsigned long long smid_u32() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}
constexpr int kTraceChunks = 64, kTraceStamps = 16, kSpanCtas = 8192;
__device__ unsigned long long g_trace[2][kTraceChunks][kTraceStamps];
__device__ unsigned long long g_span[kSpanCtas][6];
__device__ long long g_trace_c0;
#define TRACE(grp, chunk, k)                                                                    \
    do {                                                                                        \
        if (blockIdx.x == 0 && blockIdx.y == 0 && (chunk) >= g_trace_c0 &&                      \
            (chunk) - g_trace_c0 < kTraceChunks)                                                \
            g_trace[grp][(chunk) - g_trace_c0][k] = clock64();                                  \
    } while (0)
#define SPAN(which, value)                                                                      \
    do {                                                                                        \
        const int cta_ = blockIdx.y * gridDim.x + blockIdx.x;                                   \
        if (cta_ < kSpanCtas) g_span[cta_][which] = (value);                                    \
    } while (0)
#else
#define TRACE(grp, chunk, k) \
    do {                     \
    } while (0)
#define SPAN(which, value) \
    do {                   \
    } while (0)
#endif

using namespace tc;

constexpr int C = 64;              // tokens per chunk
constexpr int D = 128;             // d_k = d_v
constexpr int NPREP = 256;         // prep threads (warps 0-7)
constexpr int NCHAIN = 256;        // chain threads (warps 8-15, two per TMEM lane quadrant)
constexpr int NT = NPREP + NCHAIN;
constexpr int TCOPY = 128;  // prep thread that issues the TMA loads and bulk stores
constexpr int BAR_PREP = 1, BAR_CHAIN = 2;  // named barriers of the two groups
constexpr float LOG2E = 1.4426950408889634f;

// FWD: forward from the true incoming state, every chunk's operands recomputed.
// TRANS: segment transitions.  TRANS_CACHE: segment transitions that also leave every
// chunk's operand images in the chunk cache for cached_kernel.  DUMP: operand images
// for the test entry point.
enum Mode : int { FWD = 0, TRANS = 1, DUMP = 2, TRANS_CACHE = 3 };

// ---------------------------------------------------------------- shared memory map
// Ring slot (two of them; chunk c uses slot c % 2), 1024-byte aligned pieces.  Each
// piece first receives one of the chunk's raw tiles by TMA, which the prep reads before
// it writes the piece's operand image over it:
//   S_W   v tile (two 64-channel boxes, 128-byte swizzle: the A operand of U'^T), then
//         W^T, MN-major (K rows = channels, MN = tokens); after the chain's U product
//         the chunk's output-gate tile, then its bf16 output tile [64][128] for the TMA
//         store (forward pass)
//   S_KD  k tile [64][128] bf16, then K_dec = K e^{g_last - g}, MN-major (K rows = tokens)
//   S_QT  q tile, then Q~ = Q e^g, K-major [64][128]          (forward pass)
//   S_PB  the eight warps' gate sums (fp32 [8][128]), then P, K-major [64][64]
//                                                             (forward pass)
//   S_GAM gamma = e^{g_last}, fp32 [128]
// Prep scratch:
//   X1    [A;P] A operand, K-major 128 x 128: rows 0-63 k e^{g-rho}, rows 64-127
//         q e^{g-rho} (forward pass)
//   BT    [A;P] B operand, K-major 96 x 128: rows 0-63 k e^{rho-g}, rows 64-95
//         the cross-half keys k e^{rho_b-g} of tokens 0-31
//   after the [A;P] product X1 and BT hold As, Ts, Ys (the inversion's fp32
//   scratch) and TB = T diag(beta) (bf16, K-major [r][s])
//   KG    K e^g, MN-major (K rows = tokens): A operand of W^T
//   LA    the next chunk's log alpha tile [64][128] fp32 (TMA)
//   GSUM  the gate sums when the slot has no P piece (transitions)
template <int MODE>
struct Lay {
    static constexpr bool Q = MODE != TRANS;  // the prep builds q~ rows, Q~ and P
    static constexpr uint32_t S_W = 0, S_KD = 16384, S_QT = 32768, S_PB = 49152;
    static constexpr uint32_t S_GAM = Q ? 57344 : 32768;
    static constexpr uint32_t SLOT = Q ? 58368 : 33792;
    static constexpr uint32_t X1 = 2 * SLOT;
    static constexpr uint32_t BT = X1 + 32768;
    static constexpr uint32_t KG = BT + 24576;
    static constexpr uint32_t LA = KG + 16384;
    static constexpr uint32_t AS = X1, TS = AS + 17408, YS = TS + 18432, TB = YS + 5120;
    static constexpr uint32_t BTILE = LA + 32768;  // the log alpha tile's beta: fp32 [64][4 heads]
    static constexpr uint32_t GSUM = BTILE + 1024; // fp32 [14][128] (transitions only)
    static constexpr uint32_t BETA = GSUM + (Q ? 0 : 8192);  // fp32 [64]
    static constexpr uint32_t BAR = BETA + 256;    // mbarriers
    static constexpr uint32_t TMEMP = BAR + 256;   // TMEM base address
    static constexpr uint32_t BYTES = TMEMP + 16 + 1024;  // + alignment slack
};
static_assert(Lay<FWD>::S_GAM + 512 <= Lay<FWD>::SLOT && Lay<FWD>::SLOT % 1024 == 0, "slot");
static_assert(Lay<TRANS>::S_GAM + 512 <= Lay<TRANS>::SLOT && Lay<TRANS>::SLOT % 1024 == 0, "slot");
static_assert(Lay<FWD>::TB % 1024 == 0 && Lay<FWD>::TB + 8192 <= Lay<FWD>::KG, "TB in X1/BT");
static_assert(Lay<FWD>::BYTES <= 232448 && Lay<TRANS>::BYTES <= 232448, "shared memory");

// mbarriers (index into BAR)
enum Bars : int {
    B_AP = 0,      // prep: [A;P] product done
    B_WU = 1,      // W and U' products done (issued by the chain, waited for by both groups)
    B_V = 2,       // prep: a chunk's v tile landed in slot 0 (TMA; one per use of the slot)
    B_FULL = 3,    // [2] ring slot filled (prep -> chain)
    B_EMPTY = 5,   // [2] the chain's products have read the slot (MMA commit)
    B_WFREE = 7,   // [2] the slot's W area is free again (output tile stored)
    B_U = 10,      // chain: U product done
    B_S = 11,      // chain: state update done
    B_O = 12,      // [2] chain: output products of O buffer 0/1 done
    B_GATE = 14,   // chain: output-gate tile landed (TMA)
    B_LA = 15,     // prep: a chunk's log alpha tile landed (TMA; one per chunk)
    B_KQ = 16,     // prep: a chunk's k (and q) tiles landed in its slot (TMA; one per chunk)
    B_V1 = 17,     // prep: a chunk's v tile landed in slot 1
    B_WREAD = 18,  // chain: the chunk's W^T has left TMEM (the prep may overwrite its columns)
    NBARS = 19
};

// TMEM columns (512 allocated).
//   forward:     AP [0,96) (W in [0,64) after the inversion) U [96,160)
//                O0 [160,224) O1 [224,288) SB [288,352) UB [352,384) S [384,512)
//   transition:  AP/W as above, U [96,160) SB [160,224) UB [224,256)
//                B [256,384) M [384,512)
constexpr uint32_t TM_AP = 0, TM_W = 0, TM_U = 96;
constexpr uint32_t TM_O = 160, TM_SB = 288, TM_UB = 352, TM_S = 384;  // forward
constexpr uint32_t TT_SB = 160, TT_UB = 224, TT_B = 256, TT_M = 384;  // transition

// Chunk operand images written by the DUMP mode (kChunkImageBytes per chunk and
// head): the bf16 operand images as they sit in shared memory, in 1024-byte
// aligned pieces, then gamma.
constexpr uint32_t CI_W = 0;        // W^T: MN-major, K rows = channels, MN = tokens
constexpr uint32_t CI_U = 16384;    // U'^T: [128][64], 16-byte pieces of row e XOR-swizzled by e & 7
constexpr uint32_t CI_KD = 32768;   // K_dec: MN-major, K rows = tokens, MN = channels
constexpr uint32_t CI_QT = 49152;   // Q~: K-major, 64 rows x 128
constexpr uint32_t CI_PB = 65536;   // P: K-major, 64 x 64
constexpr uint32_t CI_GAM = 73728;  // fp32 [128] e^{g_last}
static_assert(CI_GAM + 512 == kChunkImageBytes, "chunk image");

// Chunk cache entry (kCacheEntryBytes per chunk and head), written by pass 1 with the
// cache and read by cached_kernel: the bf16 operand images as they sit in shared memory,
// in 1024-byte aligned pieces (one bulk copy into a 1024-byte aligned buffer keeps their
// 128-byte swizzle), then gamma.
constexpr uint32_t CE_W = 0;        // W^T: MN-major, K rows = channels, MN = tokens
constexpr uint32_t CE_KD = 16384;   // K_dec: MN-major, K rows = tokens
constexpr uint32_t CE_QT = 32768;   // Q~: K-major, 64 rows
constexpr uint32_t CE_PB = 49152;   // P: K-major 64 x 64
constexpr uint32_t CE_TB = 57344;   // T diag(beta): K-major [r][s] 64 x 64
constexpr uint32_t CE_GAM = 65536;  // fp32 [128] e^{g_last}
static_assert(CE_GAM + 512 == kCacheEntryBytes, "cache entry");

__device__ __forceinline__ float clamp_gate(float x) { return fminf(fmaxf(x, -5.f), 0.f); }
// 2^x by the SFU instruction (relative error about 2^-22, flushes results
// below 2^-126 to zero, which is harmless for the factors here)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// (r0, r1) = (a0 * b0, a1 * b1) and (a0 + b0, a1 + b1) in one packed f32x2 instruction; each
// element is rounded exactly as the scalar operation rounds it
__device__ __forceinline__ void mul2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
    asm("{\n .reg .b64 x, y, z;\n mov.b64 x, {%2, %3};\n mov.b64 y, {%4, %5};\n"
        " mul.rn.f32x2 z, x, y;\n mov.b64 {%0, %1}, z;\n}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void add2(float& r0, float& r1, float a0, float a1, float b0, float b1) {
    asm("{\n .reg .b64 x, y, z;\n mov.b64 x, {%2, %3};\n mov.b64 y, {%4, %5};\n"
        " add.rn.f32x2 z, x, y;\n mov.b64 {%0, %1}, z;\n}"
        : "=f"(r0), "=f"(r1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void add8(float (&r)[8], const float (&a)[8], const float (&b)[8]) {
#pragma unroll
    for (int p = 0; p < 8; p += 2) add2(r[p], r[p + 1], a[p], a[p + 1], b[p], b[p + 1]);
}



// read-only global load
__device__ __forceinline__ float ld_nc_f1(const float* p) {
    float v;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// Copy NB x 16 fp32 TMEM columns at tm (tile columns col0..) of this thread's
// lane into NB x 8 packed-bf16 columns at tb (an A operand read from TMEM);
// optionally scale the fp32 copy by gam[col0 + i] in place.
template <int NB>
__device__ __forceinline__ void stage_cols_tmem(uint32_t tm, uint32_t tb, int col0, const float* gam,
                                                bool scale_back) {
    float v[NB][16];
#pragma unroll
    for (int b = 0; b < NB; ++b) tmem_ld16(tm + 16 * b, v[b]);
#pragma unroll
    for (int b = 0; b < NB; ++b) tmem_wait16(v[b]);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        uint32_t u[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) u[i] = pack_bf16(v[b][2 * i], v[b][2 * i + 1]);
        tmem_st8(tb + 8 * b, u);
    }
    if (scale_back) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            const float4* g4 = reinterpret_cast<const float4*>(gam + col0 + 16 * b);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 gg = g4[i];
                mul2(v[b][4 * i + 0], v[b][4 * i + 1], v[b][4 * i + 0], v[b][4 * i + 1], gg.x, gg.y);
                mul2(v[b][4 * i + 2], v[b][4 * i + 3], v[b][4 * i + 2], v[b][4 * i + 3], gg.z, gg.w);
            }
            tmem_st16(tm + 16 * b, v[b]);
        }
    }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void mbar_expect_tx(void* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
// one [64 tokens][box width] tile of a [T, H, 128] tensor at (x, h, t0); rows
// past the tensor's end are filled with zeros
__device__ __forceinline__ void tma_tile(void* dst, const CUtensorMap* map, int x, int h, int t0,
                                         void* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(h), "r"(t0), "r"(smem_u32(bar))
        : "memory");
}
// the same tile into L2 only
__device__ __forceinline__ void tma_prefetch(const CUtensorMap* map, int x, int h, int t0) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(h), "r"(t0)
                 : "memory");
}
// shared [64 tokens][128 channels] tile -> global tile at (0, h, t0) of a [T, H, 128] tensor
__device__ __forceinline__ void tma_store_tile(const CUtensorMap* map, const void* src, int h, int t0) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(0), "r"(h), "r"(t0), "r"(smem_u32(src))
        : "memory");
}
// plain bulk copies: shared -> global (bulk group), global -> shared (mbarrier)
// Bulk copy shared -> global (bulk async-group) whose lines are the first to leave L2: the
// chunk cache is read back only after the whole pass, so keeping it in L2 would only push
// out the prefetched input tiles
__device__ __forceinline__ void bulk_store_stream(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile(
        "{\n .reg .b64 pol;\n createpolicy.fractional.L2::evict_first.b64 pol, 1.0;\n"
        " cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, pol;\n}" ::"l"(gdst),
        "r"(smem_u32(ssrc)), "r"(bytes)
        : "memory");
}
__device__ __forceinline__ void bulk_load(void* sdst, const void* gsrc, uint32_t bytes, void* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(sdst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// all but the most recent of the issuing thread's bulk groups have read shared memory
__device__ __forceinline__ void bulk_wait_read1() {
    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the issuing thread's bulk stores have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// ... and have completed
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// bounded wait with the kernel's status word
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity) {
    return mbar_wait(bar, parity, &g_tc_status, ERR_WAIT_TIMEOUT);
}

// ---------------------------------------------------------------- (I + A)^-1
constexpr int AS_LD = 68;  // row stride (floats) of As: A-fragment loads hit 32 banks
constexpr int TS_LD = 72;  // row stride of Ts: B-fragment loads hit 32 banks
constexpr int YS_LD = 40;  // row stride of the intermediate products

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// d (16 x 8, fp32) += a (16 x 8) . b (8 x 8) on the warp's tensor core (tf32 in,
// fp32 accumulate).  a: element (m, k) at a[m*lda + k]; b: (k, n) at b[k*ldb + n].
// Fragments (PTX m16n8k8 .tf32): g = lane/4, t = lane%4; a: (g,t) (g+8,t)
// (g,t+4) (g+8,t+4); b: (t,g) (t+4,g); d: (g,2t) (g,2t+1) (g+8,2t) (g+8,2t+1).
__device__ __forceinline__ void warp_mma_tf32(float (&d)[4], const float* a, int lda,
                                              const float* b, int ldb, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const uint32_t a0 = to_tf32(a[g * lda + t]), a1 = to_tf32(a[(g + 8) * lda + t]);
    const uint32_t a2 = to_tf32(a[g * lda + t + 4]), a3 = to_tf32(a[(g + 8) * lda + t + 4]);
    const uint32_t b0 = to_tf32(b[t * ldb + g]), b1 = to_tf32(b[(t + 4) * ldb + g]);
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void warp_store16x8(float* dst, int ld, const float (&d)[4], float sgn,
                                               int lane) {
    const int g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2*>(dst + g * ld + 2 * t) = make_float2(sgn * d[0], sgn * d[1]);
    *reinterpret_cast<float2*>(dst + (g + 8) * ld + 2 * t) = make_float2(sgn * d[2], sgn * d[3]);
}

// Run by the 256 prep threads once the [A;P] product is in TMEM.  Writes TB =
// T diag(beta) as the bf16 K-major [r][j] tile tbp, where T = (I + A)^-1 and A is
// read from the product (rows of A in TMEM lanes 0-63; tq = the calling warp's
// lane quadrant), using As, Ts (fp32) and Ys as scratch:
//  1. warp h (h = 0, 1) reads rows 32h..32h+31 of A from TMEM (scaled by beta,
//     strictly-lower mask) and builds the 32 x 32 diagonal half h of T: its two
//     16 x 16 diagonal blocks in fp32 by forward substitution (one column per lane,
//     both blocks at once), then T_21 = -T_22 (A_21 T_11) inside the half with tf32
//     warp MMAs; warps 2-5 zero the upper-right 32 x 32 block of TB; `side(warp)`
//     runs on warps 2-7 meanwhile;
//  2. TB of the two diagonal halves (all threads), and Z = A[32:64, 0:32] T_lo
//     (warps 0-7, one 16 x 8 tile each);
//  3. T[32:64, 0:32] = -T_hi Z, scaled by beta_j, straight into TB.
// The block products are tf32 warp MMAs with fp32 accumulation (T then enters the
// chunk products as bf16).
template <typename Side>
__device__ void invert_to_tb(float* As, float* Ts, float* Ys, const float* beta, uint32_t tbp,
                             int tid, uint32_t tq, Side side, int64_t chunk) {
    (void)chunk;  // phase trace only
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    if (warp < 2) {
        const int o = 32 * warp;
        const int r = o + lane;                  // this lane's row of A
        const int blk = lane >> 4, i = lane & 15, ob = o + 16 * blk;
        const float br = beta[r];
        // diagonal 16 x 16 block blk of this half, transposed: At[m][i] = A[ob+i][ob+m]
        // (block 1 sixteen banks after block 0; in rows of As the products never read)
        float* At = As + warp * 544 + blk * 272;
        {  // 1a. rows o..o+31 of A from TMEM in 32-column batches, one wait each: rows
           // 0-31 need columns 0-31; columns j < 32 of rows >= 32 are the cross-half
           // product (TMEM 64 + j), columns 32-63 of those rows the second half's block
#pragma unroll
            for (int bb = 0; bb < 2; ++bb) {
                if (warp == 0 && bb == 1) break;
                const int j0 = 32 * bb;  // tile columns j0 .. j0+31
                const uint32_t src = tq + TM_AP + (warp == 1 && bb == 0 ? 64 : j0);
                float v0[16], v1[16];
                tmem_ld16(src, v0);
                tmem_ld16(src + 16, v1);
                tmem_wait16(v0);
                tmem_wait16(v1);
                if (j0 == o) {
                    // the lane's row inside its diagonal block (strictly lower), transposed
#pragma unroll
                    for (int m = 0; m < 16; ++m) At[m * 16 + i] = m < i ? br * (blk ? v1[m] : v0[m]) : 0.f;
                    if (blk) {  // A_21 of the half (rows o+16.., columns o..o+15): row-major
#pragma unroll
                        for (int m4 = 0; m4 < 4; ++m4)
                            *reinterpret_cast<float4*>(As + r * AS_LD + o + 4 * m4) =
                                make_float4(br * v0[4 * m4], br * v0[4 * m4 + 1], br * v0[4 * m4 + 2],
                                            br * v0[4 * m4 + 3]);
                    }
                } else {  // rows 32-63, columns 0-31 (all below the diagonal): row-major
#pragma unroll
                    for (int m4 = 0; m4 < 8; ++m4) {
                        const float* vv = m4 < 4 ? v0 + 4 * m4 : v1 + 4 * (m4 - 4);
                        *reinterpret_cast<float4*>(As + r * AS_LD + 4 * m4) =
                            make_float4(br * vv[0], br * vv[1], br * vv[2], br * vv[3]);
                    }
                }
            }
            __syncwarp();
            if (tid == 0) TRACE(0, chunk, 8);
            // forward substitution in fp32, one column per lane: lane (blk, i) solves
            // (I + A_bb) x = e_i, updating every later row as soon as x_m is known, so
            // the steps are chained by one FMA each
            float xc[16];
#pragma unroll
            for (int m = 0; m < 16; ++m) xc[m] = m == i ? 1.f : 0.f;
#pragma unroll
            for (int m = 0; m < 15; ++m) {
                const float xm = xc[m];
#pragma unroll
                for (int i4 = (m + 1) >> 2; i4 < 4; ++i4) {
                    const float4 a = *reinterpret_cast<const float4*>(At + m * 16 + 4 * i4);
                    const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (4 * i4 + k > m) xc[4 * i4 + k] = fmaf(-av[k], xm, xc[4 * i4 + k]);
                }
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) Ts[(ob + m) * TS_LD + ob + i] = xc[m];
            // zero the upper-right 16 x 16 block of this half (rows o..o+15, cols o+16..o+31)
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int e = lane + 32 * x;
                *reinterpret_cast<float4*>(Ts + (o + (e >> 2)) * TS_LD + o + 16 + 4 * (e & 3)) =
                    make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
        __syncwarp();
        if (tid == 0) TRACE(0, chunk, 9);
        // 1b. Y = A_21 T_11 (16 x 16 x 16), then T_21 = -T_22 Y, within the half
        float* Yh = Ys + warp * 16 * YS_LD;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += 8)
                warp_mma_tf32(d, As + (o + 16) * AS_LD + o + k0, AS_LD,
                              Ts + (o + k0) * TS_LD + o + 8 * nt, TS_LD, lane);
            warp_store16x8(Yh + 8 * nt, YS_LD, d, 1.f, lane);
        }
        __syncwarp();
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k0 = 0; k0 < 16; k0 += 8)
                warp_mma_tf32(d, Ts + (o + 16) * TS_LD + o + 16 + k0, TS_LD, Yh + k0 * YS_LD + 8 * nt,
                              YS_LD, lane);
            warp_store16x8(Ts + (o + 16) * TS_LD + o + 8 * nt, TS_LD, d, -1.f, lane);
        }
        __syncwarp();
        if (tid == 0) TRACE(0, chunk, 10);
    } else {
        if (warp < 6) {  // zero TB rows 0..31, columns 32..63: 128 chunks
            const int id = tid - 64, r = id >> 2, j8 = 4 + (id & 3);
            st_shared_v4(tbp + kmajor_chunk_off(r, j8, 64), 0u, 0u, 0u, 0u);
        }
        side(warp);
    }
    bar_named(BAR_PREP, NPREP);
    if (tid == 0) TRACE(0, chunk, 11);
    {  // 2a. TB of the two diagonal halves: 2 x 32 rows x 4 chunks of 8 columns
        const int hf = tid >> 7, r = 32 * hf + ((tid >> 2) & 31), j8 = 4 * hf + (tid & 3);
        const float4 ta = *reinterpret_cast<const float4*>(Ts + r * TS_LD + 8 * j8);
        const float4 tb = *reinterpret_cast<const float4*>(Ts + r * TS_LD + 8 * j8 + 4);
        const float tr[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
        const float* bj = beta + 8 * j8;
        st_shared_v4(tbp + kmajor_chunk_off(r, j8, 64), pack_bf16(tr[0] * bj[0], tr[1] * bj[1]),
                     pack_bf16(tr[2] * bj[2], tr[3] * bj[3]), pack_bf16(tr[4] * bj[4], tr[5] * bj[5]),
                     pack_bf16(tr[6] * bj[6], tr[7] * bj[7]));
    }
    // 2b. Z = A[32:64, 0:32] T_lo: warp (mt, nt)
    const int mt = (warp >> 2) & 1, nt = warp & 3;
    {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 8)
            warp_mma_tf32(d, As + (32 + 16 * mt) * AS_LD + k0, AS_LD, Ts + k0 * TS_LD + 8 * nt,
                          TS_LD, lane);
        warp_store16x8(Ys + 16 * mt * YS_LD + 8 * nt, YS_LD, d, 1.f, lane);
    }
    bar_named(BAR_PREP, NPREP);
    if (tid == 0) TRACE(0, chunk, 12);
    // 3. T[32:64, 0:32] = -T_hi Z, scaled by beta_j, straight into TB
    {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 8)
            warp_mma_tf32(d, Ts + (32 + 16 * mt) * TS_LD + 32 + k0, TS_LD, Ys + k0 * YS_LD + 8 * nt,
                          YS_LD, lane);
        const int r = 32 + 16 * mt + g, j = 8 * nt + 2 * t4;
        const float b0 = beta[j], b1 = beta[j + 1];
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(tbp + kmajor_off(r, j, 64)),
                     "r"(pack_bf16(-d[0] * b0, -d[1] * b1)));
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(tbp + kmajor_off(r + 8, j, 64)),
                     "r"(pack_bf16(-d[2] * b0, -d[3] * b1)));
    }
}

// Row r (0-63) of P, columns j0..j0+15 (j0 a multiple of 16), from the [A;P] product
// in TMEM (P's rows in lanes 64-127; tq = the calling warp's lane quadrant): the
// lower-inclusive mask, bf16, into the K-major 64 x 64 image at pb.  Columns j < 32
// of rows r >= 32 are the cross-half product (TMEM columns 64 + j); rows r < 32 have
// nothing in columns j >= 32.  Warp-uniform: r < 32 for the whole quadrant or none.
__device__ __forceinline__ void extract_p16(uint32_t tq, int r, int j0, uint32_t pb) {
    float x[16];
    if (j0 >= 32 && r < 32) {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = 0.f;
    } else {
        float v[16];
        tmem_ld16(tq + TM_AP + (j0 < 32 && r >= 32 ? 64 + j0 : j0), v);
        tmem_wait16(v);
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = j0 + i <= r ? v[i] : 0.f;
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
        st_shared_v4(pb + kmajor_chunk_off(r, (j0 >> 3) + hh, 64), pack_bf16(x[8 * hh], x[8 * hh + 1]),
                     pack_bf16(x[8 * hh + 2], x[8 * hh + 3]), pack_bf16(x[8 * hh + 4], x[8 * hh + 5]),
                     pack_bf16(x[8 * hh + 6], x[8 * hh + 7]));
}

// ---------------------------------------------------------------- per-CTA context
struct Ctx {
    uint8_t* sm;           // 1024-aligned shared memory
    uint64_t* bar;         // mbarriers
    uint32_t tmem;         // TMEM base
    int h, u;              // head, unit
    SegEntry sg;           // the unit's segment
    int64_t nc;            // chunks of the segment
};

// ---------------------------------------------------------------- prep (warps 0-7)
__device__ __forceinline__ void unpack_bf16x8(const uint4 raw, float (&f)[8]) {
    const uint32_t u[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(u[i] << 16);
        f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
}
// 8 products a[i] * b[i], bf16, as one 16-byte shared store
// Element-wise r = a * b and r = a * b + c over 8 fp32 values, two per packed f32x2
// instruction: each element is rounded exactly as the scalar operation rounds it.
__device__ __forceinline__ void mul8(float (&r)[8], const float (&a)[8], const float (&b)[8]) {
#pragma unroll
    for (int p = 0; p < 8; p += 2) mul2(r[p], r[p + 1], a[p], a[p + 1], b[p], b[p + 1]);
}
__device__ __forceinline__ void fma8(float (&r)[8], const float (&a)[8], float b, const float (&c)[8]) {
#pragma unroll
    for (int p = 0; p < 8; p += 2)
        asm("{\n .reg .b64 x, y, z, w;\n mov.b64 x, {%2, %3};\n mov.b64 y, {%4, %4};\n"
            " mov.b64 z, {%5, %6};\n fma.rn.f32x2 w, x, y, z;\n mov.b64 {%0, %1}, w;\n}"
            : "=f"(r[p]), "=f"(r[p + 1])
            : "f"(a[p]), "f"(a[p + 1]), "f"(b), "f"(c[p]), "f"(c[p + 1]));
}
__device__ __forceinline__ void st_prod8(uint32_t addr, const float (&a)[8], const float (&b)[8]) {
    float r[8];
    mul8(r, a, b);
    st_shared_v4(addr, pack_bf16(r[0], r[1]), pack_bf16(r[2], r[3]), pack_bf16(r[4], r[5]),
                 pack_bf16(r[6], r[7]));
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// The copy thread's TMA issues for chunk index cc (tokens t0 = t_begin + 64 cc of head h):
// its log alpha tile into LA, its k (and q) tiles into its slot's K_dec (and Q~)
// pieces, its v tile into its slot's W piece, each on its own mbarrier; and the L2
// prefetch of a later chunk's tiles.
template <int MODE>
__device__ __forceinline__ void tma_la(uint8_t* sm, uint64_t* bar, const TcMaps& maps, int h, int t0) {
    using L = Lay<MODE>;
    mbar_expect_tx(bar + B_LA, maps.beta_tma ? 32768 + 1024 : 32768);
    tma_tile(sm + L::LA, &maps.la, 0, h, t0, bar + B_LA);
    if (maps.beta_tma)  // beta of the four heads 4 (h / 4) .. + 3 for the chunk's tokens
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(sm + L::BTILE)),
            "l"(reinterpret_cast<uint64_t>(&maps.beta)), "r"(h & ~3), "r"(t0), "r"(smem_u32(bar + B_LA))
            : "memory");
}
template <int MODE>
__device__ __forceinline__ void tma_kq(uint8_t* slot, uint64_t* bar, const TcMaps& maps, int h, int t0) {
    using L = Lay<MODE>;
    mbar_expect_tx(bar + B_KQ, L::Q ? 32768 : 16384);
    tma_tile(slot + L::S_KD, &maps.k, 0, h, t0, bar + B_KQ);
    if (L::Q) tma_tile(slot + L::S_QT, &maps.q, 0, h, t0, bar + B_KQ);
}
// v tile of the chunk at t0 into the slot's W piece (offset 0); vbar = the slot's B_V barrier
__device__ __forceinline__ void tma_v(uint8_t* slot, uint64_t* vbar, const TcMaps& maps, int h, int t0) {
    mbar_expect_tx(vbar, 16384);
    tma_tile(slot, &maps.v, 0, h, t0, vbar);
    tma_tile(slot + 8192, &maps.v, 64, h, t0, vbar);
}
// mbarrier of slot s's v tile
__device__ __forceinline__ uint64_t* v_bar(uint64_t* bar, int s) { return bar + (s ? B_V1 : B_V); }
template <bool Q>
__device__ __forceinline__ void prefetch_chunk(const TcMaps& maps, int h, int t0) {
    tma_prefetch(&maps.la, 0, h, t0);
    tma_prefetch(&maps.k, 0, h, t0);
    if (Q) tma_prefetch(&maps.q, 0, h, t0);
    tma_prefetch(&maps.v, 0, h, t0);
    tma_prefetch(&maps.v, 64, h, t0);
}

// Prep warps: for every chunk of the unit, in order, the chunk-local work into the
// chunk's ring slot (and W, U' into their TMEM accumulators; the chain stages W into the
// slot).  Thread mapping for the
// elementwise phases: warp w, lane l = 16 hl + cg holds tokens 8w + 4hl + i (i < 4)
// and channels 8cg .. 8cg + 7.
template <int MODE>
__device__ void prep_loop(const Ctx& x, const TcArgs& a, const TcMaps& maps, int tid) {
    using L = Lay<MODE>;
    constexpr bool Q = L::Q;
    uint8_t* sm = x.sm;
    uint64_t* bar = x.bar;
    const int w = tid >> 5, lane = tid & 31, h = x.h, H = a.H;
    const int hl = lane >> 4, cg = lane & 15, c0 = 8 * cg;
    const uint32_t gsw = (uint32_t)(cg >> 2) & 1u;  // bank spread of the lane's 32-byte reads
    const bool half_b = w >= 4;  // this warp's tokens lie in the chunk's second half
    const uint32_t tq = x.tmem + ((uint32_t)((w & 3) * 32) << 16);
    float* beta_s = reinterpret_cast<float*>(sm + L::BETA);
    const int64_t tb = x.sg.t_begin, te = x.sg.t_end;
    // Shared addresses of this thread's 16-byte piece of each operand image row: every
    // image stores row r = 8w + 4hl + i, channels c0..c0+7 at base + (r & 7) 128 +
    // (((c0 / 8) % 8) ^ (r & 7)) 16 (128-byte swizzle); the bases differ by the image's
    // row count (K-major R rows, or MN-major with K = 64 token rows).
    const uint32_t blk = (uint32_t)w * 1024u;
    const uint32_t a_x1 = smem_u32(sm + L::X1) + (uint32_t)(cg >> 3) * 16384u + blk;
    const uint32_t a_bt = smem_u32(sm + L::BT) + (uint32_t)(cg >> 3) * 12288u + blk;
    const uint32_t a_kg = smem_u32(sm + L::KG) + (uint32_t)(cg >> 3) * 8192u + blk;
    const uint32_t a_r64 = (uint32_t)(cg >> 3) * 8192u + blk;  // slot images, 64 rows
    // this thread's row of the raw [64][128] tiles: token 8w + 4hl + i, channels c0..
    const uint32_t raw_row0 = (uint32_t)(8 * w + 4 * hl) * 128u + (uint32_t)c0;

    // pass 1 with the chunk cache: chunk c's entry (the copy thread bulk-stores TB and the
    // slot's images but W after the barrier that follows the inversion, and W, which the
    // chain writes into the slot, one chunk later)
    constexpr bool CACHE = MODE == TRANS_CACHE;
    auto cache_entry = [&](int64_t cc) {
        return a.cache + ((x.sg.c_base + cc) * H + h) * (int64_t)kCacheEntryBytes;
    };
    // Thread 0 issues the [A;P] product; the copy thread TCOPY (lane 0 of warp
    // 4, whose share of the inversion is the shortest) issues every TMA load and bulk
    // store, so that no warp with a full share of a phase also carries the copies.
    // Each keeps what it has in flight, for the waits after a timeout.
    bool ap_out = false, v_out[2] = {false, false}, la_out = false, kq_out = false;
    uint32_t ap_par = 0, v_par[2] = {0, 0}, la_par = 0, kq_par = 0;
    // In the transition modes chunk c+1's v tile goes into its slot together with its k
    // tile (the slot's W piece is free once its k piece is); the forward and dump chains
    // put chunk c-2's output tile there, so chunk c's v waits for it in chunk c.
    constexpr bool V_AHEAD = MODE == TRANS || MODE == TRANS_CACHE;
    if (x.nc > 0 && tid == TCOPY) {  // chunk 0's tiles (slot 0 is free)
        tma_la<MODE>(sm, bar, maps, h, (int)tb);
        tma_kq<MODE>(sm, bar, maps, h, (int)tb);
        tma_v(sm, v_bar(bar, 0), maps, h, (int)tb);
        la_out = kq_out = v_out[0] = true;
        if (x.nc > 1) prefetch_chunk<Q>(maps, h, (int)(tb + C));
        if (x.nc > 2) prefetch_chunk<Q>(maps, h, (int)(tb + 2 * C));
    }
    // beta of token tid of the next chunk (threads 0-63): from the tile that arrives with
    // the log alpha tile, or (heads not a multiple of 4) loaded a chunk ahead
    float beta_next = (!maps.beta_tma && tid < C && tb + tid < te) ? ld_nc_f1(a.beta + (tb + tid) * H + h) : 0.f;
    bool ok = true;
    for (int64_t c = 0; c < x.nc; ++c) {
        const int64_t t0 = tb + c * C;
        const int Lc = (int)((te - t0) < C ? (te - t0) : C);
        const int s = (int)(c & 1);
        const uint32_t use = (uint32_t)((c >> 1) & 1);  // phase of this slot use
        uint8_t* slot = sm + s * L::SLOT;
        float* gsum = reinterpret_cast<float*>(Q ? slot + L::S_PB : sm + L::GSUM);
        if (tid == 0) TRACE(0, c, 0);

        // ============ raw tiles of this chunk -> registers; gates
        float g[4][8];
        uint4 kr[4], qr[4];
        {
            const bool lok = wait_bar(bar + B_LA, (uint32_t)(c & 1)) &&
                             wait_bar(bar + B_KQ, (uint32_t)(c & 1));
            if (lok && tid == 0) TRACE(0, c, 14);
            if (lok && tid == TCOPY) {
                la_out = kq_out = false;
                // the previous chunk's TB store (all but the latest bulk group) has read
                // X1/BT before this chunk's images go there (after the gate barrier)
                if (CACHE) bulk_wait_read1();
            }
            const float* la_t = reinterpret_cast<const float*>(sm + L::LA);
            const uint32_t kt = smem_u32(slot + L::S_KD), qt = smem_u32(slot + L::S_QT);
            float acc[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const bool live = 8 * w + 4 * hl + i < Lc;  // rows past the segment end:
                const uint32_t ro = raw_row0 + (uint32_t)i * 128u;  // identity steps
                // the two 16-byte halves of the lane's 32 bytes in an order that puts
                // lanes 4-7 of each quarter on the banks lanes 0-3 leave free
                const float4 la0 = *reinterpret_cast<const float4*>(la_t + ro + 4u * gsw);
                const float4 la1 = *reinterpret_cast<const float4*>(la_t + ro + 4u * (gsw ^ 1u));
                float4 l0 = gsw ? la1 : la0, l1 = gsw ? la0 : la1;
                kr[i] = ld_shared_v4(kt + 2u * ro);
                if (Q) qr[i] = ld_shared_v4(qt + 2u * ro);
                if (!live) {
                    l0 = l1 = make_float4(0.f, 0.f, 0.f, 0.f);
                    kr[i] = make_uint4(0u, 0u, 0u, 0u);
                    if (Q) qr[i] = make_uint4(0u, 0u, 0u, 0u);
                }
                const float cl[8] = {clamp_gate(l0.x), clamp_gate(l0.y), clamp_gate(l0.z), clamp_gate(l0.w),
                                     clamp_gate(l1.x), clamp_gate(l1.y), clamp_gate(l1.z), clamp_gate(l1.w)};
                add8(acc, acc, cl);
#pragma unroll
                for (int j = 0; j < 8; ++j) g[i][j] = acc[j];
            }
            // the second half-warp's tokens follow the first's: add the partner's total
            float pt[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) pt[j] = __shfl_xor_sync(0xffffffffu, acc[j], 16);
            if (hl) {
                add8(acc, acc, pt);
#pragma unroll
                for (int i = 0; i < 4; ++i) add8(g[i], g[i], pt);
            }
            if (hl) {  // the warp's 8-token sums
                *reinterpret_cast<float4*>(gsum + w * D + c0 + 4u * gsw) =
                    make_float4(acc[0], acc[1], acc[2], acc[3]);
                *reinterpret_cast<float4*>(gsum + w * D + c0 + 4u * (gsw ^ 1u)) =
                    make_float4(acc[4], acc[5], acc[6], acc[7]);
            }
            if (tid < C)
                beta_s[tid] = maps.beta_tma ? (tid < Lc ? reinterpret_cast<const float*>(sm + L::BTILE)[4 * tid + (h & 3)] : 0.f)
                                            : beta_next;
            // every raw tile has been read: LA may take the next chunk's log alpha
            if (bar_named_or(BAR_PREP, NPREP, !lok)) {
                ok = false;
                break;
            }
        }
        // copy thread: the next chunk's k (and q, and in the transition modes v) tiles go
        // into the next slot as soon as the chain's products of chunk c-1 (and its cache
        // stores) have read it; in the forward and dump modes this chunk's v tile goes
        // into this slot's W piece as soon as chunk c-2's output tile has left it; polled
        // at a few points of the chunk, waited for at the last one
        bool kq_next = c + 1 >= x.nc, v_this = c == 0 || V_AHEAD;
        uint8_t* nslot = sm + (s ^ 1) * L::SLOT;
        const uint32_t nuse = (uint32_t)(((c + 1) >> 1) & 1);
        auto poll_tma = [&](bool block_kq, bool block_v) -> bool {
            if (!kq_next && (block_kq ? wait_bar(bar + B_EMPTY + (s ^ 1), nuse ^ 1u)
                                      : mbar_try_wait(bar + B_EMPTY + (s ^ 1), nuse ^ 1u))) {
                if (CACHE) bulk_wait_read();  // chunk c-1's cache stores have read that slot
                tma_kq<MODE>(nslot, bar, maps, h, (int)(t0 + C));
                TRACE(0, c + 1, 13);
                kq_next = kq_out = true;
                kq_par = (uint32_t)((c + 1) & 1);
                if (V_AHEAD) {
                    tma_v(nslot, v_bar(bar, s ^ 1), maps, h, (int)(t0 + C));
                    v_out[s ^ 1] = true;
                    v_par[s ^ 1] = nuse;
                }
            }
            // (only the forward chain puts output tiles into the W piece; the dump chain
            // arrives on B_WFREE anyway)
            if (!v_this && (block_v ? wait_bar(bar + B_WFREE + s, use ^ 1u)
                                    : mbar_try_wait(bar + B_WFREE + s, use ^ 1u))) {
                tma_v(slot, v_bar(bar, s), maps, h, (int)t0);
                v_this = v_out[s] = true;
                v_par[s] = use;
            }
            return kq_next && v_this;
        };
        if (tid == 0) TRACE(0, c, 1);
        // Per-channel references, once per channel by threads 0-127 (channel tid): the
        // offsets of the eight 8-token groups (exclusive prefix of the warps' sums), rho_a
        // = g_15 (end of group 1), rho_b = g_47 (end of group 5), g_last = g_63, and the
        // factors eR = e^{rho}, dRb = e^{g_last - rho_b}, sh = e^{(rho_b - rho_a) / 2}
        // (>= e^-80 since rho_b - rho_a >= -160) and gamma = e^{g_last}.  Rows of fac
        // ([14][128], over the sums' rows 0-7, same column order; each thread reads its
        // column before writing it): 0-7 offsets, 8/9 -rho_a/-rho_b (log2 units), 10/11
        // e^rho_a / e^rho_b, 12 dRb, 13 sh.
        float* fac = gsum;
        if (tid < D) {
            const int cgt = tid >> 3, jt = tid & 7;
            const int p = 8 * cgt + 4 * (((jt >> 2) ^ (cgt >> 2)) & 1) + (jt & 3);  // swizzled column
            float gs[8];
#pragma unroll
            for (int ww = 0; ww < 8; ++ww) gs[ww] = gsum[ww * D + p];
            float run = 0.f, ra = 0.f, rb = 0.f;
#pragma unroll
            for (int ww = 0; ww < 8; ++ww) {
                fac[ww * D + p] = run;
                run += gs[ww];
                if (ww == 1) ra = run;
                if (ww == 5) rb = run;
            }
            fac[8 * D + p] = -(ra * LOG2E);
            fac[9 * D + p] = -(rb * LOG2E);
            fac[10 * D + p] = ex2(ra * LOG2E);
            fac[11 * D + p] = ex2(rb * LOG2E);
            fac[12 * D + p] = ex2((run - rb) * LOG2E);
            fac[13 * D + p] = ex2((rb - ra) * (0.5f * LOG2E));
            reinterpret_cast<float*>(slot + L::S_GAM)[tid] = ex2(run * LOG2E);
        }
        // thread 0: the previous chunk's W and U' products, which read KG and TB, are done
        // before this chunk's images (after this barrier) overwrite them
        const bool wu_ok = tid != 0 || c == 0 || wait_bar(bar + B_WU, (uint32_t)((c - 1) & 1));
        if (bar_named_or(BAR_PREP, NPREP, !wu_ok)) {
            ok = false;
            break;
        }
        float nrho[8], sh[8], eR[8], dRb[8];
        {
            auto row8 = [&](int row, float (&o)[8]) {  // channels c0..c0+7 of a fac row
                const float4 u0 = *reinterpret_cast<const float4*>(fac + row * D + c0 + 4u * gsw);
                const float4 u1 = *reinterpret_cast<const float4*>(fac + row * D + c0 + 4u * (gsw ^ 1u));
                o[0] = u0.x, o[1] = u0.y, o[2] = u0.z, o[3] = u0.w;
                o[4] = u1.x, o[5] = u1.y, o[6] = u1.z, o[7] = u1.w;
            };
            float off[8];
            row8(w, off);
            row8(8 + (half_b ? 1 : 0), nrho);
            row8(10 + (half_b ? 1 : 0), eR);
            row8(12, dRb);
            row8(13, sh);
#pragma unroll
            for (int i = 0; i < 4; ++i) add8(g[i], g[i], off);  // inclusive cumsum over the chunk
        }

        // ============ operand images (one factor at a time, to keep registers few)
        {
            const uint32_t a_slot = smem_u32(slot) + a_r64;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int rr = 4 * hl + i;  // row within the warp's 8-row swizzle atom
                const uint32_t ro = (uint32_t)rr * 128u + ((uint32_t)((cg & 7) ^ rr) << 4);
                float kf[8], f[8], p[8], t[8];
                unpack_bf16x8(kr[i], kf);
                fma8(t, g[i], LOG2E, nrho);  // (g - rho_h) log2 e
#pragma unroll
                for (int j = 0; j < 8; ++j) f[j] = ex2(t[j]);  // e^{g-rho_h}
                st_prod8(a_x1 + ro, kf, f);
                if (Q) {
                    unpack_bf16x8(qr[i], p);
                    st_prod8(a_x1 + 8192u + ro, p, f);
                }
                mul8(f, f, eR);  // e^{g}
                st_prod8(a_kg + ro, kf, f);
                if (Q) st_prod8(a_slot + L::S_QT + ro, p, f);
#pragma unroll
                for (int j = 0; j < 8; ++j) f[j] = ex2(-t[j]);  // e^{rho_h-g}
                st_prod8(a_bt + ro, kf, f);
                if (!half_b) {
                    // e^{rho_b - g} for the first half's keys (cross-half block) as
                    // (e^{rho_a - g} sh) sh: an intermediate below the normal range means a
                    // true value below it, so flushing to zero is the right limit
                    mul8(f, f, sh);
                    mul8(f, f, sh);
                    st_prod8(a_bt + 8192u + ro, kf, f);
                }
                mul8(f, f, dRb);  // e^{g_last - g}
                st_prod8(a_slot + L::S_KD + ro, kf, f);
            }
        }
        fence_async_smem();
        tc_fence_before();
        // thread 0: the chain has taken the previous chunk's W^T out of the TMEM columns
        // the [A;P] product is about to overwrite
        const bool wr_ok = tid != 0 || c == 0 || wait_bar(bar + B_WREAD, (uint32_t)((c - 1) & 1));
        if (bar_named_or(BAR_PREP, NPREP, !wr_ok)) {
            ok = false;
            break;
        }
        if (tid == 0) TRACE(0, c, 2);

        // ============ [A;P] = X1 . BT^T   (M=128, N=96, K=128)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t x1 = smem_u32(sm + L::X1), bt = smem_u32(sm + L::BT);
            constexpr uint32_t id = idesc_bf16(128, 96, false, false);
#pragma unroll
            for (int st = 0; st < 8; ++st)
                mma_bf16(x.tmem + TM_AP, kmajor_desc(x1, 128, st), kmajor_desc(bt, 96, st), id, st > 0);
            mma_commit(bar + B_AP);
            ap_out = true;
            ap_par = (uint32_t)(c & 1);
        }
        // the next chunk's beta (without the tile): its load has until the proxy fence after
        // the inversion
        if (!maps.beta_tma && tid < C) beta_next = (t0 + C + tid < te) ? ld_nc_f1(a.beta + (t0 + C + tid) * H + h) : 0.f;
        {
            const bool aok = wait_bar(bar + B_AP, (uint32_t)(c & 1));
            if (aok && tid == 0) ap_out = false;
            if (bar_named_or(BAR_PREP, NPREP, !aok)) {
                ok = false;
                break;
            }
            tc_fence_after();
        }
        if (tid == 0) TRACE(0, c, 3);

        // ============ A -> (I + A)^-1 -> TB; P into the slot beside the inversion
        {
            float* As = reinterpret_cast<float*>(sm + L::AS);
            float* Ts = reinterpret_cast<float*>(sm + L::TS);
            float* Ys = reinterpret_cast<float*>(sm + L::YS);
            invert_to_tb(As, Ts, Ys, beta_s, smem_u32(sm + L::TB), tid, tq, [&](int ww) {
                if (Q && (ww & 3) >= 2) {  // warps 2, 3: columns 0-31; 6, 7: 32-63
                    const int j0 = 32 * (ww >> 2), r = (ww & 3) * 32 + lane - 64;
                    extract_p16(tq, r, j0, smem_u32(slot + L::S_PB));
                    extract_p16(tq, r, j0 + 16, smem_u32(slot + L::S_PB));
                }
                if (tid == TCOPY) {  // the next chunk's copies while warps 0-1 invert
                    // the previous chunk's W image, written by the chain, into its cache entry
                    // (before the next k/q/v copies, which wait for it to be read, reuse the slot)
                    if (CACHE && c > 0 && wait_bar(bar + B_WREAD, (uint32_t)((c - 1) & 1))) {
                        bulk_store_stream(cache_entry(c - 1) + CE_W, sm + (s ^ 1) * L::SLOT + L::S_W, 16384);
                        bulk_commit();
                    }
                    if (c + 1 < x.nc) {  // LA is free since the gate barrier
                        tma_la<MODE>(sm, bar, maps, h, (int)(t0 + C));
                        la_out = true;
                        la_par = (uint32_t)((c + 1) & 1);
                    }
                    // the chain usually frees the next slot during this phase: keep polling
                    // for it a bounded while (warps 0-1 have longer work before the next
                    // barrier), so that its tiles go out now rather than after the hand-off
                    const long long poll_end = clock64() + 1500;
                    do {
                        poll_tma(false, false);
                    } while (!kq_next && clock64() < poll_end);
                    if (c + 3 < x.nc) prefetch_chunk<Q>(maps, h, (int)(t0 + 3 * C));
                }
            }, c);
        }
        fence_async_smem();
        if (tid == 0) TRACE(0, c, 4);
        if (tid == TCOPY) poll_tma(false, true);  // v must be on its way before the hand-off
        tc_fence_before();
        bar_named(BAR_PREP, NPREP);
        // the slot is complete but for W: the chain issues the W and U' products (after the
        // v tile has landed) and stages W itself
        if (tid == 0) {
            mbar_arrive(bar + B_FULL + s);
            TRACE(0, c, 5);
        }
        if (tid == TCOPY) {
            if (CACHE) {  // the chunk's T diag(beta), complete since the barrier, into its entry,
                          // then the slot's images but W (the chain writes W after the hand-off)
                uint8_t* ce = cache_entry(c);
                bulk_store_stream(ce + CE_TB, sm + L::TB, 8192);
                bulk_commit();
                bulk_store_stream(ce + CE_KD, slot + L::S_KD, 16384);
                bulk_store_stream(ce + CE_QT, slot + L::S_QT, 16384);
                bulk_store_stream(ce + CE_PB, slot + L::S_PB, 8192);
                bulk_store_stream(ce + CE_GAM, slot + L::S_GAM, 512);
                bulk_commit();
            }
            poll_tma(true, true);  // the next chunk's k (and q, v) must be on their way
        }

    }
    if (CACHE && tid == TCOPY) {
        // the last chunk's W image, then every cache entry is written
        if (ok && x.nc > 0 && wait_bar(bar + B_WREAD, (uint32_t)((x.nc - 1) & 1))) {
            bulk_store_stream(cache_entry(x.nc - 1) + CE_W, sm + ((x.nc - 1) & 1) * L::SLOT + L::S_W, 16384);
            bulk_commit();
        }
        bulk_wait_all();
    }
    // after a timeout: bounded waits for what may still be in flight
    if (!ok && tid == 0 && ap_out) wait_bar(bar + B_AP, ap_par);
    if (!ok && tid == TCOPY) {
        for (int vs = 0; vs < 2; ++vs)
            if (v_out[vs]) wait_bar(v_bar(bar, vs), v_par[vs]);
        if (la_out) wait_bar(bar + B_LA, la_par);
        if (kq_out) wait_bar(bar + B_KQ, kq_par);
    }
}

// ---------------------------------------------------------------- chain: forward (warps 8-11)
// Chain warps, at the start of chunk c (its slot full): thread ct == 0 waits for the chunk's
// v tile and issues W^T = KG^T (T diag(beta))^T and U'^T = V^T (T diag(beta))^T (M=128,
// N=64, K=64) from the prep's KG and TB buffers and the v tile in the slot's W piece (the U
// columns are free: this chain read the previous chunk's U before it got here); then all
// wait for the two products and write W^T (TMEM, lane = channel) into the slot's W piece as
// the bf16 MN-major image (K rows = channels) that the chain's U product reads.  The
// caller's next named barrier makes the image visible to the chain's products; ct == 0 then
// arrives on B_WREAD.  last_bar / last_par: the commit ct == 0 issued, for the waits after a
// timeout.
template <int MODE>
__device__ bool chain_stage_w(const Ctx& x, uint8_t* slot, int64_t c, int ct, int& last_bar,
                              uint32_t& last_par) {
    using L = Lay<MODE>;
    if (ct == 0 && wait_bar(v_bar(x.bar, (int)(c & 1)), (uint32_t)((c >> 1) & 1))) {
        tc_fence_after();
        const uint32_t kg = smem_u32(x.sm + L::KG), tbb = smem_u32(x.sm + L::TB),
                       vv = smem_u32(slot + L::S_W);
        constexpr uint32_t id = idesc_bf16(128, 64, true, false);
#pragma unroll
        for (int st = 0; st < 4; ++st)
            mma_bf16(x.tmem + TM_W, mnmajor_desc(kg, 64, st), kmajor_desc(tbb, 64, st), id, st > 0);
#pragma unroll
        for (int st = 0; st < 4; ++st)
            mma_bf16(x.tmem + TM_U, mnmajor_desc(vv, 64, st), kmajor_desc(tbb, 64, st), id, st > 0);
        mma_commit(x.bar + B_WU);
        last_bar = B_WU;
        last_par = (uint32_t)(c & 1);
    }
    if (!wait_bar(x.bar + B_WU, (uint32_t)(c & 1))) return false;
    tc_fence_after();
    const int cw = ct >> 5, chn = (cw & 3) * 32 + (ct & 31), r0 = 32 * (cw >> 2);
    const uint32_t tq = x.tmem + ((uint32_t)((cw & 3) * 32) << 16);
    float v0[16], v1[16];
    tmem_ld16(tq + TM_W + r0, v0);
    tmem_ld16(tq + TM_W + r0 + 16, v1);
    tmem_wait16(v0);
    tmem_wait16(v1);
    const uint32_t wb = smem_u32(slot + L::S_W);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float* p = k < 2 ? v0 + 8 * k : v1 + 8 * (k - 2);
        st_shared_v4(wb + mnmajor_chunk_off(chn, (r0 >> 3) + k, 128), pack_bf16(p[0], p[1]),
                     pack_bf16(p[2], p[3]), pack_bf16(p[4], p[5]), pack_bf16(p[6], p[7]));
    }
    fence_async_smem();
    return true;
}

__device__ void chain_fwd(const Ctx& x, const TcArgs& a, const TcMaps& maps, int tid) {
    using L = Lay<FWD>;
    uint8_t* sm = x.sm;
    uint64_t* bar = x.bar;
    // chain warp cw (0-7): TMEM lane quadrant cw % 4, column half ch = cw / 4; e = row of
    // S^T (TMEM lane) of this thread
    const int ct = tid - NPREP, cw = ct >> 5, ch = cw >> 2, e = (cw & 3) * 32 + (ct & 31);
    const uint32_t tmem = x.tmem, tq = tmem + ((uint32_t)((cw & 3) * 32) << 16);
    const int h = x.h, H = a.H;
    const SegEntry& sg = x.sg;
    const bool snap_on = a.snap_pool != nullptr;
    const bool gate_on = a.gate != nullptr;
    const int64_t seq_lo = snap_on ? (a.cu ? (int64_t)a.cu[sg.n] : (int64_t)sg.n * a.T) : 0;

    // initial state S^T
    {
        const float* s0 = nullptr;
        const float* sin = nullptr;
        if (sg.j == 0 && sg.last)  // single segment: the caller's state
            s0 = a.s0 ? a.s0 + ((int64_t)sg.n * H + h) * D * D : nullptr;
        else
            sin = a.sin + ((int64_t)x.u * H + h) * D * D + (int64_t)e * D;
        for (int cc = 64 * ch; cc < 64 * ch + 64; cc += 16) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                v[i] = sin ? sin[cc + i] : (s0 ? s0[(int64_t)(cc + i) * D + e] : 0.f);
            tmem_st16(tq + TM_S + cc, v);
        }
        tmem_st_wait();
        tc_fence_before();
        bar_named(BAR_CHAIN, NCHAIN);
    }

    bool ok = true;
    bool s_waited = true;  // the last state update has been waited for
    // thread ct == 0: the last commit issued (products complete in issue order, so it
    // covers all of them) and the output-gate tile in flight, for the waits after a timeout
    int last_bar = -1;
    uint32_t last_par = 0;
    bool gate_out = false;
    uint32_t gate_par = 0;
    // O^T of chunk cc (in O buffer cc & 1) -> out: a full chunk as one [64][128] bf16 tile in
    // its slot's W area by TMA, a partial one row by row; with an output gate, each element
    // gated first (the gate tile was loaded into the W area).  Returns false if a wait gave up.
    auto epilogue = [&](int64_t cc) -> bool {
        const int s = (int)(cc & 1);
        const int64_t t0 = sg.t_begin + cc * C;
        const int Lc = (int)((sg.t_end - t0) < C ? (sg.t_end - t0) : C);
        bool wok = wait_bar(bar + B_O + s, (uint32_t)((cc >> 1) & 1));
        if (gate_on) wok = wok && wait_bar(bar + B_GATE, (uint32_t)(cc & 1));
        if (bar_named_or(BAR_CHAIN, NCHAIN, !wok)) return false;
        if (ct == 0 && gate_on) gate_out = false;
        if (ct == 0) TRACE(1, cc + 1, 7);
        tc_fence_after();
        // this thread: tokens r0 .. r0+31 of column e of O^T
        const int r0 = 32 * ch;
        float v[2][16];
#pragma unroll
        for (int b = 0; b < 2; ++b) tmem_ld16(tq + TM_O + 64 * s + r0 + 16 * b, v[b]);
#pragma unroll
        for (int b = 0; b < 2; ++b) tmem_wait16(v[b]);
        if (ct == 0) TRACE(1, cc + 1, 8);
        uint8_t* os = sm + s * L::SLOT + L::S_W;  // [64][128] bf16 tile (row = token)
        const uint32_t oa = smem_u32(os) + 2u * (uint32_t)e + (uint32_t)r0 * 256u;
        if (gate_on) {
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    uint16_t gb;
                    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(gb) : "r"(oa + (uint32_t)(16 * b + i) * 256u));
                    v[b][i] *= __uint_as_float((uint32_t)gb << 16);
                }
        }
        if (Lc == C) {
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const uint16_t ob = __bfloat16_as_ushort(__float2bfloat16_rn(v[b][i]));
                    asm volatile("st.shared.u16 [%0], %1;" ::"r"(oa + (uint32_t)(16 * b + i) * 256u), "h"(ob)
                                 : "memory");
                }
            if (ct == 0) TRACE(1, cc + 1, 9);
            fence_async_smem();
            bar_named(BAR_CHAIN, NCHAIN);
            if (ct == 32) {
                tma_store_tile(&maps.out, os, h, (int)t0);
                bulk_commit();
                bulk_wait_read();
                mbar_arrive(bar + B_WFREE + s);
            }
        } else {
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + (int64_t)h * D + e;
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (r0 + 16 * b + i < Lc)
                        out[(t0 + r0 + 16 * b + i) * H * (int64_t)D] = __float2bfloat16_rn(v[b][i]);
            bar_named(BAR_CHAIN, NCHAIN);
            if (ct == 32) mbar_arrive(bar + B_WFREE + s);
        }
        return true;
    };

    for (int64_t c = 0; c < x.nc; ++c) {
        const int s = (int)(c & 1);
        uint8_t* slot = sm + s * L::SLOT;
        const int64_t t0 = sg.t_begin + c * C;
        if (ct == 0) TRACE(1, c, 0);
        bool wok = wait_bar(bar + B_FULL + s, (uint32_t)((c >> 1) & 1));
        if (!s_waited) wok = wok && wait_bar(bar + B_S, (uint32_t)((c - 1) & 1));
        s_waited = true;
        tc_fence_after();
        if (ct == 0) TRACE(1, c, 1);
        wok = wok && chain_stage_w<FWD>(x, slot, c, ct, last_bar, last_par);
        if (wok) {  // bf16 S^T -> SB; S^T *= gamma (per column = key channel) in place
            const float* gam = reinterpret_cast<const float*>(slot + L::S_GAM);
            stage_cols_tmem<4>(tq + TM_S + 64 * ch, tq + TM_SB + 32 * ch, 64 * ch, gam, true);
            tmem_st_wait();
        }
        tc_fence_before();
        if (bar_named_or(BAR_CHAIN, NCHAIN, !wok)) {
            ok = false;
            break;
        }
        if (ct == 0) {
            TRACE(1, c, 2);
            mbar_arrive(bar + B_WREAD);
            tc_fence_after();
            const uint32_t wb = smem_u32(slot + L::S_W), qt = smem_u32(slot + L::S_QT);
            constexpr uint32_t id_neg = idesc_bf16(128, 64, false, true, true);
            constexpr uint32_t id = idesc_bf16(128, 64, false, false);
            // U^T -= S^T W^T   (U holds U'^T from the prep)
#pragma unroll
            for (int st = 0; st < 8; ++st)
                mma_bf16_ts(tmem + TM_U, tmem + TM_SB + 8 * st, mnmajor_desc(wb, 128, st), id_neg, 1);
            mma_commit(bar + B_U);
            // O^T = S^T Q~^T
#pragma unroll
            for (int st = 0; st < 8; ++st)
                mma_bf16_ts(tmem + TM_O + 64 * s, tmem + TM_SB + 8 * st, kmajor_desc(qt, 64, st), id,
                            st > 0);
            last_bar = B_U;
            last_par = (uint32_t)(c & 1);
        }
        // meanwhile: the previous chunk's output
        if (c > 0 && !(ok = epilogue(c - 1))) break;
        if (ct == 0) TRACE(1, c, 3);
        wok = wait_bar(bar + B_U, (uint32_t)(c & 1));
        if (bar_named_or(BAR_CHAIN, NCHAIN, !wok)) {
            ok = false;
            break;
        }
        tc_fence_after();
        if (ct == 0) TRACE(1, c, 4);
        if (ct == 0) {
            // the W area is read: this chunk's output-gate tile goes there
            if (gate_on) {
                gate_out = true;
                gate_par = (uint32_t)(c & 1);
                mbar_expect_tx(bar + B_GATE, 16384);
                tma_tile(slot + L::S_W, &maps.gate, 0, h, (int)t0, bar + B_GATE);
            }
        }
        // bf16 U^T -> UB (this thread: tokens 32 ch .. 32 ch + 31)
        stage_cols_tmem<2>(tq + TM_U + 32 * ch, tq + TM_UB + 16 * ch, 32 * ch, nullptr, false);
        tmem_st_wait();
        tc_fence_before();
        bar_named(BAR_CHAIN, NCHAIN);
        if (ct == 0) {
            TRACE(1, c, 5);
            tc_fence_after();
            const uint32_t kd = smem_u32(slot + L::S_KD), pb = smem_u32(slot + L::S_PB);
            constexpr uint32_t id_s = idesc_bf16(128, 128, false, true);
            constexpr uint32_t id = idesc_bf16(128, 64, false, false);
            // S^T += U^T K_dec
#pragma unroll
            for (int st = 0; st < 4; ++st)
                mma_bf16_ts(tmem + TM_S, tmem + TM_UB + 8 * st, mnmajor_desc(kd, 64, st), id_s, 1);
            mma_commit(bar + B_S);
            // O^T += U^T P^T
#pragma unroll
            for (int st = 0; st < 4; ++st)
                mma_bf16_ts(tmem + TM_O + 64 * s, tmem + TM_UB + 8 * st, kmajor_desc(pb, 64, st), id, 1);
            mma_commit(bar + B_O + s);
            mma_commit(bar + B_EMPTY + s);
            last_bar = B_EMPTY + s;
            last_par = (uint32_t)((c >> 1) & 1);
            TRACE(1, c, 6);
        }
        s_waited = false;
        if (snap_on) {  // state snapshot at this chunk end, if one is requested
            const int Lc = (int)((sg.t_end - t0) < C ? (sg.t_end - t0) : C);
            const int64_t pos = t0 + Lc - seq_lo;
            if (pos % a.snap_interval == 0 && pos / a.snap_interval <= a.snap_max) {
                const int slot_id = a.snap_slots[(int64_t)sg.n * a.snap_max + pos / a.snap_interval - 1];
                wok = wait_bar(bar + B_S, (uint32_t)(c & 1));
                s_waited = true;
                if (bar_named_or(BAR_CHAIN, NCHAIN, !wok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (slot_id >= a.snap_num_slots) {
                    if (ct == 0) atomicCAS(&g_tc_status, 0, ERR_BAD_SLOT);
                } else if (slot_id >= 0) {
                    float* sp = a.snap_pool + ((int64_t)slot_id * H + h) * D * D;
                    for (int cc = 64 * ch; cc < 64 * ch + 64; cc += 16) {
                        float v[16];
                        tmem_ld16(tq + TM_S + cc, v);
                        tmem_wait16(v);
#pragma unroll
                        for (int i = 0; i < 16; ++i) sp[(int64_t)(cc + i) * D + e] = v[i];
                    }
                }
            }
        }
    }
    if (ok && x.nc > 0) ok = epilogue(x.nc - 1);
    if (ok && !s_waited) {
        const bool wok = wait_bar(bar + B_S, (uint32_t)((x.nc - 1) & 1));
        ok = !bar_named_or(BAR_CHAIN, NCHAIN, !wok);
    }
    if (!ok && ct == 0) {  // after a timeout: bounded waits for what may still be in flight
        if (last_bar >= 0) wait_bar(bar + last_bar, last_par);
        if (gate_out) wait_bar(bar + B_GATE, gate_par);
    }
    if (ct == 32) bulk_wait_all();  // output stores are complete
    tc_fence_after();
    if (ok && sg.last && a.s_final) {
        float* sf = a.s_final + ((int64_t)sg.n * H + h) * D * D;
        for (int cc = 64 * ch; cc < 64 * ch + 64; cc += 16) {
            float v[16];
            tmem_ld16(tq + TM_S + cc, v);
            tmem_wait16(v);
#pragma unroll
            for (int i = 0; i < 16; ++i) sf[(int64_t)(cc + i) * D + e] = v[i];
        }
    }
}

// ---------------------------------------------------------------- chain: transition (warps 8-11)
// B from 0 and M from I through the segment's chunks: per chunk the B step
// (U = U' - B W, B <- gamma B + K_dec^T U) and then the M step (U = -M W,
// M <- gamma M + K_dec^T U), sharing the U, SB and UB columns.
template <int MODE>
__device__ void chain_trans(const Ctx& x, const TcArgs& a, int tid) {
    using L = Lay<MODE>;
    uint8_t* sm = x.sm;
    uint64_t* bar = x.bar;
    const int ct = tid - NPREP, cw = ct >> 5, ch = cw >> 2, e = (cw & 3) * 32 + (ct & 31);
    const uint32_t tmem = x.tmem, tq = tmem + ((uint32_t)((cw & 3) * 32) << 16);
    const int h = x.h, H = a.H;
    // B^T = 0, M^T = I
    for (int cc = 64 * ch; cc < 64 * ch + 64; cc += 16) {
        float z[16], m[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            z[i] = 0.f;
            m[i] = cc + i == e ? 1.f : 0.f;
        }
        tmem_st16(tq + TT_B + cc, z);
        tmem_st16(tq + TT_M + cc, m);
    }
    tmem_st_wait();
    tc_fence_before();
    bar_named(BAR_CHAIN, NCHAIN);

    constexpr uint32_t id_neg = idesc_bf16(128, 64, false, true, true);
    constexpr uint32_t id_s = idesc_bf16(128, 128, false, true);
    bool ok = true;
    int last_bar = -1;  // thread ct == 0: the last commit issued (see chain_fwd)
    uint32_t last_par = 0;
    for (int64_t c = 0; c < x.nc; ++c) {
        const int s = (int)(c & 1);
        uint8_t* slot = sm + s * L::SLOT;
        const uint32_t wb = smem_u32(slot + L::S_W), kd = smem_u32(slot + L::S_KD);
        const float* gam = reinterpret_cast<const float*>(slot + L::S_GAM);
        if (ct == 0) TRACE(1, c, 0);
        bool wok = wait_bar(bar + B_FULL + s, (uint32_t)((c >> 1) & 1));
        if (c > 0) wok = wok && wait_bar(bar + B_S, (uint32_t)((c - 1) & 1));
        tc_fence_after();
        if (ct == 0) TRACE(1, c, 1);
        wok = wok && chain_stage_w<MODE>(x, slot, c, ct, last_bar, last_par);
        for (int step = 0; step < 2 && ok; ++step) {  // 0: B, 1: M
            const uint32_t tstate = step == 0 ? TT_B : TT_M;
            if (wok) {
                stage_cols_tmem<4>(tq + tstate + 64 * ch, tq + TT_SB + 32 * ch, 64 * ch, gam, true);
                tmem_st_wait();
            }
            tc_fence_before();
            if (bar_named_or(BAR_CHAIN, NCHAIN, !wok)) {
                ok = false;
                break;
            }
            if (ct == 0) {
                TRACE(1, c, 2 + 3 * step);
                if (step == 0) mbar_arrive(bar + B_WREAD);
                tc_fence_after();
                // B step: U^T -= B^T W^T on top of U'^T;  M step: U^T = -M^T W^T
#pragma unroll
                for (int st = 0; st < 8; ++st)
                    mma_bf16_ts(tmem + TM_U, tmem + TT_SB + 8 * st, mnmajor_desc(wb, 128, st), id_neg,
                                (step == 0 || st > 0) ? 1u : 0u);
                mma_commit(bar + B_U);
                last_bar = B_U;
                last_par = (uint32_t)step;
            }
            wok = wait_bar(bar + B_U, (uint32_t)step);
            if (bar_named_or(BAR_CHAIN, NCHAIN, !wok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (ct == 0) TRACE(1, c, 3 + 3 * step);
            stage_cols_tmem<2>(tq + TM_U + 32 * ch, tq + TT_UB + 16 * ch, 32 * ch, nullptr, false);
            tmem_st_wait();
            tc_fence_before();
            bar_named(BAR_CHAIN, NCHAIN);
            if (ct == 0) {
                TRACE(1, c, 4 + 3 * step);
                tc_fence_after();
                // state^T += U^T K_dec
#pragma unroll
                for (int st = 0; st < 4; ++st)
                    mma_bf16_ts(tmem + tstate, tmem + TT_UB + 8 * st, mnmajor_desc(kd, 64, st), id_s, 1);
                if (step == 1) {
                    mma_commit(bar + B_S);
                    mma_commit(bar + B_EMPTY + s);
                    last_bar = B_EMPTY + s;
                    last_par = (uint32_t)((c >> 1) & 1);
                }
            }
        }
        if (!ok) break;
    }
    if (ok && x.nc > 0) {
        const bool wok = wait_bar(bar + B_S, (uint32_t)((x.nc - 1) & 1));
        ok = !bar_named_or(BAR_CHAIN, NCHAIN, !wok);
    }
    if (!ok && ct == 0 && last_bar >= 0) wait_bar(bar + last_bar, last_par);
    tc_fence_after();
    if (ok) {  // B^T then M^T of the segment
        float* tp = a.trans + ((int64_t)x.u * H + h) * 2 * D * D + (int64_t)e * D;
        for (int half = 0; half < 2; ++half) {
            for (int cc = 64 * ch; cc < 64 * ch + 64; cc += 16) {
                float v[16];
                tmem_ld16(tq + (half ? TT_M : TT_B) + cc, v);
                tmem_wait16(v);
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4*>(tp + half * D * D + cc + i) =
                        make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            }
        }
    }
}

// ---------------------------------------------------------------- chain: operand dump (test aid)
__device__ void chain_dump(const Ctx& x, const TcArgs& a, int tid) {
    using L = Lay<DUMP>;
    uint8_t* sm = x.sm;
    uint64_t* bar = x.bar;
    const int ct = tid - NPREP, cw = ct >> 5, ch = cw >> 2, e = (cw & 3) * 32 + (ct & 31);
    const uint32_t tq = x.tmem + ((uint32_t)((cw & 3) * 32) << 16);
    const int h = x.h, H = a.H;
    int last_bar = -1;  // thread ct == 0: the last commit issued, for the wait after a timeout
    uint32_t last_par = 0;
    bool ok = true;
    for (int64_t c = 0; c < x.nc && ok; ++c) {
        const int s = (int)(c & 1);
        uint8_t* slot = sm + s * L::SLOT;
        bool wok = wait_bar(bar + B_FULL + s, (uint32_t)((c >> 1) & 1));
        wok = wok && chain_stage_w<DUMP>(x, slot, c, ct, last_bar, last_par);
        tc_fence_before();
        if (bar_named_or(BAR_CHAIN, NCHAIN, !wok)) {
            ok = false;
            break;
        }
        if (ct == 0) mbar_arrive(bar + B_WREAD);
        tc_fence_after();
        uint8_t* ent = a.dump + ((x.sg.c_base + c) * H + h) * (int64_t)kChunkImageBytes;
        auto copy = [&](uint32_t dst, uint32_t src, uint32_t bytes) {
            for (uint32_t o = 16u * ct; o < bytes; o += 16u * NCHAIN)
                *reinterpret_cast<uint4*>(ent + dst + o) = *reinterpret_cast<const uint4*>(slot + src + o);
        };
        copy(CI_W, L::S_W, 16384);
        copy(CI_KD, L::S_KD, 16384);
        copy(CI_QT, L::S_QT, 16384);
        copy(CI_PB, L::S_PB, 8192);
        copy(CI_GAM, L::S_GAM, 512);
        {  // U'^T (row e, tokens 32 ch ..) -> [128][64] bf16, 16-byte pieces XOR-swizzled by e & 7
            float v[2][16];
#pragma unroll
            for (int b = 0; b < 2; ++b) tmem_ld16(tq + TM_U + 32 * ch + 16 * b, v[b]);
#pragma unroll
            for (int b = 0; b < 2; ++b) tmem_wait16(v[b]);
#pragma unroll
            for (int pp = 0; pp < 4; ++pp) {
                const int p = 4 * ch + pp;
                const float* q = v[pp >> 1] + 8 * (pp & 1);
                uint4 pk;
                pk.x = pack_bf16(q[0], q[1]);
                pk.y = pack_bf16(q[2], q[3]);
                pk.z = pack_bf16(q[4], q[5]);
                pk.w = pack_bf16(q[6], q[7]);
                *reinterpret_cast<uint4*>(ent + CI_U + e * 128 + ((p ^ (e & 7)) << 4)) = pk;
            }
        }
        tc_fence_before();
        bar_named(BAR_CHAIN, NCHAIN);
        if (ct == 0) {
            mbar_arrive(bar + B_EMPTY + s);
            mbar_arrive(bar + B_WFREE + s);
        }
    }
    if (!ok && ct == 0 && last_bar >= 0) wait_bar(bar + last_bar, last_par);
}

// ---------------------------------------------------------------- the kernel
template <int MODE>
__global__ void __launch_bounds__(NT, 1) chunk_kernel(TcArgs a, const __grid_constant__ TcMaps maps) {
    using L = Lay<MODE>;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, formed by pointer arithmetic on the shared array so that the
    // compiler keeps every access through it in the shared state space (no generic loads)
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int u = blockIdx.x, h = blockIdx.y;
    KDA_DCHECK(*a.n_units >= 0 && *a.n_units <= (int)gridDim.x);  // the table has gridDim.x entries
    if (u >= *a.n_units) return;
    const SegEntry sg = a.segs[u];
    KDA_DCHECK(seg_entry_ok(a, sg));
    // transitions only for segments with a successor, unless all are asked for
    if ((MODE == TRANS || MODE == TRANS_CACHE) && sg.last && !a.trans_all) return;
    const int64_t nc = sg.t_end > sg.t_begin ? (sg.t_end - sg.t_begin + C - 1) / C : 0;
    if ((MODE == DUMP || MODE == TRANS_CACHE) && (sg.c_base < 0 || sg.c_base + nc > a.total_chunks)) {
        if (tid == 0) atomicCAS(&g_tc_status, 0, ERR_SEG_OVERFLOW);  // malformed cu_seqlens
        return;
    }
    if ((MODE == TRANS || MODE == TRANS_CACHE) && tid == 0) {
        SPAN(0, globaltimer_ns());
        SPAN(2, smid_u32());
        SPAN(3, (unsigned long long)nc);
        SPAN(4, clock64());
    }
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::BAR);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sm + L::TMEMP);
    if (warp == 0) {
        tmem_alloc(tmem_ptr, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < NBARS; ++i) mbar_init(bar + i, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    Ctx x;
    x.sm = sm;
    x.bar = bar;
    x.tmem = *tmem_ptr;
    x.h = h;
    x.u = u;
    x.sg = sg;
    x.nc = nc;
    // Register split: the CTA is launched with 512 x 128 registers; the chain's two
    // warpgroups give 24 per thread to the prep's two (8 x 32 x (152 + 104) = 65536).
    if (tid < NPREP) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 152;" ::: "memory");
        prep_loop<MODE>(x, a, maps, tid);
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 104;" ::: "memory");
    }
    if (tid < NPREP) {
    } else if (MODE == FWD) {
        chain_fwd(x, a, maps, tid);
    } else if (MODE == TRANS || MODE == TRANS_CACHE) {
        chain_trans<MODE>(x, a, tid);
    } else {
        chain_dump(x, a, tid);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(x.tmem, 512);
    if ((MODE == TRANS || MODE == TRANS_CACHE) && tid == 0) {
        SPAN(1, globaltimer_ns());
        SPAN(5, clock64());
    }
}

// ---------------------------------------------------------------- pass 3 from the chunk cache
// Shared memory: two chunk images (the cache entry as pass 1 wrote it, 1024-byte
// aligned) with their v tiles, the output tile and the output gate's tile.
struct LayC {
    static constexpr uint32_t IMG_STRIDE = 66560;          // kCacheEntryBytes rounded to 1 KB
    static constexpr uint32_t V = 2 * IMG_STRIDE;          // [2] v tiles (two 64-channel boxes)
    static constexpr uint32_t OUT = V + 2 * 16384;         // bf16 [64][128]
    static constexpr uint32_t GATE = OUT + 16384;          // bf16 [64][128]
    static constexpr uint32_t BAR = GATE + 16384;          // mbarriers: MMA, image 0, image 1, gate
    static constexpr uint32_t TMEMP = BAR + 32;
    static constexpr uint32_t BYTES = TMEMP + 16 + 1024;   // + alignment slack
};
static_assert(LayC::IMG_STRIDE >= kCacheEntryBytes && LayC::IMG_STRIDE % 1024 == 0, "image stride");
static_assert(LayC::BYTES <= 232448, "shared memory");

// Per (segment, head): the state chain from the true incoming state and the output, every
// chunk's operands taken from the chunk cache (image and v tile loaded two chunks ahead):
//   bf16 S^T -> TMEM, S^T *= gamma                                      (all threads)
//   U^T = V^T TB^T ;  U^T -= S^T W^T ;  O^T = S^T Q~^T                 (one thread)
//   bf16 U^T -> TMEM                                                   (all threads)
//   O^T += U^T P^T ;  S^T += U^T K_dec                                 (one thread)
//   O^T (x gate) -> bf16 tile -> TMA store                             (all threads)
// Sixteen warps: lane quadrant warp % 4, column slice warp / 4.  The same products in
// the same precision as chunk_kernel<FWD>: the two differ only in where W, TB, Q~, K_dec,
// P and gamma come from.
__global__ void __launch_bounds__(NT, 1) cached_kernel(TcArgs a, const __grid_constant__ TcMaps maps) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int u = blockIdx.x, h = blockIdx.y, H = a.H;
    KDA_DCHECK(*a.n_units >= 0 && *a.n_units <= (int)gridDim.x);
    if (u >= *a.n_units) return;
    const SegEntry sg = a.segs[u];
    KDA_DCHECK(seg_entry_ok(a, sg));
    const bool snap_on = a.snap_pool != nullptr;
    const bool gate_on = a.gate != nullptr;
    const int64_t seq_lo = snap_on ? (a.cu ? (int64_t)a.cu[sg.n] : (int64_t)sg.n * a.T) : 0;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + LayC::BAR);  // MMA completion
    uint64_t* bar_img = bar + 1;                                  // [2] image and v loads
    uint64_t* bar_gate = bar + 3;                                 // output-gate tile
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sm + LayC::TMEMP);
    if (sg.c_base < 0 || sg.c_base + (sg.t_end - sg.t_begin + C - 1) / C > a.total_chunks) {
        if (tid == 0) atomicCAS(&g_tc_status, 0, ERR_SEG_OVERFLOW);  // malformed cu_seqlens
        return;
    }
    auto entry = [&](int64_t tt) {  // the chunk cache entry of the chunk at tt, head h
        return a.cache + ((sg.c_base + (tt - sg.t_begin) / C) * H + h) * (int64_t)kCacheEntryBytes;
    };
    uint32_t pending = 0;  // thread 0: bit b = a load into image b in flight; bit 2 = gate tile
    auto load_img = [&](int64_t tt, int b) {
        pending |= 1u << b;
        mbar_expect_tx(bar_img + b, (uint32_t)kCacheEntryBytes + 16384u);
        bulk_load(sm + b * LayC::IMG_STRIDE, entry(tt), (uint32_t)kCacheEntryBytes, bar_img + b);
        uint8_t* vb = sm + LayC::V + b * 16384;
        tma_tile(vb, &maps.v, 0, h, (int)tt, bar_img + b);
        tma_tile(vb + 8192, &maps.v, 64, h, (int)tt, bar_img + b);
    };
    auto load_gate = [&](int64_t tt) {
        pending |= 4u;
        mbar_expect_tx(bar_gate, 16384);
        tma_tile(sm + LayC::GATE, &maps.gate, 0, h, (int)tt, bar_gate);
    };

    if (warp == 0) {
        tmem_alloc(tmem_ptr, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar_img, 1);
        mbar_init(bar_img + 1, 1);
        mbar_init(bar_gate, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    const int quad = warp & 3, wg = warp >> 2, lrow = quad * 32 + lane;
    const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16);
    if (tid == 0 && sg.t_begin < sg.t_end) {  // the first two chunks' images
        load_img(sg.t_begin, 0);
        if (sg.t_begin + C < sg.t_end) load_img(sg.t_begin + C, 1);
        if (gate_on) load_gate(sg.t_begin);
    }
    // initial state: slice wg writes columns 32wg..32wg+31 of S^T
    {
        const int e = lrow, cb = 32 * wg;
        for (int c0 = cb; c0 < cb + 32; c0 += 16) {
            float v[16];
            if (sg.j == 0 && sg.last) {  // single segment: the caller's state
                const float* s0 = a.s0 ? a.s0 + ((int64_t)sg.n * H + h) * D * D : nullptr;
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = s0 ? s0[(int64_t)(c0 + i) * D + e] : 0.f;
            } else {
                const float* sin = a.sin + ((int64_t)u * H + h) * D * D + (int64_t)e * D;
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = sin[c0 + i];
            }
            tmem_st16(tq + TM_S + c0, v);
        }
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    uint32_t parity = 0, img_parity = 0, gate_parity = 0;  // img_parity: bit b for image b
    bool mma_out = false;  // thread 0: a commit not yet waited for, on phase mma_par
    uint32_t mma_par = 0;
    // O^T of the chunk at tt (Lcc tokens) from the O accumulator at tm_o -> out: a full chunk
    // as one [64][128] bf16 tile by TMA, a partial last chunk row by row from registers; with
    // an output gate, each element gated first (then the next chunk's gate tile is loaded).
    // Called by all threads; false if a wait gave up.
    auto emit = [&](int64_t tt, int Lcc, uint32_t tm_o) -> bool {
        const int r0 = 16 * wg;
        float v[16];
        tmem_ld16(tq + tm_o + r0, v);
        tmem_wait16(v);
        __nv_bfloat16* os = reinterpret_cast<__nv_bfloat16*>(sm + LayC::OUT);
        if (gate_on) {
            const __nv_bfloat16* gs = reinterpret_cast<const __nv_bfloat16*>(sm + LayC::GATE);
            if (__syncthreads_or(!mbar_wait(bar_gate, gate_parity, &g_tc_status, ERR_WAIT_TIMEOUT)))
                return false;
            gate_parity ^= 1u;
            pending &= ~4u;
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= __bfloat162float(gs[(r0 + i) * D + lrow]);
        }
        if (Lcc == C) {
#pragma unroll
            for (int i = 0; i < 16; ++i) os[(r0 + i) * D + lrow] = __float2bfloat16_rn(v[i]);
            fence_async_smem();
            __syncthreads();
            if (tid == 0) {
                tma_store_tile(&maps.out, sm + LayC::OUT, h, (int)tt);
                bulk_commit();
                if (gate_on && tt + C < sg.t_end) load_gate(tt + C);  // GATE has been read
            }
        } else {
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + (int64_t)h * D + lrow;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (r0 + i < Lcc) out[(tt + r0 + i) * H * (int64_t)D] = __float2bfloat16_rn(v[i]);
        }
        return true;
    };
    // block-wide bounded wait on the MMA barrier; false (uniformly) if any thread gave up
    auto wait_mma = [&]() -> bool {
        const bool okw = mbar_wait(bar, parity, &g_tc_status, ERR_WAIT_TIMEOUT);
        parity ^= 1u;
        tc_fence_after();
        return !__syncthreads_or(!okw);
    };
    bool ok = true;
    int b = 0;
    int64_t last_t0 = sg.t_begin;  // the chunk whose output is still in TMEM
    int last_Lc = 0;
    uint32_t last_o = TM_O;
    for (int64_t t0 = sg.t_begin; t0 < sg.t_end && ok; t0 += C, b ^= 1) {
        const int Lc = (int)((sg.t_end - t0) < C ? (sg.t_end - t0) : C);
        uint8_t* img = sm + b * LayC::IMG_STRIDE;
        // O accumulators alternate between chunks, so a chunk's output leaves TMEM while
        // the next chunk's first products run
        const uint32_t tm_o = TM_O + 64u * (uint32_t)(((t0 - sg.t_begin) / C) & 1);
        if (!(ok = !__syncthreads_or(!mbar_wait(bar_img + b, (img_parity >> b) & 1u, &g_tc_status,
                                                ERR_WAIT_TIMEOUT)))) break;
        img_parity ^= 1u << b;
        pending &= ~(1u << b);
        // bf16 S^T into TMEM (A operand), S^T *= gamma in place
        {
            const float* gam = reinterpret_cast<const float*>(img + CE_GAM);
            const int c0 = 32 * wg;
            stage_cols_tmem<2>(tq + TM_S + c0, tq + TM_SB + c0 / 2, c0, gam, true);
            tmem_st_wait();
        }
        tc_fence_before();
        __syncthreads();
        // U^T = V^T TB^T ;  U^T -= S^T W^T ;  O^T = S^T Q~^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t wb = smem_u32(img + CE_W), qt = smem_u32(img + CE_QT),
                           tb = smem_u32(img + CE_TB), vv = smem_u32(sm + LayC::V + b * 16384);
            constexpr uint32_t id_uv = idesc_bf16(128, 64, true, false);
            constexpr uint32_t id_neg = idesc_bf16(128, 64, false, true, true);
            constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int st = 0; st < 4; ++st)
                mma_bf16(tmem + TM_U, mnmajor_desc(vv, 64, st), kmajor_desc(tb, 64, st), id_uv, st > 0);
#pragma unroll
            for (int st = 0; st < 8; ++st)
                mma_bf16_ts(tmem + TM_U, tmem + TM_SB + 8 * st, mnmajor_desc(wb, 128, st), id_neg, 1);
#pragma unroll
            for (int st = 0; st < 8; ++st)
                mma_bf16_ts(tmem + tm_o, tmem + TM_SB + 8 * st, kmajor_desc(qt, 64, st), id, st > 0);
            mma_commit(bar);
            mma_out = true;
            mma_par = parity;
        }
        // meanwhile: the previous chunk's output (a full chunk: only a segment's last is partial)
        if (t0 > sg.t_begin && !(ok = emit(t0 - C, C, last_o))) break;
        if (!(ok = wait_mma())) break;
        mma_out = false;
        // bf16 U^T into TMEM; the last output store has left OUT by the next barrier
        {
            const int c0 = 16 * wg;
            stage_cols_tmem<1>(tq + TM_U + c0, tq + TM_UB + c0 / 2, c0, nullptr, false);
            tmem_st_wait();
        }
        if (tid == 0) bulk_wait_read();
        tc_fence_before();
        __syncthreads();
        // O^T += U^T P^T ; S^T += U^T K_dec
        if (tid == 0) {
            tc_fence_after();
            const uint32_t pb = smem_u32(img + CE_PB), kd = smem_u32(img + CE_KD);
            constexpr uint32_t id = idesc_bf16(128, 64, false, false);
            constexpr uint32_t id_s = idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int st = 0; st < 4; ++st)
                mma_bf16_ts(tmem + tm_o, tmem + TM_UB + 8 * st, kmajor_desc(pb, 64, st), id, 1);
#pragma unroll
            for (int st = 0; st < 4; ++st)
                mma_bf16_ts(tmem + TM_S, tmem + TM_UB + 8 * st, mnmajor_desc(kd, 64, st), id_s, 1);
            mma_commit(bar);
            mma_out = true;
            mma_par = parity;
        }
        if (!(ok = wait_mma())) break;
        mma_out = false;
        // this image (and v tile) is consumed: the chunk after next may load into it
        if (tid == 0 && t0 + 2 * C < sg.t_end) load_img(t0 + 2 * C, b);
        last_t0 = t0;
        last_Lc = Lc;
        last_o = tm_o;
        if (snap_on) {  // state snapshot at this chunk end, if one is requested
            const int64_t pos = t0 + Lc - seq_lo;
            if (pos % a.snap_interval == 0 && pos / a.snap_interval <= a.snap_max) {
                const int slot = a.snap_slots[(int64_t)sg.n * a.snap_max + pos / a.snap_interval - 1];
                if (slot >= a.snap_num_slots) {
                    if (tid == 0) atomicCAS(&g_tc_status, 0, ERR_BAD_SLOT);
                } else if (slot >= 0) {  // slice wg: columns 32wg..32wg+31 of S^T
                    float* sp = a.snap_pool + ((int64_t)slot * H + h) * D * D;
                    for (int c0 = 32 * wg; c0 < 32 * wg + 32; c0 += 16) {
                        float v[16];
                        tmem_ld16(tq + TM_S + c0, v);
                        tmem_wait16(v);
#pragma unroll
                        for (int i = 0; i < 16; ++i) sp[(int64_t)(c0 + i) * D + lrow] = v[i];
                    }
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (ok && last_Lc > 0) ok = emit(last_t0, last_Lc, last_o);  // the last chunk's output
    if (!ok && tid == 0) {  // after a timeout: bounded waits for what may still be in flight
        if (mma_out) mbar_wait(bar, mma_par, &g_tc_status, ERR_WAIT_TIMEOUT);
        for (int bb = 0; bb < 2; ++bb)
            if (pending & (1u << bb))
                mbar_wait(bar_img + bb, (img_parity >> bb) & 1u, &g_tc_status, ERR_WAIT_TIMEOUT);
        if (pending & 4u) mbar_wait(bar_gate, gate_parity, &g_tc_status, ERR_WAIT_TIMEOUT);
    }
    if (tid == 0) bulk_wait_all();  // output stores are complete
    if (ok && sg.last && a.s_final) {  // slice wg: columns 32wg..32wg+31 of S^T
        float* sf = a.s_final + ((int64_t)sg.n * H + h) * D * D;
        for (int c0 = 32 * wg; c0 < 32 * wg + 32; c0 += 16) {
            float v[16];
            tmem_ld16(tq + TM_S + c0, v);
            tmem_wait16(v);
#pragma unroll
            for (int i = 0; i < 16; ++i) sf[(int64_t)(c0 + i) * D + lrow] = v[i];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- bounded-wait self-test
// One thread waits through the kernels' bounded mbarrier wait, with the given limit, on
// a fresh mbarrier of arrival count 1.  With arrive = 1 it arrives first, so the wait
// completes at once; otherwise nothing ever arrives, the wait gives up after timeout_ns
// and records ERR_WAIT_TIMEOUT in the device status word, and the kernel returns.
__global__ void wait_probe_kernel(uint64_t timeout_ns, int arrive) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (arrive) mbar_arrive(&bar);
    (void)mbar_wait(&bar, 0, &g_tc_status, ERR_WAIT_TIMEOUT, timeout_ns);
}

// ---------------------------------------------------------------- segment table
// One CTA.  Sequence n has nch = ceil(len/64) chunks and G_n = max(1,
// ceil(nch / seg_chunks)) segments; segment j covers chunks [j*seg_chunks,
// min(nch, (j+1)*seg_chunks)).
__global__ void __launch_bounds__(1024) seg_setup_kernel(const int32_t* cu, int N, int T,
                                                         int seg_chunks, int max_units,
                                                         SegEntry* segs, int32_t* seg_off,
                                                         int32_t* n_units) {
    __shared__ int32_t warp_sums[32];
    __shared__ int64_t warp_csums[32];
    __shared__ int32_t carry;
    __shared__ int64_t carry_c;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) {
        carry = 0;
        carry_c = 0;
    }
    __syncthreads();
    for (int base = 0; base < N; base += 1024) {
        const int n = base + tid;
        int64_t lo = 0, hi = 0;
        if (n < N) {
            lo = cu ? cu[n] : (int64_t)n * T;
            hi = cu ? cu[n + 1] : lo + T;
        }
        const int64_t nch = hi > lo ? (hi - lo + C - 1) / C : 0;
        int g = n < N ? (int)(nch > 0 ? (nch + seg_chunks - 1) / seg_chunks : 1) : 0;
        // block-wide exclusive scans of g (segments) and nch (chunks)
        int xg = g;
        long long xc = nch;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, xg, o);
            const long long yc = __shfl_up_sync(0xffffffffu, xc, o);
            if (lane >= o) {
                xg += y;
                xc += yc;
            }
        }
        if (lane == 31) {
            warp_sums[warp] = xg;
            warp_csums[warp] = xc;
        }
        __syncthreads();
        if (warp == 0) {
            int w = warp_sums[lane];
            long long wc = warp_csums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                const long long yc = __shfl_up_sync(0xffffffffu, wc, o);
                if (lane >= o) {
                    w += y;
                    wc += yc;
                }
            }
            warp_sums[lane] = w;
            warp_csums[lane] = wc;
        }
        __syncthreads();
        const int excl = carry + xg - g + (warp > 0 ? warp_sums[warp - 1] : 0);
        const int64_t cexcl = carry_c + xc - nch + (warp > 0 ? warp_csums[warp - 1] : 0);
        if (n < N) {
            seg_off[n] = excl;
            for (int j = 0; j < g; ++j) {
                const int uidx = excl + j;
                if (uidx >= max_units) {
                    atomicCAS(&g_tc_status, 0, ERR_SEG_OVERFLOW);
                    break;
                }
                SegEntry en;
                en.n = n;
                en.j = j;
                en.t_begin = lo + (int64_t)j * seg_chunks * C;
                const int64_t end = lo + (int64_t)(j + 1) * seg_chunks * C;
                en.t_end = end < hi ? end : hi;
                en.last = (j == g - 1) ? 1 : 0;
                en.pad = 0;
                en.c_base = cexcl + (int64_t)j * seg_chunks;
                segs[uidx] = en;
            }
        }
        __syncthreads();
        if (tid == 1023) {
            carry = excl + g;
            carry_c = cexcl + nch;
        }
        __syncthreads();
    }
    if (tid == 0) {
        seg_off[N] = carry;
        *n_units = carry < max_units ? carry : max_units;
    }
}

// ---------------------------------------------------------------- segment scan
// S_in^T(j+1) = S_in^T(j) M_j^T + B_j^T for the 8 rows e in [8*blockIdx.z, +8) of S^T,
// sequentially over the segments of sequence n, head h (rows of S^T are independent, so
// the CTAs of one head need nothing from each other).  M_j^T (64 KB) sits in shared
// memory; the next one, and the next B_j^T rows, are loaded into registers while the
// current product runs.  Thread (el, cg) owns row el and columns 4cg..4cg+3; each output
// is B + sum over c of S[c] M[c][col] in order of c.
constexpr int SCAN_ROWS = 8;
constexpr int SCAN_SMEM = D * D * 4 + SCAN_ROWS * D * 4;
__global__ void __launch_bounds__(256) seg_scan_kernel(TcArgs a) {
    extern __shared__ float4 scan_smem4[];
    float* Ms = reinterpret_cast<float*>(scan_smem4);  // [128][128]
    float* S = Ms + D * D;                            // [SCAN_ROWS][128]
    const int n = blockIdx.x, h = blockIdx.y, e0 = SCAN_ROWS * blockIdx.z, H = a.H;
    const int tid = threadIdx.x, el = tid >> 5, cg = tid & 31;
    const int32_t u0 = a.seg_off[n], u1 = a.seg_off[n + 1];
    const int32_t nu = *a.n_units;
    KDA_DCHECK(0 <= u0 && u0 <= u1 && nu >= 0);  // transitions and states indexed below nu
    if (u1 - u0 <= 1 || u0 >= nu) return;
    const int32_t last = (u1 < nu ? u1 : nu) - 1;  // segments u0 .. last; transitions u0 .. last-1
    // S_in of segment 0, also copied to the workspace so that pass 3 never reads
    // initial_state while another segment may be writing final_state (they may
    // be the same buffer)
    for (int x = tid; x < SCAN_ROWS * D; x += 256) {
        const int r = x / D, c = x % D;
        const float v = a.s0 ? a.s0[(((int64_t)n * H + h) * D + c) * D + e0 + r] : 0.f;
        S[r * D + c] = v;
        a.sin[((int64_t)u0 * H + h) * D * D + (int64_t)(e0 + r) * D + c] = v;
    }
    float4 pre[16], bpre;
    auto load_next = [&](int32_t uu) {  // M_uu^T and this thread's four entries of B_uu^T
        const float4* T = reinterpret_cast<const float4*>(a.trans + ((int64_t)uu * H + h) * 2 * D * D);
#pragma unroll
        for (int i = 0; i < 16; ++i) pre[i] = __ldg(T + D * D / 4 + tid + 256 * i);
        bpre = __ldg(T + ((e0 + el) * D + 4 * cg) / 4);
    };
    auto store_m = [&]() {
        float4* dst = reinterpret_cast<float4*>(Ms);
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[tid + 256 * i] = pre[i];
    };
    if (u0 < last) {
        load_next(u0);
        store_m();
    }
    __syncthreads();
    for (int32_t uu = u0; uu < last; ++uu) {
        float acc[4] = {bpre.x, bpre.y, bpre.z, bpre.w};
        if (uu + 1 < last) load_next(uu + 1);
#pragma unroll 8
        for (int c = 0; c < D; ++c) {
            const float sv = S[el * D + c];
            const float4 m = *reinterpret_cast<const float4*>(Ms + c * D + 4 * cg);
            acc[0] = fmaf(sv, m.x, acc[0]);
            acc[1] = fmaf(sv, m.y, acc[1]);
            acc[2] = fmaf(sv, m.z, acc[2]);
            acc[3] = fmaf(sv, m.w, acc[3]);
        }
        __syncthreads();  // everyone is done reading S and M_uu
        *reinterpret_cast<float4*>(S + el * D + 4 * cg) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4*>(a.sin + ((int64_t)(uu + 1) * H + h) * D * D + (int64_t)(e0 + el) * D +
                                   4 * cg) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        if (uu + 1 < last) store_m();
        __syncthreads();
    }
}

}  // namespace

size_t tc_smem_bytes() { return Lay<FWD>::BYTES; }

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [T, H, 128] tensor, tile box (128 channels, 1 head, 64 tokens) without swizzle,
// or (64 channels, 1 head, 64 tokens) with the 128-byte swizzle of the MMA operand
// layouts; zero fill past the end.
cudaError_t tile_map(CUtensorMap* m, const void* base, bool f32, int H, int64_t T, bool sw128) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t e = f32 ? 4 : 2;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * e, (cuuint64_t)H * D * e};
    const cuuint32_t box[3] = {(cuuint32_t)(sw128 ? 64 : D), 1, (cuuint32_t)C};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r =
        fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
           const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
           sw128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// tensor maps of every input (and the output and gate) that are present
cudaError_t make_maps(const TcArgs& a, TcMaps* maps) {
    memset(maps, 0, sizeof *maps);
    const int64_t tokens = (int64_t)a.B * a.T;
    if (tokens <= 0) return cudaSuccess;
    cudaError_t err;
    if ((err = tile_map(&maps->k, a.k, false, a.H, tokens, false)) != cudaSuccess ||
        (err = tile_map(&maps->v, a.v, false, a.H, tokens, true)) != cudaSuccess ||
        (err = tile_map(&maps->la, a.log_alpha, true, a.H, tokens, false)) != cudaSuccess)
        return err;
    if (a.H % 4 == 0) {  // beta as [T][H] fp32, box (4 heads, 64 tokens)
        EncodeTiledFn fn = encode_tiled();
        if (!fn) return cudaErrorNotSupported;
        const cuuint64_t dims[2] = {(cuuint64_t)a.H, (cuuint64_t)tokens};
        const cuuint64_t strides[1] = {(cuuint64_t)a.H * 4};
        const cuuint32_t box[2] = {4, (cuuint32_t)C};
        const cuuint32_t estr[2] = {1, 1};
        if (fn(&maps->beta, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(a.beta), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        maps->beta_tma = 1;
    }
    if (a.q && (err = tile_map(&maps->q, a.q, false, a.H, tokens, false)) != cudaSuccess) return err;
    if (a.out && (err = tile_map(&maps->out, a.out, false, a.H, tokens, false)) != cudaSuccess)
        return err;
    if (a.gate && (err = tile_map(&maps->gate, a.gate, false, a.H, tokens, false)) != cudaSuccess)
        return err;
    return cudaSuccess;
}

// per device, once: the kernels' shared-memory limits
cudaError_t set_attributes() {
    static bool done[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < kMaxDevices && done[dev]) return cudaSuccess;
    if ((err = cudaFuncSetAttribute(chunk_kernel<FWD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)Lay<FWD>::BYTES)) != cudaSuccess ||
        (err = cudaFuncSetAttribute(chunk_kernel<TRANS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)Lay<TRANS>::BYTES)) != cudaSuccess ||
        (err = cudaFuncSetAttribute(chunk_kernel<DUMP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)Lay<DUMP>::BYTES)) != cudaSuccess ||
        (err = cudaFuncSetAttribute(chunk_kernel<TRANS_CACHE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)Lay<TRANS_CACHE>::BYTES)) != cudaSuccess ||
        (err = cudaFuncSetAttribute(cached_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)LayC::BYTES)) != cudaSuccess ||
        (err = cudaFuncSetAttribute(seg_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    SCAN_SMEM)) != cudaSuccess)
        return err;
    if (dev < kMaxDevices) done[dev] = true;
    return cudaSuccess;
}

cudaError_t launch_setup(const TcArgs& a, const TcPlan& p, cudaStream_t stream, int* launches) {
    profile_mark(SLOT_SETUP, true, stream);
    seg_setup_kernel<<<1, 1024, 0, stream>>>(a.cu, a.N, a.T, p.seg_chunks, p.max_units, a.segs,
                                             a.seg_off, a.n_units);
    profile_mark(SLOT_SETUP, false, stream);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_pass1(const TcArgs& a, const TcPlan& p, const TcMaps& maps, cudaStream_t stream,
                         int* launches) {
    profile_mark(SLOT_PASS1, true, stream);
    const dim3 grid((unsigned)p.max_units, (unsigned)a.H);
    if (a.cache)
        chunk_kernel<TRANS_CACHE><<<grid, NT, Lay<TRANS_CACHE>::BYTES, stream>>>(a, maps);
    else
        chunk_kernel<TRANS><<<grid, NT, Lay<TRANS>::BYTES, stream>>>(a, maps);
    profile_mark(SLOT_PASS1, false, stream);
    *launches += 1;
    return cudaGetLastError();
}
}  // namespace

cudaError_t status_word(int** p) {
    static int* addr[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* a = nullptr;
        e = cudaGetSymbolAddress(&a, g_tc_status);
        if (e != cudaSuccess) return e;
        addr[dev] = (int*)a;
    }
    *p = addr[dev];
    return cudaSuccess;
}

#ifdef KDA_PHASE_TRACE
extern "C" int kda_trace_read(unsigned long long* host, int n) {
    const int total = 2 * kTraceChunks * kTraceStamps;
    if (n > total) n = total;
    if (cudaMemcpyFromSymbol(host, g_trace, (size_t)n * sizeof(unsigned long long)) != cudaSuccess)
        return -1;
    return n;
}
extern "C" int kda_trace_spans(unsigned long long* host, int n) {
    const int total = kSpanCtas * 6;
    if (n > total) n = total;
    if (cudaMemcpyFromSymbol(host, g_span, (size_t)n * sizeof(unsigned long long)) != cudaSuccess)
        return -1;
    return n;
}
extern "C" int kda_trace_first_chunk(long long c0) {
    return cudaMemcpyToSymbol(g_trace_c0, &c0, sizeof(c0)) == cudaSuccess ? 0 : -1;
}
#endif

cudaError_t tc_take_status(int* code) {
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_tc_status, sizeof(int));
    if (e == cudaSuccess && *code) e = cudaMemcpyToSymbol(g_tc_status, &zero, sizeof(int));
    return e;
}

cudaError_t launch_tc(const TcArgs& a, const TcPlan& p, cudaStream_t stream, int* launches,
                      bool from_span) {
    cudaError_t err = set_attributes();
    if (err != cudaSuccess) return err;
    TcMaps maps;
    if ((err = make_maps(a, &maps)) != cudaSuccess) return err;
    if (!from_span) {  // else the segment table and the transitions are in the workspace
        {
            NvtxRange r("kda.segment_table");
            if ((err = launch_setup(a, p, stream, launches)) != cudaSuccess) return err;
        }
        if (p.segmented) {
            NvtxRange r("kda.pass1_transitions");
            if ((err = launch_pass1(a, p, maps, stream, launches)) != cudaSuccess) return err;
        }
    }
    if (p.segmented) {
        NvtxRange r("kda.segment_scan");
        profile_mark(SLOT_SCAN, true, stream);
        seg_scan_kernel<<<dim3((unsigned)a.N, (unsigned)a.H, D / SCAN_ROWS), 256, SCAN_SMEM, stream>>>(a);
        profile_mark(SLOT_SCAN, false, stream);
        *launches += 1;
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    NvtxRange r("kda.pass3_forward");
    profile_mark(SLOT_PASS3, true, stream);
    const dim3 grid((unsigned)p.max_units, (unsigned)a.H);
    if (p.segmented && a.cache)
        cached_kernel<<<grid, NT, LayC::BYTES, stream>>>(a, maps);
    else
        chunk_kernel<FWD><<<grid, NT, Lay<FWD>::BYTES, stream>>>(a, maps);
    profile_mark(SLOT_PASS3, false, stream);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_transition(const TcArgs& a_in, const TcPlan& p, float* out, cudaStream_t stream,
                              int* launches) {
    TcArgs a = a_in;
    a.trans_all = 1;
    cudaError_t err = set_attributes();
    if (err != cudaSuccess) return err;
    TcMaps maps;
    if ((err = make_maps(a, &maps)) != cudaSuccess) return err;
    if ((err = launch_setup(a, p, stream, launches)) != cudaSuccess) return err;
    if ((err = launch_pass1(a, p, maps, stream, launches)) != cudaSuccess) return err;
    // compose each sequence's segment transitions into one
    ChainArgs c;
    c.trans = a.trans;
    c.off = a.seg_off;
    c.n_units = a.n_units;
    c.count = 0;
    c.B = a.N;
    c.H = a.H;
    c.s0 = nullptr;
    c.out = out;
    c.compose = 1;
    return launch_chain(c, stream, launches);
}

// Debug builds: each guard band around a workspace buffer still holds kGuardWord.
__global__ void __launch_bounds__(256) guard_check_kernel(GuardBands g) {
    const int b = blockIdx.x;
    bool bad = false;
    for (int i = threadIdx.x; i < (int)(kGuardBytes / 4); i += 256) bad |= g.band[b][i] != kGuardWord;
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicCAS(&g_tc_status, 0, ERR_DEBUG_GUARD | (b << 8));
}

cudaError_t launch_guard_check(const GuardBands& g, cudaStream_t stream) {
    if (g.n <= 0 || g.n > kMaxGuards) return cudaErrorInvalidValue;
    guard_check_kernel<<<g.n, 256, 0, stream>>>(g);
    return cudaGetLastError();
}

cudaError_t launch_wait_probe(uint64_t timeout_ns, int arrive, cudaStream_t stream) {
    wait_probe_kernel<<<1, 32, 0, stream>>>(timeout_ns, arrive);
    return cudaGetLastError();
}

cudaError_t launch_dump(const TcArgs& a, const TcPlan& p, cudaStream_t stream, int* launches) {
    cudaError_t err = set_attributes();
    if (err != cudaSuccess) return err;
    TcMaps maps;
    if ((err = make_maps(a, &maps)) != cudaSuccess) return err;
    if ((err = launch_setup(a, p, stream, launches)) != cudaSuccess) return err;
    chunk_kernel<DUMP><<<dim3((unsigned)p.max_units, (unsigned)a.H), NT, Lay<DUMP>::BYTES, stream>>>(a, maps);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace kda
