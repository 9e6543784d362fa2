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
//   seg_setup   : segment table from cu_seqlens (or B x T) on the device.
//   tc_kernel<1> "pass 1": per (segment, head) the transition (B, M) of the
//                 segment, computed as the chunk loop applied to the augmented
//                 state [B | M] from [0 | I].  When sequences are cut into
//                 segments it runs over every segment and also leaves in a
//                 chunk cache, for every chunk, the operand images pass 3
//                 needs: W^T, U'^T, K_dec, Q~ and P (bf16) and gamma.
//   seg_scan    : S_in(j+1) = M_j S_in(j) + B_j, sequential over the segments
//                 of a sequence, parallel over (sequence, head, 16-row block).
//   cached_kernel "pass 3" with the cache: per (segment, head) the state chain
//                 from the true incoming state and the output, every chunk's
//                 operands bulk-loaded from the cache (double-buffered), so
//                 only the four state/output products remain per chunk.
//   tc_kernel<0> "pass 3" without a cache (one segment per sequence): the full
//                 chunk loop, writing o and the final state.
//
// Per chunk of C = 64 tokens (g = in-chunk inclusive cumsum of the clamped
// log-gates, per key channel), everything in the transposed orientation so
// that every tensor-core product has M = 128 rows:
//   A  = strict_lower(diag(beta) (K e^g)(K e^-g)^T),  P = lower_incl((Q e^g)(K e^-g)^T)
//   T  = (I + A)^-1                                      (fp32, CUDA cores)
//   W^T = (diag(beta) K e^g)^T T^T,   U'^T = (diag(beta) V)^T T^T
//   U^T = U'^T - S^T W^T
//   O^T = S^T (Q e^g)^T + U^T P^T
//   S^T <- S^T Diag(e^{g_last}) + U^T (K e^{g_last - g})
// The state S^T (d_v x d_k, fp32) stays in tensor memory for the whole
// segment; it enters the products as a bf16 copy.  Gate factors are
// referenced to the middle of each 32-token half (rho_a = g_15, rho_b = g_47)
// so every factor handed to the tensor core lies in [e^-80, e^80], inside the
// bf16/fp32 exponent range; the cross-half block of A and P is a separate
// product whose factors are both <= 1 (underflow to 0 is the correct limit).
#include <cuda_bf16.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "kda_internal.h"
#include "tc_common.cuh"

namespace kda {
namespace {

__device__ int g_tc_status = 0;  // first device-side error code of this device (0 = none)


using namespace tc;

constexpr int C = 64;     // tokens per chunk
constexpr int D = 128;    // d_k = d_v
constexpr int NT = 512;   // threads per CTA: 16 warps, 4 per TMEM lane quadrant
constexpr float LOG2E = 1.4426950408889634f;


// ---------------------------------------------------------------- shared memory map
// Region R1 is reused across the phases of one chunk:
//   phases 0-3: X1 (A operand, 128 x 128, K-major: rows 0-63 k e^{g-rho}, rows
//               64-127 q e^{g-rho}); its k rows (bytes [0,8K) and [16K,24K)) are read
//               again by the phase-3 W products, as an MN-major operand.
//               BT (B operand, 96 x 128) until the phase-1 product completes.
//   phase  2  : As, Ts (fp32, strides 68 and 72) in BT's place, Ys in a q-row hole,
//               then TB (bf16 T diag(beta)) in the other q-row hole
//   phases 3-8: WB (W^T) over X1; pass 1 also UA (U'^T, kept with W^T for pass 3)
//               over X1 and MA (bf16 M^T) after Ts.  The bf16 copies of S^T, B^T,
//               U^T, U_B^T and U_M^T that the state products take as A operands
//               live in tensor memory.
//   pass 1 with the chunk cache also builds q~ in X1's rows 64-127 (so the phase-1
//               product yields P in TMEM lanes 64-127) and P's bf16 image in GSUM.
// RAW holds the next chunk's k, log alpha (and q) tiles, written by TMA while
// the current chunk is processed; RV0/RV1 alternate as the chunk's v tile, which
// TMA writes directly in the 128-byte-swizzled MN-major operand layout.
template <bool SEG>
struct LayT {
    static constexpr uint32_t X1 = 0, BT = 32768;
    static constexpr uint32_t AS = 32768, TS = AS + 17408, YS = 24576, TB = 8192;
    static constexpr uint32_t WB = 0, UA = 16384, MA = 69632;
    static constexpr uint32_t R1 = SEG ? 102400 : 69632;
    static constexpr uint32_t QT = R1;                            // pass 3: 64 x 128, K-major
    static constexpr uint32_t KD = SEG ? R1 : QT + 16384;         // 64 x 128, MN-major
    static constexpr uint32_t PB = KD + 16384;                    // pass 3: 64 x 64, K-major
    static constexpr uint32_t RAW = SEG ? KD + 32768 : PB + 8192;
    static constexpr uint32_t RK = RAW, RL = RAW + 16384;
    static constexpr uint32_t RQ = SEG ? KD + 16384 : RAW + 49152;  // pass 1: only with the cache
    static constexpr uint32_t RV = RAW + (SEG ? 49152 : 65536);   // two 16 KB buffers
    static constexpr uint32_t GSUM = RV + 32768;                  // fp32 [16][128]
    static constexpr uint32_t GAM = GSUM + 8192;                  // fp32 [128] e^{g_last}
    static constexpr uint32_t EHA = GAM + 512;                    // fp32 [128] e^{rho_a}
    static constexpr uint32_t EHB = EHA + 512;                    // fp32 [128] e^{rho_b}
    static constexpr uint32_t FAC = EHB + 512;                    // fp32 [5][128] gate factors
    static constexpr uint32_t BETA = FAC + 2560;                  // fp32 [64]
    static constexpr uint32_t BAR = BETA + 256;                   // mbarriers: MMA, TMA, gate, W
    static constexpr uint32_t TMEMP = BAR + 32;                   // TMEM base address
    static constexpr uint32_t END = TMEMP + 16;
    static constexpr uint32_t BYTES = END + 1024;                 // + alignment slack
};
static_assert(LayT<false>::TS + 64 * 72 * 4 <= LayT<false>::R1, "As/Ts overflow");
static_assert(LayT<false>::YS + 32 * 40 * 4 <= 32768 && LayT<false>::TB + 8192 <= 16384,
              "Ys/TB must sit in the q-row holes of X1");
static_assert(LayT<true>::WB + 16384 == LayT<true>::UA, "pass 1 stores W^T and U'^T as one 32 KB copy");
static_assert(LayT<true>::MA + 32768 <= LayT<true>::R1, "MA overflow");
static_assert(LayT<true>::RQ + 16384 <= LayT<true>::RAW, "pass 1 q tile");
static_assert(LayT<false>::BYTES <= 232448 && LayT<true>::BYTES <= 232448, "shared memory");

// TMEM columns (512 allocated).  Pass 3: AP [0,96) W [96,160) U [160,224)
// O [224,288) bf16 S^T [288,352) bf16 U^T [352,384) S [384,512).  Pass 1: AP/U_M [0,96) W U as
// above (W's columns later hold bf16 U_B^T [96,128) and U_M^T [128,160)), B [256,384), M [384,512).
constexpr uint32_t TM_AP = 0, TM_W = 96, TM_U = 160, TM_O = 224;
constexpr uint32_t TM_O2 = 0;  // cached_kernel: the second O accumulator (TM_AP's columns, unused there)
constexpr uint32_t TM_SB = 288, TM_UB = 352;  // pass 3: bf16 copies of S^T and U^T (A operands)
constexpr uint32_t TM_B = 256, TM_S = 384, TM_M = 384;
constexpr uint32_t TM_UBB = 96, TM_UBM = 128;  // pass 1: bf16 U_B^T, U_M^T (A operands) in the W columns
// pass 1: bf16 B^T (A operand of U_B -= B W): K steps 0-3 (channels 0-63) in [64,96), which the
// cross-half block of A has left, and K steps 4-7 in [224,256), unused in pass 1
__device__ __forceinline__ uint32_t sbb_col(int s) { return s < 4 ? 64 + 8 * s : 224 + 8 * (s - 4); }

// Chunk cache entry (kChunkImageBytes per chunk and head): the bf16 operand images as
// they sit in shared memory, in 1024-byte aligned pieces (a bulk copy into a 1024-byte
// aligned buffer keeps their 128-byte swizzle), then gamma.
constexpr uint32_t CI_W = 0;        // W^T: MN-major, K rows = channels, MN = tokens
constexpr uint32_t CI_U = 16384;    // U'^T: [128][64], 16-byte pieces of row e XOR-swizzled by e & 7
constexpr uint32_t CI_KD = 32768;   // K_dec: MN-major, K rows = tokens, MN = channels
constexpr uint32_t CI_QT = 49152;   // Q~ (q e^{g - rho} e^{rho}): K-major, 64 rows x 128
constexpr uint32_t CI_PB = 65536;   // P: K-major, 64 x 64
constexpr uint32_t CI_GAM = 73728;  // fp32 [128] e^{g_last}
static_assert(CI_GAM + 512 == kChunkImageBytes, "chunk cache entry");

__device__ __forceinline__ float clamp_gate(float x) { return fminf(fmaxf(x, -5.f), 0.f); }
// 2^x by the SFU instruction (relative error about 2^-22, flushes results
// below 2^-126 to zero, which is harmless for the factors here)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void st8(uint8_t* base, uint32_t off, float a, float b, float c,
                                    float d) {
    uint2 v;
    v.x = pack_bf16(a, b);
    v.y = pack_bf16(c, d);
    *reinterpret_cast<uint2*>(base + off) = v;
}

__device__ __forceinline__ void unpack_bf16x4(const uint2 raw, float (&f)[4]) {
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
    f[0] = __low2float(lo);
    f[1] = __high2float(lo);
    f[2] = __low2float(hi);
    f[3] = __high2float(hi);
}

// Block-wide bounded wait on the MMA barrier; returns false (uniformly) if any
// thread gave up.
__device__ __forceinline__ bool wait_mma(void* bar, uint32_t& parity) {
    const bool ok = mbar_wait(bar, parity, &g_tc_status, ERR_WAIT_TIMEOUT);
    parity ^= 1u;
    tc_fence_after();
    return !__syncthreads_or(!ok);
}

// Copy NB x 16 TMEM columns (starting at TMEM address tm, tile column col0) of
// this thread's lane into row `row` of a bf16 tile (K-major with R rows, or
// MN-major with R K-rows when MN is true); optionally scale the TMEM copy by
// gam[col0 + i] in place.  All loads are issued before the first wait.
template <int NB, bool MN = false>
__device__ __forceinline__ void stage_cols(uint32_t tm, uint8_t* tile, int R, int row, int col0,
                                           const float* gam, bool scale_back) {
    float v[NB][16];
#pragma unroll
    for (int b = 0; b < NB; ++b) tmem_ld16(tm + 16 * b, v[b]);
#pragma unroll
    for (int b = 0; b < NB; ++b) tmem_wait16(v[b]);
    const uint32_t base = smem_u32(tile);
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int c8 = ((col0 + 16 * b) >> 3) + hh;
            const uint32_t off = MN ? mnmajor_chunk_off(row, c8, R) : kmajor_chunk_off(row, c8, R);
            st_shared_v4(base + off, pack_bf16(v[b][8 * hh + 0], v[b][8 * hh + 1]),
                         pack_bf16(v[b][8 * hh + 2], v[b][8 * hh + 3]),
                         pack_bf16(v[b][8 * hh + 4], v[b][8 * hh + 5]),
                         pack_bf16(v[b][8 * hh + 6], v[b][8 * hh + 7]));
        }
    if (scale_back) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[b][i] *= gam[col0 + 16 * b + i];
            tmem_st16(tm + 16 * b, v[b]);
        }
    }
}

// Copy 16 x NB fp32 TMEM columns at tm (tile columns col0..) of this thread's
// lane into NB x 8 packed-bf16 columns at tb (for an A operand read from TMEM);
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
#pragma unroll
            for (int i = 0; i < 16; ++i) v[b][i] *= gam[col0 + 16 * b + i];
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

// shared [64 tokens][128 channels] tile -> global tile at (0, h, t0) of a [T, H, 128] tensor
__device__ __forceinline__ void tma_store_tile(const CUtensorMap* map, const void* src, int h, int t0) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(0), "r"(h), "r"(t0), "r"(smem_u32(src))
        : "memory");
}
// plain bulk copies (8 KB T tiles): shared -> global (bulk group), global -> shared (mbarrier)
__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
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
    dst[g * ld + 2 * t] = sgn * d[0];
    dst[g * ld + 2 * t + 1] = sgn * d[1];
    dst[(g + 8) * ld + 2 * t] = sgn * d[2];
    dst[(g + 8) * ld + 2 * t + 1] = sgn * d[3];
}

// As: strictly lower 64 x 64 (fp32, stride AS_LD).  Writes TB = T diag(beta) as
// the bf16 K-major [r][j] tile tbp, where T = (I + A)^-1, using Ts (fp32, stride
// TS_LD) and Ys as scratch:
//  1. warp h (h = 0, 1) alone builds the 32 x 32 diagonal half h of T: its two
//     16 x 16 diagonal blocks by substitution (one lane per column, eliminating one
//     known entry at a time), then T_21 = -T_22 (A_21 T_11) inside the half with
//     tf32 warp MMAs -- warp-level synchronisation only;  the other warps zero the
//     upper-right 32 x 32 block of TB;
//  2. Z = A[32:64, 0:32] T_lo (8 warps, one 16 x 8 tile each);
//  3. T[32:64, 0:32] = -T_hi Z, written straight into TB.
// The block products are tf32 warp MMAs with fp32 accumulation (T then enters
// the chunk products as bf16).
// `side(warp)` runs on warps 2-15 while warps 0-1 invert the diagonal blocks
// (work that does not touch As, Ts, Ys or TB).  OWN_A: As has not been
// extracted; warps 0-1 (TMEM lanes 0-63 = rows of A, tq = their lane quadrant)
// read their rows of A from the product in TMEM, scale by beta, mask, and write
// the parts of As the later steps read (rows 0-31: columns 0-31; rows 32-63:
// columns 0-63), keeping their diagonal blocks in registers, so the inversion
// starts as soon as the product is complete.
template <bool OWN_A, typename Side>
__device__ void invert_to_tb(float* As, float* Ts, float* Ys, const float* beta, uint32_t tbp,
                             int tid, uint32_t tq, Side side) {
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t4 = lane & 3;
    if (warp < 2) {
        const int o = 32 * warp;
        {  // 1a. diagonal blocks o (lanes 0-15) and o+16 (lanes 16-31): lane i holds
           // row i of its block; T_i = e_i - sum_{m<i} A_im T_m, rows finished in order
           // and broadcast to the 16 lanes of the block by shuffles
            const int i = lane & 15, ob = o + 16 * (lane >> 4), src0 = lane & 16;
            float arow[16], trow[16];
            if (OWN_A) {
                const int r = o + lane;  // this lane's row of A
                const float br = beta[r];
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int j0 = 16 * cc;
                    if (warp == 0 && j0 >= 32) break;  // rows 0-31 need columns 0-31 only
                    float v[16];
                    // columns j < 32 of rows >= 32 are the cross-half product (TMEM 64 + j)
                    tmem_ld16(tq + TM_AP + (warp == 1 && j0 < 32 ? 64 + j0 : j0), v);
                    tmem_wait16(v);
#pragma unroll
                    for (int m = 0; m < 16; ++m) {
                        const float x = j0 + m < r ? br * v[m] : 0.f;
                        As[r * AS_LD + j0 + m] = x;
                        if (j0 == ob) arow[m] = x;
                    }
                }
                __syncwarp();
            } else {
#pragma unroll
                for (int m = 0; m < 16; ++m) arow[m] = m < i ? As[(ob + i) * AS_LD + ob + m] : 0.f;
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) trow[m] = m == i ? 1.f : 0.f;
#pragma unroll
            for (int m = 0; m < 15; ++m) {
                const float am = arow[m];
#pragma unroll
                for (int c = 0; c <= m; ++c) {  // row m has entries in columns 0..m only
                    const float tmc = __shfl_sync(0xffffffffu, trow[c], src0 + m);
                    trow[c] = fmaf(-am, tmc, trow[c]);
                }
            }
#pragma unroll
            for (int c = 0; c < 16; ++c) Ts[(ob + i) * TS_LD + ob + c] = trow[c];
            // zero the upper-right 16 x 16 block of this half (rows o..o+15, cols o+16..o+31)
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const int e = lane + 32 * x;
                Ts[(o + (e >> 4)) * TS_LD + o + 16 + (e & 15)] = 0.f;
            }
        }
        __syncwarp();
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
    } else {
        if (warp < 6) {  // zero TB rows 0..31, columns 32..63: 128 chunks
            const int id = tid - 64, r = id >> 2, j8 = 4 + (id & 3);
            st_shared_v4(tbp + kmajor_chunk_off(r, j8, 64), 0u, 0u, 0u, 0u);
        }
        side(warp);
    }
    __syncthreads();
    // 1c (warps 8-15, beside step 2). TB of the two diagonal halves: 2 x 32 rows x 4
    // chunks of 8 columns, one chunk per thread
    if (warp >= 8) {
        const int id = tid - 256, hf = id >> 7, r = 32 * hf + ((id >> 2) & 31), j8 = 4 * hf + (id & 3);
        const float* tr = Ts + r * TS_LD + 8 * j8;
        const float* bj = beta + 8 * j8;
        st_shared_v4(tbp + kmajor_chunk_off(r, j8, 64), pack_bf16(tr[0] * bj[0], tr[1] * bj[1]),
                     pack_bf16(tr[2] * bj[2], tr[3] * bj[3]), pack_bf16(tr[4] * bj[4], tr[5] * bj[5]),
                     pack_bf16(tr[6] * bj[6], tr[7] * bj[7]));
    }
    // 2. Z = A[32:64, 0:32] T_lo: warp (mt, nt) for warps 0-7
    const int mt = (warp >> 2) & 1, nt = warp & 3;
    if (warp < 8) {
        float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 8)
            warp_mma_tf32(d, As + (32 + 16 * mt) * AS_LD + k0, AS_LD, Ts + k0 * TS_LD + 8 * nt,
                          TS_LD, lane);
        warp_store16x8(Ys + 16 * mt * YS_LD + 8 * nt, YS_LD, d, 1.f, lane);
    }
    __syncthreads();
    // 3. T[32:64, 0:32] = -T_hi Z, scaled by beta_j, straight into TB
    if (warp < 8) {
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

// ---------------------------------------------------------------- the chunk loop
// MODE 0: pass 3 without a cache (forward from the true incoming state); MODE 1:
// pass 1 (segment transitions; with a.wu set, also the chunk cache for pass 3).
template <int MODE>
__global__ void __launch_bounds__(NT, 1) tc_kernel(TcArgs a, const __grid_constant__ TcMaps maps) {
    constexpr bool SEG = MODE == 1;
    using Lay = LayT<SEG>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int u = blockIdx.x, h = blockIdx.y, H = a.H;
    if (u >= *a.n_units) return;
    const SegEntry sg = a.segs[u];
    // transitions only for segments with a successor, unless all are asked for
    if (SEG && sg.last && !a.trans_all) return;
    const bool snap_on = !SEG && a.snap_pool != nullptr;
    const bool gate_on = !SEG && a.gate != nullptr;
    uint32_t gate_parity = 0;
    // Chunk cache (pass 1): the entry of the chunk at tt (the unit's chunk (tt - t_begin)/C,
    // chunk c_base + that among all chunks) and head h at
    // wu + ((c_base + (tt - t_begin)/C) H + h) * kChunkImageBytes, pieces at the CI_* offsets.
    const bool wu_cache = SEG && a.wu != nullptr;
    if (wu_cache && (sg.c_base < 0 || sg.c_base + (sg.t_end - sg.t_begin + C - 1) / C > a.total_chunks)) {
        if (tid == 0) atomicCAS(&g_tc_status, 0, ERR_SEG_OVERFLOW);  // malformed cu_seqlens
        return;
    }
    auto wu_tile = [&](int64_t tt) {
        return a.wu + ((sg.c_base + (tt - sg.t_begin) / C) * H + h) * (int64_t)kChunkImageBytes;
    };
    const int64_t seq_lo = snap_on ? (a.cu ? (int64_t)a.cu[sg.n] : (int64_t)sg.n * a.T) : 0;

    float* gsum = reinterpret_cast<float*>(sm + Lay::GSUM);
    float* gam = reinterpret_cast<float*>(sm + Lay::GAM);
    float* eha = reinterpret_cast<float*>(sm + Lay::EHA);
    float* ehb = reinterpret_cast<float*>(sm + Lay::EHB);
    float* beta_s = reinterpret_cast<float*>(sm + Lay::BETA);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Lay::BAR);
    uint64_t* bar_raw = bar + 1;
    uint64_t* bar_gate = bar + 2;  // output-gate tile (pass 3 with a gate)
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sm + Lay::TMEMP);

    if (warp == 0) {
        tmem_alloc(tmem_ptr, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init(bar_raw, 1);
        mbar_init(bar_gate, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    const int quad = warp & 3;                       // TMEM lane quadrant of this warp
    const int wg = warp >> 2;                        // column slice within the quadrant (0-3)
    const int lrow = quad * 32 + lane;               // TMEM lane / tile row owned by this thread
    const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16);
    uint32_t parity = 0;

    // ---- initial state (pass 3: each column slice wg writes 32 columns of S^T;
    // pass 1: wg 0-1 write B = 0, wg 2-3 write M = I, 64 columns each)
    if (!SEG) {
        const int e = lrow, cb = 32 * wg;
        for (int c0 = cb; c0 < cb + 32; c0 += 16) {
            float v[16];
            if (sg.j == 0 && sg.last) {  // single segment: read the caller's state
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
    } else {
        const int cb = 64 * (wg & 1);
        const bool is_m = wg >= 2;
        for (int c0 = cb; c0 < cb + 64; c0 += 16) {
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = (is_m && c0 + i == lrow) ? 1.f : 0.f;
            tmem_st16(tq + (is_m ? TM_M : TM_B) + c0, v);
        }
    }
    tmem_st_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // The next chunk's q, k, v and log alpha tiles are copied by TMA into RAW
    // while the current chunk is processed (issued once every thread has read
    // the current tiles into registers); beta goes through registers.
    const bool with_q = !SEG || wu_cache;  // pass 1 needs q only to fill the chunk cache
    // The raw tiles' tensor copies take long to issue: pass 1 issues them from warp 8,
    // which has no part in the per-channel prefix that follows; pass 3 from thread 0, which
    // must first see its output store leave the v buffer.  raw_pending (on that thread) /
    // gate_pending (thread 0): copies in flight.
    const int raw_tid = SEG ? 256 : 0;
    bool raw_pending = false, gate_pending = false;
    auto issue_raw = [&](int64_t tn, int vbuf) {
        raw_pending = true;
        mbar_expect_tx(bar_raw, with_q ? 81920u : 65536u);  // k, log alpha, v (, q)
        tma_tile(sm + Lay::RK, &maps.k, 0, h, (int)tn, bar_raw);
        tma_tile(sm + Lay::RL, &maps.la, 0, h, (int)tn, bar_raw);
        if (with_q) tma_tile(sm + Lay::RQ, &maps.q, 0, h, (int)tn, bar_raw);
        uint8_t* rv = sm + Lay::RV + vbuf * 16384;  // two 64-channel swizzled halves
        tma_tile(rv, &maps.v, 0, h, (int)tn, bar_raw);
        tma_tile(rv + 8192, &maps.v, 64, h, (int)tn, bar_raw);
    };
    uint32_t raw_parity = 0;
    float beta_ld = 0.f;
    if (sg.t_begin < sg.t_end) {
        if (tid == raw_tid) issue_raw(sg.t_begin, 0);
        if (tid < C && sg.t_begin + tid < sg.t_end) beta_ld = __ldg(a.beta + (sg.t_begin + tid) * H + h);
    }

    bool ok = true;
    int vbuf = 0;  // RV buffer and O buffer of the current chunk
    for (int64_t t0 = sg.t_begin; t0 < sg.t_end && ok; t0 += C, vbuf ^= 1) {
        const int Lc = (int)((sg.t_end - t0) < C ? (sg.t_end - t0) : C);

        // ============ phase 0: gates, scaled operands
        {
            const int c4 = lane, tg = warp, c0 = 4 * c4;  // tokens 4tg..4tg+3, channels c0..c0+3
            float4 la[4];
            uint2 kr[4], qr[4];
            // the last chunk's cache stores have read WB, UA, KD, GSUM and GAM
            if (wu_cache && tid == 0) bulk_wait_read();
            if (!(ok = !__syncthreads_or(!mbar_wait(bar_raw, raw_parity, &g_tc_status,
                                                    ERR_WAIT_TIMEOUT)))) break;
            raw_parity ^= 1u;
            raw_pending = false;
#pragma unroll
            for (int i = 0; i < 4; ++i) {  // rows past the segment end act as identity steps
                const int r = 4 * tg + i;
                la[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                kr[i] = qr[i] = make_uint2(0u, 0u);
                if (r < Lc) {
                    la[i] = *reinterpret_cast<const float4*>(sm + Lay::RL + (r * D + c0) * 4);
                    kr[i] = *reinterpret_cast<const uint2*>(sm + Lay::RK + (r * D + c0) * 2);
                    if (with_q) qr[i] = *reinterpret_cast<const uint2*>(sm + Lay::RQ + (r * D + c0) * 2);
                } else {  // the v tile is an operand as TMA wrote it: clear rows past the end
                    *reinterpret_cast<uint2*>(sm + Lay::RV + vbuf * 16384 + mnmajor_off(r, c0, 64)) =
                        make_uint2(0u, 0u);
                }
            }
            float g[4][4];
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[0] += clamp_gate(la[i].x);
                acc[1] += clamp_gate(la[i].y);
                acc[2] += clamp_gate(la[i].z);
                acc[3] += clamp_gate(la[i].w);
#pragma unroll
                for (int c = 0; c < 4; ++c) g[i][c] = acc[c];
            }
            *reinterpret_cast<float4*>(gsum + tg * D + c0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            if (tid < C) beta_s[tid] = beta_ld;
            __syncthreads();
            // every thread holds its raw inputs: RAW may now receive the next chunk
            if (t0 + C < sg.t_end) {
                if (tid == raw_tid) {
                    if (!SEG) bulk_wait_read();  // the v buffer may still be feeding an output store
                    issue_raw(t0 + C, vbuf ^ 1);
                }
                beta_ld = (tid < C && t0 + C + tid < sg.t_end) ? __ldg(a.beta + (t0 + C + tid) * H + h) : 0.f;
            }
            // one thread per channel: exclusive prefix of the 16 token groups (in place),
            // references rho_a = g_15, rho_b = g_47, g_last = g_63 and the factors
            //   FAC[0] rho_a, FAC[1] rho_b (log2 units), FAC[2] e^{g_last - rho_a},
            //   FAC[3] e^{g_last - rho_b}, FAC[4] e^{rho_b - rho_a}
            float* fac = reinterpret_cast<float*>(sm + Lay::FAC);
            if (tid < D) {
                const int c = tid;
                float run = 0.f, ra = 0.f, rb = 0.f;
#pragma unroll
                for (int t2 = 0; t2 < 16; ++t2) {
                    const float x = gsum[t2 * D + c];
                    gsum[t2 * D + c] = run;
                    run += x;
                    if (t2 == 3) ra = run;
                    if (t2 == 11) rb = run;
                }
                fac[c] = ra * LOG2E;
                fac[D + c] = rb * LOG2E;
                fac[2 * D + c] = ex2((run - ra) * LOG2E);
                fac[3 * D + c] = ex2((run - rb) * LOG2E);
                fac[4 * D + c] = ex2((rb - ra) * LOG2E);
                gam[c] = ex2(run * LOG2E);
                eha[c] = ex2(ra * LOG2E);
                ehb[c] = ex2(rb * LOG2E);
            }
            __syncthreads();
            const bool hb = tg >= 8;  // tokens 4tg.. lie in the second half
            const float4 off4 = *reinterpret_cast<const float4*>(gsum + tg * D + c0);
            const float4 rho4 = *reinterpret_cast<const float4*>(fac + (hb ? D : 0) + c0);
            const float4 eh4 = *reinterpret_cast<const float4*>((hb ? ehb : eha) + c0);
            const float4 dh4 = *reinterpret_cast<const float4*>(fac + (hb ? 3 : 2) * D + c0);
            const float4 fba4 = *reinterpret_cast<const float4*>(fac + 4 * D + c0);
            const float off[4] = {off4.x, off4.y, off4.z, off4.w};
            const float rho2[4] = {rho4.x, rho4.y, rho4.z, rho4.w};  // log2 units
            const float Eh[4] = {eh4.x, eh4.y, eh4.z, eh4.w};
            const float Dh[4] = {dh4.x, dh4.y, dh4.z, dh4.w};
            const float fba[4] = {fba4.x, fba4.y, fba4.z, fba4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 4 * tg + i;
                float kf[4], qf[4];
                unpack_bf16x4(kr[i], kf);
                unpack_bf16x4(qr[i], qf);
                float e1[4], e2[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float d2 = fmaf(g[i][c] + off[c], LOG2E, -rho2[c]);
                    e1[c] = ex2(d2);
                    e2[c] = ex2(-d2);
                }
                st8(sm + Lay::X1, kmajor_off(r, c0, 128), kf[0] * e1[0], kf[1] * e1[1],
                    kf[2] * e1[2], kf[3] * e1[3]);
                if (with_q)
                    st8(sm + Lay::X1, kmajor_off(64 + r, c0, 128), qf[0] * e1[0],
                        qf[1] * e1[1], qf[2] * e1[2], qf[3] * e1[3]);
                st8(sm + Lay::BT, kmajor_off(r, c0, 96), kf[0] * e2[0], kf[1] * e2[1],
                    kf[2] * e2[2], kf[3] * e2[3]);
                if (r < 32)
                    st8(sm + Lay::BT, kmajor_off(64 + r, c0, 96), kf[0] * e2[0] * fba[0],
                        kf[1] * e2[1] * fba[1], kf[2] * e2[2] * fba[2], kf[3] * e2[3] * fba[3]);
                if (!SEG)
                    st8(sm + Lay::QT, kmajor_off(r, c0, 64), qf[0] * e1[0] * Eh[0],
                        qf[1] * e1[1] * Eh[1], qf[2] * e1[2] * Eh[2], qf[3] * e1[3] * Eh[3]);
                else if (wu_cache)  // Q~'s image straight into the cache: each warp row is
                                    // two contiguous 128-byte pieces
                    st8(wu_tile(t0) + CI_QT, kmajor_off(r, c0, 64), qf[0] * e1[0] * Eh[0],
                        qf[1] * e1[1] * Eh[1], qf[2] * e1[2] * Eh[2], qf[3] * e1[3] * Eh[3]);
                st8(sm + Lay::KD, mnmajor_off(r, c0, 64), kf[0] * e2[0] * Dh[0],
                    kf[1] * e2[1] * Dh[1], kf[2] * e2[2] * Dh[2], kf[3] * e2[3] * Dh[3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ============ phase 1: [A;P] = X1 . BT^T   (M=128, N=96, K=128)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t x1 = smem_u32(sm + Lay::X1), bt = smem_u32(sm + Lay::BT);
            constexpr uint32_t id = idesc_bf16(128, 96, false, false);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16(tmem + TM_AP, kmajor_desc(x1, 128, s), kmajor_desc(bt, 96, s), id, s > 0);
            mma_commit(bar);
            if (wu_cache) {  // K_dec and gamma are final: into the chunk cache
                bulk_store(wu_tile(t0) + CI_KD, sm + Lay::KD, 16384);
                bulk_store(wu_tile(t0) + CI_GAM, sm + Lay::GAM, 512);
                bulk_commit();
            }
        }
        if (!(ok = wait_mma(bar, parity))) break;

        // ============ phase 2: masks, beta, (I + A)^-1, P
        {
            float* As = reinterpret_cast<float*>(sm + Lay::AS);
            float* Ts = reinterpret_cast<float*>(sm + Lay::TS);
            float* Ys = reinterpret_cast<float*>(sm + Lay::YS);
            // MODE 0: rows r of A (lanes 0-63) into As and of P (lanes 64-127) into PB; warp
            // slice wg handles the 16 columns j in [16wg, 16wg+16).  Pass 1 extracts A
            // inside the inversion (and, with the cache, P beside it).
            if (!SEG) {
                const int r = lrow & 63, j0 = 16 * wg;
                if (quad >= 2) {
                    extract_p16(tq, r, j0, smem_u32(sm + Lay::PB));
                } else {
                    float x[16];
                    if (j0 >= 32 && r < 32) {  // warp-uniform
#pragma unroll
                        for (int i = 0; i < 16; ++i) x[i] = 0.f;
                    } else {  // columns j < 32 of rows r >= 32: the cross-half product
                        float v[16];
                        tmem_ld16(tq + TM_AP + (j0 < 32 && r >= 32 ? 64 + j0 : j0), v);
                        tmem_wait16(v);
                        const float br = beta_s[r];
#pragma unroll
                        for (int i = 0; i < 16; ++i) x[i] = j0 + i < r ? br * v[i] : 0.f;
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) As[r * AS_LD + j0 + i] = x[i];
                }
                __syncthreads();
            }
            // beside the diagonal inversions, pass 1 stages M (bf16 M^T -> MA, M scaled by
            // gamma in TMEM) on warps 8-15, which own two 64-column slices per quadrant, and
            // with the cache puts P (TMEM lanes 64-127) into GSUM on warps 2, 3, 6, 7
            invert_to_tb<SEG>(As, Ts, Ys, beta_s, smem_u32(sm + Lay::TB), tid, tq, [&](int w) {
                if (!SEG) return;
                if (w >= 8) {
                    const int c0 = 64 * ((w >> 2) - 2);
                    stage_cols<4>(tq + TM_M + c0, sm + Lay::MA, 128, lrow, c0, gam, true);
                    tmem_st_wait();
                } else if (wu_cache && (w & 3) >= 2) {
                    const int j0 = 32 * (w >> 2);  // warps 2, 3: columns 0-31; 6, 7: 32-63
                    extract_p16(tq, lrow - 64, j0, smem_u32(sm + Lay::GSUM));
                    extract_p16(tq, lrow - 64, j0 + 16, smem_u32(sm + Lay::GSUM));
                }
            });
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ============ phase 3: with TB = T diag(beta) and the per-half factors e^{rho_h}:
        //   W^T  = e^{rho_a} (X1k_a)^T TB_a^T + e^{rho_b} (X1k_b)^T TB_b^T  (combined at staging)
        //   U'^T = V^T TB^T
        // X1's k rows serve as an MN-major operand (K rows = tokens, MN blocks 16 KB apart);
        // the v tile is used as TMA wrote it.
        if (tid == 0) {
            tc_fence_after();
            const uint32_t x1 = smem_u32(sm + Lay::X1), tb = smem_u32(sm + Lay::TB),
                           rv = smem_u32(sm + Lay::RV + vbuf * 16384);
            constexpr uint32_t id = idesc_bf16(128, 64, true, false);
#pragma unroll
            for (int s = 0; s < 2; ++s)
                mma_bf16(tmem + TM_W, sdesc(x1 + s * 2048, 16384, 1024), kmajor_desc(tb, 64, s), id,
                         s > 0);
#pragma unroll
            for (int s = 0; s < 2; ++s)
                mma_bf16(tmem + TM_AP, sdesc(x1 + 4096 + s * 2048, 16384, 1024),
                         kmajor_desc(tb, 64, s + 2), id, s > 0);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16(tmem + TM_U, mnmajor_desc(rv, 64, s), kmajor_desc(tb, 64, s), id, s > 0);
            mma_commit(bar);
        }
        // meanwhile: bf16 copy of the state, state scaled by gamma in TMEM.  Slice wg
        // takes columns 32wg..32wg+31 (pass 3: S^T into TMEM; pass 1: B^T into SA).
        if (!SEG) {
            const int c0 = 32 * wg;
            stage_cols_tmem<2>(tq + TM_S + c0, tq + TM_SB + c0 / 2, c0, gam, true);
            tmem_st_wait();
        } else {  // pass 1: bf16 B^T into two free 32-column TMEM ranges (M was staged
                  // beside the inversion)
            const int c0 = 32 * wg;
            stage_cols_tmem<2>(tq + TM_B + c0, tq + sbb_col(c0 >> 4), c0, gam, true);
            tmem_st_wait();
        }
        if (!(ok = wait_mma(bar, parity))) break;
        // The v tile is consumed: the output gate's [64][128] tile (if any) goes into
        // its buffer now, for the epilogue.
        if (gate_on && tid == 0) {
            gate_pending = true;
            mbar_expect_tx(bar_gate, 16384);
            tma_tile(sm + Lay::RV + vbuf * 16384, &maps.gate, 0, h, (int)t0, bar_gate);
        }
        // W^T = e^{rho_a} Wa^T + e^{rho_b} Wb^T (lane = channel c) -> WB (MN-major B
        // operand: K rows = c, MN = token r)
        {
            const int r0 = 16 * wg;  // tokens r0..r0+15 of this thread's channel row
            float wa[16], wbv[16], up[16];
            tmem_ld16(tq + TM_W + r0, wa);
            tmem_ld16(tq + TM_AP + r0, wbv);
            if (SEG && wu_cache) tmem_ld16(tq + TM_U + r0, up);  // U' (before phase 5 changes it)
            tmem_wait16(wa);
            tmem_wait16(wbv);
            const float ea = eha[lrow], eb = ehb[lrow];
            const uint32_t wbs = smem_u32(sm + Lay::WB);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float w[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) w[i] = fmaf(ea, wa[8 * hh + i], eb * wbv[8 * hh + i]);
                st_shared_v4(wbs + mnmajor_chunk_off(lrow, (r0 >> 3) + hh, 128),
                             pack_bf16(w[0], w[1]), pack_bf16(w[2], w[3]), pack_bf16(w[4], w[5]),
                             pack_bf16(w[6], w[7]));
            }
            if (SEG && wu_cache) {  // U'^T (before phase 5 changes it), bf16, next to W^T in UA
                tmem_wait16(up);
                const uint32_t ru = smem_u32(sm + Lay::UA + lrow * 128);
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
                    st_shared_v4(ru + ((((r0 >> 3) + hh) ^ (lrow & 7)) << 4),
                                 pack_bf16(up[8 * hh], up[8 * hh + 1]),
                                 pack_bf16(up[8 * hh + 2], up[8 * hh + 3]),
                                 pack_bf16(up[8 * hh + 4], up[8 * hh + 5]),
                                 pack_bf16(up[8 * hh + 6], up[8 * hh + 7]));
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (wu_cache && tid == 0) {  // W^T, U'^T (WB, UA: 32 KB) and P (GSUM) into the chunk cache
            bulk_store(wu_tile(t0) + CI_W, sm + Lay::WB, 32768);
            bulk_store(wu_tile(t0) + CI_PB, sm + Lay::GSUM, 8192);
            bulk_commit();
        }

        // ============ phase 5: U^T -= S^T W^T ; O^T = S^T Q~^T  (pass 1: U_M^T = -M^T W^T)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t wb = smem_u32(sm + Lay::WB);
            constexpr uint32_t id_neg = idesc_bf16(128, 64, false, true, true);
            if (!SEG) {  // A = bf16 S^T from TMEM
                const uint32_t qt = smem_u32(sm + Lay::QT);
                constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16_ts(tmem + TM_U, tmem + TM_SB + 8 * s, mnmajor_desc(wb, 128, s), id_neg, 1);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16_ts(tmem + TM_O, tmem + TM_SB + 8 * s, kmajor_desc(qt, 64, s), id, s > 0);
            } else {
                const uint32_t ma = smem_u32(sm + Lay::MA);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16_ts(tmem + TM_U, tmem + sbb_col(s), mnmajor_desc(wb, 128, s), id_neg, 1);
#pragma unroll
                for (int s = 0; s < 8; ++s)
                    mma_bf16(tmem + TM_AP, kmajor_desc(ma, 128, s), mnmajor_desc(wb, 128, s), id_neg,
                             s > 0);
            }
            mma_commit(bar);
        }
        if (!(ok = wait_mma(bar, parity))) break;

        // ============ phase 6: bf16 U^T into TMEM as the next products' A operand (pass 1:
        // U_B^T and U_M^T, in the W columns, which W staging has emptied)
        if (!SEG) {
            const int c0 = 16 * wg;
            stage_cols_tmem<1>(tq + TM_U + c0, tq + TM_UB + c0 / 2, c0, nullptr, false);
            tmem_st_wait();
        } else {
            const bool is_m = wg >= 2;
            const int c0 = 32 * (wg & 1);
            stage_cols_tmem<2>(tq + (is_m ? TM_AP : TM_U) + c0, tq + (is_m ? TM_UBM : TM_UBB) + c0 / 2,
                               c0, nullptr, false);
            tmem_st_wait();
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ============ phase 7: O^T += U^T P^T ; S^T += U^T Kdec  (pass 1: B, M updates)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t kd = smem_u32(sm + Lay::KD);
            constexpr uint32_t id_s = idesc_bf16(128, 128, false, true);
            if (!SEG) {  // A = bf16 U^T from TMEM
                const uint32_t pb = smem_u32(sm + Lay::PB);
                constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16_ts(tmem + TM_O, tmem + TM_UB + 8 * s, kmajor_desc(pb, 64, s), id, 1);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16_ts(tmem + TM_S, tmem + TM_UB + 8 * s, mnmajor_desc(kd, 64, s), id_s, 1);
            } else {  // A = bf16 U_B^T, U_M^T from TMEM
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16_ts(tmem + TM_B, tmem + TM_UBB + 8 * s, mnmajor_desc(kd, 64, s), id_s, 1);
#pragma unroll
                for (int s = 0; s < 4; ++s)
                    mma_bf16_ts(tmem + TM_M, tmem + TM_UBM + 8 * s, mnmajor_desc(kd, 64, s), id_s, 1);
            }
            mma_commit(bar);
        }
        if (!(ok = wait_mma(bar, parity))) break;

        if (!SEG) {
            // O^T -> out.  A full chunk is staged as a [64][128] bf16 tile in this chunk's
            // v buffer (dead since phase 3) and written by one TMA store; a partial last
            // chunk is stored from registers, row by row.  With an output gate, the
            // buffer holds the gate tile, and each element is gated in place.
            const int r0 = 16 * wg;
            float v[16];
            tmem_ld16(tq + TM_O + r0, v);
            tmem_wait16(v);
            __nv_bfloat16* os = reinterpret_cast<__nv_bfloat16*>(sm + Lay::RV + vbuf * 16384);
            if (gate_on) {
                if (!(ok = !__syncthreads_or(!mbar_wait(bar_gate, gate_parity, &g_tc_status,
                                                        ERR_WAIT_TIMEOUT)))) break;
                gate_parity ^= 1u;
                gate_pending = false;
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] *= __bfloat162float(os[(r0 + i) * D + lrow]);
            }
            if (Lc == C) {
#pragma unroll
                for (int i = 0; i < 16; ++i) os[(r0 + i) * D + lrow] = __float2bfloat16_rn(v[i]);
                fence_async_smem();
                __syncthreads();
                if (tid == 0) {
                    tma_store_tile(&maps.out, sm + Lay::RV + vbuf * 16384, h, (int)t0);
                    bulk_commit();
                }
            } else {
                __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + (int64_t)h * D + lrow;
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (r0 + i < Lc) out[(t0 + r0 + i) * H * (int64_t)D] = __float2bfloat16_rn(v[i]);
            }
        }
        if (!SEG && snap_on) {  // state snapshot at this chunk end, if one is requested
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

    // ---- results of the segment
    if (!ok) {  // after a timeout: bounded waits for what may still be in flight
        if (tid == 0) {
            mbar_wait(bar, parity ^ 1u, &g_tc_status, ERR_WAIT_TIMEOUT);
            if (gate_pending) mbar_wait(bar_gate, gate_parity, &g_tc_status, ERR_WAIT_TIMEOUT);
        }
        if (tid == raw_tid && raw_pending) mbar_wait(bar_raw, raw_parity, &g_tc_status, ERR_WAIT_TIMEOUT);
    }
    if (tid == 0 && (!SEG || wu_cache)) bulk_wait_all();  // output / cache stores are complete
    if (ok) {
        if (SEG) {  // slices 0-1: B^T, slices 2-3: M^T, 64 columns each
            const bool is_m = wg >= 2;
            const int cb = 64 * (wg & 1);
            float* rowp = a.trans + ((int64_t)u * H + h) * 2 * D * D + (is_m ? D * D : 0) +
                          (int64_t)lrow * D;
            for (int c0 = cb; c0 < cb + 64; c0 += 16) {
                float v[16];
                tmem_ld16(tq + (is_m ? TM_M : TM_B) + c0, v);
                tmem_wait16(v);
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                    *reinterpret_cast<float4*>(rowp + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
            }
        } else if (sg.last && a.s_final) {  // slice wg: columns 32wg..32wg+31 of S^T
            float* sf = a.s_final + ((int64_t)sg.n * H + h) * D * D;
            for (int c0 = 32 * wg; c0 < 32 * wg + 32; c0 += 16) {
                float v[16];
                tmem_ld16(tq + TM_S + c0, v);
                tmem_wait16(v);
#pragma unroll
                for (int i = 0; i < 16; ++i) sf[(int64_t)(c0 + i) * D + lrow] = v[i];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- pass 3 from the chunk cache
// Shared memory: two chunk images (the cache entry as pass 1 wrote it, 1024-byte
// aligned), the output tile and the output gate's tile.
struct LayC {
    static constexpr uint32_t IMG = 0, IMG_STRIDE = 75776;  // kChunkImageBytes rounded to 1 KB
    static constexpr uint32_t OUT = 2 * IMG_STRIDE;         // bf16 [64][128]
    static constexpr uint32_t GATE = OUT + 16384;           // bf16 [64][128]
    static constexpr uint32_t BAR = GATE + 16384;           // mbarriers: MMA, image 0, image 1, gate
    static constexpr uint32_t TMEMP = BAR + 32;
    static constexpr uint32_t BYTES = TMEMP + 16 + 1024;    // + alignment slack
};
static_assert(LayC::IMG_STRIDE >= kChunkImageBytes && LayC::IMG_STRIDE % 1024 == 0, "image stride");
static_assert(LayC::BYTES <= 232448, "shared memory");

// Per (segment, head): the state chain from the true incoming state and the output.
// Per chunk, with its image in shared memory (loaded two chunks ahead):
//   bf16 S^T -> TMEM, S^T *= gamma, U'^T -> the U accumulator        (all threads)
//   U^T -= S^T W^T ;  O^T = S^T Q~^T                                   (one thread)
//   bf16 U^T -> TMEM                                                   (all threads)
//   O^T += U^T P^T ;  S^T += U^T K_dec                                 (one thread)
//   O^T (x gate) -> bf16 tile -> TMA store                             (all threads)
// TMEM columns as in tc_kernel's pass 3.  The same products in the same precision
// as tc_kernel<0>, so the two paths differ only in where W, U', Q~, K_dec, P and
// gamma come from.
__global__ void __launch_bounds__(NT, 1) cached_kernel(TcArgs a, const __grid_constant__ TcMaps maps) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int u = blockIdx.x, h = blockIdx.y, H = a.H;
    if (u >= *a.n_units) return;
    const SegEntry sg = a.segs[u];
    const bool snap_on = a.snap_pool != nullptr;
    const bool gate_on = a.gate != nullptr;
    const int64_t seq_lo = snap_on ? (a.cu ? (int64_t)a.cu[sg.n] : (int64_t)sg.n * a.T) : 0;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + LayC::BAR);  // MMA completion
    uint64_t* bar_img = bar + 1;                                  // [2] image loads
    uint64_t* bar_gate = bar + 3;                                 // output-gate tile
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sm + LayC::TMEMP);
    if (sg.c_base < 0 || sg.c_base + (sg.t_end - sg.t_begin + C - 1) / C > a.total_chunks) {
        if (tid == 0) atomicCAS(&g_tc_status, 0, ERR_SEG_OVERFLOW);  // malformed cu_seqlens
        return;
    }
    auto entry = [&](int64_t tt) {  // the chunk cache entry of the chunk at tt, head h
        return a.wu + ((sg.c_base + (tt - sg.t_begin) / C) * H + h) * (int64_t)kChunkImageBytes;
    };
    uint32_t pending = 0;  // thread 0: bit b = a load into image b in flight; bit 2 = gate tile
    auto load_img = [&](int64_t tt, int b) {
        pending |= 1u << b;
        mbar_expect_tx(bar_img + b, (uint32_t)kChunkImageBytes);
        bulk_load(sm + LayC::IMG + b * LayC::IMG_STRIDE, entry(tt), (uint32_t)kChunkImageBytes,
                  bar_img + b);
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
    bool ok = true;
    int b = 0;
    int64_t last_t0 = sg.t_begin;  // the chunk whose output is still in TMEM
    int last_Lc = 0;
    uint32_t last_o = TM_O;
    for (int64_t t0 = sg.t_begin; t0 < sg.t_end && ok; t0 += C, b ^= 1) {
        const int Lc = (int)((sg.t_end - t0) < C ? (sg.t_end - t0) : C);
        uint8_t* img = sm + LayC::IMG + b * LayC::IMG_STRIDE;
        // O accumulators alternate between chunks, so a chunk's output leaves TMEM while
        // the next chunk's first products run
        const uint32_t tm_o = (((t0 - sg.t_begin) / C) & 1) ? TM_O2 : TM_O;
        if (!(ok = !__syncthreads_or(!mbar_wait(bar_img + b, (img_parity >> b) & 1u, &g_tc_status,
                                                ERR_WAIT_TIMEOUT)))) break;
        img_parity ^= 1u << b;
        pending &= ~(1u << b);
        // bf16 S^T into TMEM (A operand), S^T *= gamma in place; U'^T into the U accumulator
        {
            const float* gam = reinterpret_cast<const float*>(img + CI_GAM);
            const int c0 = 32 * wg, r0 = 16 * wg;
            stage_cols_tmem<2>(tq + TM_S + c0, tq + TM_SB + c0 / 2, c0, gam, true);
            const uint8_t* ru = img + CI_U + lrow * 128;
            float v[16];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint4 x = *reinterpret_cast<const uint4*>(ru + ((((r0 >> 3) + hh) ^ (lrow & 7)) << 4));
                float lo4[4], hi4[4];
                unpack_bf16x4(make_uint2(x.x, x.y), lo4);
                unpack_bf16x4(make_uint2(x.z, x.w), hi4);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    v[8 * hh + i] = lo4[i];
                    v[8 * hh + 4 + i] = hi4[i];
                }
            }
            tmem_st16(tq + TM_U + r0, v);
            tmem_st_wait();
        }
        tc_fence_before();
        __syncthreads();
        // U^T -= S^T W^T ; O^T = S^T Q~^T
        if (tid == 0) {
            tc_fence_after();
            const uint32_t wb = smem_u32(img + CI_W), qt = smem_u32(img + CI_QT);
            constexpr uint32_t id_neg = idesc_bf16(128, 64, false, true, true);
            constexpr uint32_t id = idesc_bf16(128, 64, false, false);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16_ts(tmem + TM_U, tmem + TM_SB + 8 * s, mnmajor_desc(wb, 128, s), id_neg, 1);
#pragma unroll
            for (int s = 0; s < 8; ++s)
                mma_bf16_ts(tmem + tm_o, tmem + TM_SB + 8 * s, kmajor_desc(qt, 64, s), id, s > 0);
            mma_commit(bar);
            mma_out = true;
            mma_par = parity;
        }
        // meanwhile: the previous chunk's output (a full chunk: only a segment's last is partial)
        if (t0 > sg.t_begin && !(ok = emit(t0 - C, C, last_o))) break;
        if (!(ok = wait_mma(bar, parity))) break;
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
            const uint32_t pb = smem_u32(img + CI_PB), kd = smem_u32(img + CI_KD);
            constexpr uint32_t id = idesc_bf16(128, 64, false, false);
            constexpr uint32_t id_s = idesc_bf16(128, 128, false, true);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16_ts(tmem + tm_o, tmem + TM_UB + 8 * s, kmajor_desc(pb, 64, s), id, 1);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                mma_bf16_ts(tmem + TM_S, tmem + TM_UB + 8 * s, mnmajor_desc(kd, 64, s), id_s, 1);
            mma_commit(bar);
            mma_out = true;
            mma_par = parity;
        }
        if (!(ok = wait_mma(bar, parity))) break;
        mma_out = false;
        // this image is consumed: the chunk after next may load into it
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
        int x = g;
        long long xc = nch;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            const long long yc = __shfl_up_sync(0xffffffffu, xc, o);
            if (lane >= o) {
                x += y;
                xc += yc;
            }
        }
        if (lane == 31) {
            warp_sums[warp] = x;
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
        const int excl = carry + x - g + (warp > 0 ? warp_sums[warp - 1] : 0);
        const int64_t cexcl = carry_c + xc - nch + (warp > 0 ? warp_csums[warp - 1] : 0);
        if (n < N) {
            seg_off[n] = excl;
            for (int j = 0; j < g; ++j) {
                const int uidx = excl + j;
                if (uidx >= max_units) {
                    atomicCAS(&g_tc_status, 0, ERR_SEG_OVERFLOW);
                    break;
                }
                SegEntry e;
                e.n = n;
                e.j = j;
                e.t_begin = lo + (int64_t)j * seg_chunks * C;
                const int64_t end = lo + (int64_t)(j + 1) * seg_chunks * C;
                e.t_end = end < hi ? end : hi;
                e.last = (j == g - 1) ? 1 : 0;
                e.pad = 0;
                e.c_base = cexcl + (int64_t)j * seg_chunks;
                segs[uidx] = e;
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

size_t tc_smem_bytes() { return LayT<false>::BYTES; }

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

cudaError_t tc_take_status(int* code) {
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_tc_status, sizeof(int));
    if (e == cudaSuccess && *code) e = cudaMemcpyToSymbol(g_tc_status, &zero, sizeof(int));
    return e;
}

cudaError_t launch_tc(const TcArgs& a, const TcPlan& p, cudaStream_t stream, int* launches,
                      bool from_cache) {
    static bool attr_set[kMaxDevices][2] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices || !attr_set[dev][0]) {
        err = cudaFuncSetAttribute(tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)LayT<false>::BYTES);
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(cached_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)LayC::BYTES);
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(seg_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       SCAN_SMEM);
        if (err == cudaSuccess)
            err = cudaFuncSetAttribute(tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)LayT<true>::BYTES);
        if (err != cudaSuccess) return err;
        if (dev < kMaxDevices) attr_set[dev][0] = true;
    }
    TcMaps maps;
    memset(&maps, 0, sizeof maps);
    const int64_t tokens = (int64_t)a.B * a.T;
    if (tokens > 0) {
        if ((err = tile_map(&maps.q, a.q, false, a.H, tokens, false)) != cudaSuccess ||
            (err = tile_map(&maps.k, a.k, false, a.H, tokens, false)) != cudaSuccess ||
            (err = tile_map(&maps.v, a.v, false, a.H, tokens, true)) != cudaSuccess ||
            (err = tile_map(&maps.la, a.log_alpha, true, a.H, tokens, false)) != cudaSuccess ||
            (err = tile_map(&maps.out, a.out, false, a.H, tokens, false)) != cudaSuccess ||
            (err = tile_map(&maps.gate, a.gate ? a.gate : a.out, false, a.H, tokens, false)) !=
                cudaSuccess)
            return err;
    }
    const dim3 grid((unsigned)p.max_units, (unsigned)a.H);
    if (!from_cache) {  // else the segment table, transitions and W/U' cache are in place
        profile_mark(SLOT_SETUP, true, stream);
        seg_setup_kernel<<<1, 1024, 0, stream>>>(a.cu, a.N, a.T, p.seg_chunks, p.max_units, a.segs,
                                                 a.seg_off, a.n_units);
        profile_mark(SLOT_SETUP, false, stream);
        *launches += 1;
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    if (p.segmented) {
        if (!from_cache) {
            profile_mark(SLOT_PASS1, true, stream);
            tc_kernel<1><<<grid, NT, LayT<true>::BYTES, stream>>>(a, maps);
            profile_mark(SLOT_PASS1, false, stream);
            *launches += 1;
            if ((err = cudaGetLastError()) != cudaSuccess) return err;
        }
        profile_mark(SLOT_SCAN, true, stream);
        seg_scan_kernel<<<dim3((unsigned)a.N, (unsigned)a.H, D / SCAN_ROWS), 256, SCAN_SMEM, stream>>>(a);
        profile_mark(SLOT_SCAN, false, stream);
        *launches += 1;
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    profile_mark(SLOT_PASS3, true, stream);
    if (a.wu)
        cached_kernel<<<grid, NT, LayC::BYTES, stream>>>(a, maps);
    else
        tc_kernel<0><<<grid, NT, LayT<false>::BYTES, stream>>>(a, maps);
    profile_mark(SLOT_PASS3, false, stream);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_transition(const TcArgs& a_in, const TcPlan& p, float* out, cudaStream_t stream,
                              int* launches) {
    TcArgs a = a_in;
    a.trans_all = 1;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices || !attr_set[dev]) {
        err = cudaFuncSetAttribute(tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)LayT<true>::BYTES);
        if (err != cudaSuccess) return err;
        if (dev < kMaxDevices) attr_set[dev] = true;
    }
    TcMaps maps;
    memset(&maps, 0, sizeof maps);
    const int64_t tokens = (int64_t)a.B * a.T;
    if (tokens > 0) {
        if ((err = tile_map(&maps.k, a.k, false, a.H, tokens, false)) != cudaSuccess ||
            (err = tile_map(&maps.v, a.v, false, a.H, tokens, true)) != cudaSuccess ||
            (err = tile_map(&maps.la, a.log_alpha, true, a.H, tokens, false)) != cudaSuccess ||
            (a.wu && (err = tile_map(&maps.q, a.q, false, a.H, tokens, false)) != cudaSuccess))
            return err;
    }
    profile_mark(SLOT_SETUP, true, stream);
    seg_setup_kernel<<<1, 1024, 0, stream>>>(a.cu, a.N, a.T, p.seg_chunks, p.max_units, a.segs,
                                             a.seg_off, a.n_units);
    profile_mark(SLOT_SETUP, false, stream);
    *launches += 1;
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    profile_mark(SLOT_PASS1, true, stream);
    tc_kernel<1><<<dim3((unsigned)p.max_units, (unsigned)a.H), NT, LayT<true>::BYTES, stream>>>(
        a, maps);
    profile_mark(SLOT_PASS1, false, stream);
    *launches += 1;
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
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

}  // namespace kda
