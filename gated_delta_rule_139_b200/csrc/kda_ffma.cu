// kda_ffma.cu -- chunkwise KDA forward on CUDA cores (fp32 FFMA arithmetic).
//
// This is the precision path: fp32 inputs need max |error| <= 1e-4, which the
// bf16/tf32 tensor-core operands cannot give, so every product here is an fp32
// FFMA.  It also accepts bf16 q/k/v (widened exactly) and serves as the generic
// path for shapes the tensor-core path does not take.
//
// Method (aiblin.ru, "Kimi K3 -- открытая модель, которая обошла закрытых
// лидеров рынка", section "Как распараллелили последовательное обновление"):
// the tokens of a 64-token chunk are processed together, then the state is
// passed to the next chunk.  Per chunk with incoming state S0, g = inclusive
// cumulative sum of the clamped log-gates inside the chunk (per key channel):
//   A  = strict_lower(diag(beta) (K*e^g) (K*e^-g)^T)
//   [W | U'] = (I + A)^-1 [diag(beta) K*e^g | diag(beta) V]
//   U  = U' - W S0
//   O  = (Q*e^g) S0 + lower_incl_diag((Q*e^g)(K*e^-g)^T) U
//   S  = Diag(e^{g_last}) S0 + (K*e^{g_last-g})^T U
// The in-chunk product of alpha and its inverse (e^{+-g}) leave the fp32 range
// at the clamp floor (e^{-+320} over 64 tokens), which the section "Как
// хранить миллион токенов в памяти" of the same page warns about.  So every
// factor is referenced to the start of its 16-token block (rho_I = g before
// block I): within a block |g - rho_I| <= 80 < ln(FLT_MAX); across blocks the
// factors are e^{rho_I - rho_J} <= 1 (J < I), whose underflow to 0 is the
// correct limit.
//
// Work decomposition: one CTA of 256 threads per (sequence, head, 32-column
// slice of d_v).  The CTA walks the chunks of its sequence in order; the state
// slice S[:, dv0:dv0+32] stays in shared memory for the whole sequence.
#include <cuda_bf16.h>

#include "kda_internal.h"

namespace kda {
namespace {

constexpr int C = kChunk;
constexpr int NT = 256;
constexpr int DVB = 32;  // state columns per CTA

template <int DK>
struct Smem {
    static constexpr int KS = DK + 1;        // padded row stride of the chunk tiles
    static constexpr int XS = DK + DVB + 1;  // padded row stride of [W | U]
    static constexpr int AS = C + 1;
    static constexpr int kt = 0;                  // C*KS: k*e^{g-rho}
    static constexpr int qt = kt + C * KS;        // C*KS: q*e^{g-rho} -> q*e^{g}
    static constexpr int kh = qt + C * KS;        // C*KS: g -> k*e^{rho-g} -> k*e^{g_last-g}
    static constexpr int vs = kh + C * KS;        // C*DVB
    static constexpr int bs = vs + C * DVB;       // C
    static constexpr int as = bs + C;             // C*AS: diag(beta) strict-lower A
    static constexpr int ps = as + C * AS;        // C*AS: lower-incl-diag P
    static constexpr int xs = ps + C * AS;        // C*XS: [W | U'] then [W | U]
    static constexpr int ss = xs + C * XS;        // DK*DVB: state slice
    static constexpr int rho = ss + DK * DVB;     // 4*DK: g before each 16-token block
    static constexpr int erho = rho + 4 * DK;     // 4*DK: e^{rho_I}
    static constexpr int drho = erho + 4 * DK;    // 4*DK: e^{g_last - rho_I}
    static constexpr int fij = drho + 4 * DK;     // 6*DK: e^{rho_I - rho_J}, J < I
    static constexpr int gam = fij + 6 * DK;      // DK: e^{g_last}
    static constexpr int total = gam + DK;
    static constexpr size_t bytes = sizeof(float) * total;
};

template <bool BF16>
__device__ __forceinline__ float ld_in(const void* p, int64_t i) {
    if constexpr (BF16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    else
        return reinterpret_cast<const float*>(p)[i];
}

template <bool BF16>
__device__ __forceinline__ void st_out(void* p, int64_t i, float x) {
    if constexpr (BF16)
        reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
    else
        reinterpret_cast<float*>(p)[i] = x;
}

// index of pair (I, J), J < I, in the e^{rho_I - rho_J} table
__device__ __forceinline__ int pair_index(int I, int J) { return I * (I - 1) / 2 + J; }

template <bool BF16, int DK>
__device__ __forceinline__ void chunk_step(const FwdArgs& a, float* sm, int64_t t0, int Lc,
                                           int h, int dv0) {
    using L = Smem<DK>;
    constexpr int KS = L::KS, XS = L::XS, AS = L::AS;
    const int tid = threadIdx.x;
    const int H = a.H, DV = a.dv;
    float* Kt = sm + L::kt;
    float* Qt = sm + L::qt;
    float* Kh = sm + L::kh;
    float* V = sm + L::vs;
    float* Bv = sm + L::bs;
    float* A = sm + L::as;
    float* P = sm + L::ps;
    float* X = sm + L::xs;
    float* S = sm + L::ss;
    float* Rho = sm + L::rho;
    float* ERho = sm + L::erho;
    float* DRho = sm + L::drho;
    float* Fij = sm + L::fij;
    float* Gam = sm + L::gam;

    // 1. load the chunk; rows past the sequence end are the identity step
    //    (k = q = v = 0, beta = 0, log alpha = 0)
    for (int i = tid; i < C * DK; i += NT) {
        const int r = i / DK, c = i % DK;
        float kv = 0.f, qv = 0.f, g = 0.f;
        if (r < Lc) {
            const int64_t gi = ((t0 + r) * H + h) * (int64_t)DK + c;
            kv = ld_in<BF16>(a.k, gi);
            qv = ld_in<BF16>(a.q, gi);
            g = fminf(fmaxf(a.log_alpha[gi], -5.f), 0.f);
        }
        Kt[r * KS + c] = kv;
        Qt[r * KS + c] = qv;
        Kh[r * KS + c] = g;
    }
    for (int i = tid; i < C * DVB; i += NT) {
        const int r = i / DVB, e = i % DVB;
        V[r * DVB + e] = r < Lc ? ld_in<BF16>(a.v, ((t0 + r) * H + h) * (int64_t)DV + dv0 + e) : 0.f;
    }
    for (int r = tid; r < C; r += NT) Bv[r] = r < Lc ? a.beta[(t0 + r) * H + h] : 0.f;
    __syncthreads();

    // 2. inclusive cumulative sum of the clamped log-gates, per key channel
    if (tid < DK) {
        const int c = tid;
        float acc = 0.f;
        for (int r = 0; r < C; ++r) {
            if ((r & 15) == 0) Rho[(r >> 4) * DK + c] = acc;
            acc += Kh[r * KS + c];
            Kh[r * KS + c] = acc;
        }
        for (int I = 0; I < 4; ++I) {
            const float rI = Rho[I * DK + c];
            ERho[I * DK + c] = expf(rI);
            DRho[I * DK + c] = expf(acc - rI);
            for (int J = 0; J < I; ++J) Fij[pair_index(I, J) * DK + c] = expf(rI - Rho[J * DK + c]);
        }
        Gam[c] = expf(acc);
    }
    __syncthreads();

    // 3. block-referenced factors: Kt = k e^{g-rho}, Qt = q e^{g-rho}, Kh = k e^{rho-g}
    for (int i = tid; i < C * DK; i += NT) {
        const int r = i / DK, c = i % DK;
        const float d = Kh[r * KS + c] - Rho[(r >> 4) * DK + c];  // in [-80, 0]
        const float e1 = expf(d), e2 = expf(-d);
        const float kv = Kt[r * KS + c];
        Kt[r * KS + c] = kv * e1;
        Qt[r * KS + c] *= e1;
        Kh[r * KS + c] = kv * e2;
    }
    __syncthreads();

    // 4. A (times beta_r, strict lower) and P (lower incl. diagonal).
    //    Work item (I, j): column j against the 16 rows of block I, j < 16(I+1).
    //    Items 0..15 -> I=0, 16..47 -> I=1, 48..95 -> I=2, 96..159 -> I=3.
    for (int item = tid; item < 160; item += NT) {
        const int I = item < 16 ? 0 : item < 48 ? 1 : item < 96 ? 2 : 3;
        const int j = item - (I == 0 ? 0 : I == 1 ? 16 : I == 2 ? 48 : 96);
        const int J = j >> 4;
        float accA[16], accP[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) accA[rr] = accP[rr] = 0.f;
        const float* fcol = J < I ? Fij + pair_index(I, J) * DK : nullptr;
        for (int c = 0; c < DK; ++c) {
            float f = Kh[j * KS + c];
            if (fcol) f *= fcol[c];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
                const int r = 16 * I + rr;
                accA[rr] = fmaf(Kt[r * KS + c], f, accA[rr]);
                accP[rr] = fmaf(Qt[r * KS + c], f, accP[rr]);
            }
        }
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
            const int r = 16 * I + rr;
            if (r > j) A[r * AS + j] = Bv[r] * accA[rr];
            if (r >= j) P[r * AS + j] = accP[rr];
        }
    }
    __syncthreads();

    // 5. forward substitution (I + A) X = [diag(beta) k e^{g} | diag(beta) V],
    //    one thread per right-hand-side column; X = [W | U']
    if (tid < DK + DVB) {
        const int col = tid;
        float x[C];
#pragma unroll
        for (int r = 0; r < C; ++r) {
            float acc = col < DK ? Bv[r] * Kt[r * KS + col] * ERho[(r >> 4) * DK + col]
                                 : Bv[r] * V[r * DVB + (col - DK)];
#pragma unroll
            for (int j = 0; j < r; ++j) acc = fmaf(-A[r * AS + j], x[j], acc);
            x[r] = acc;
            X[r * XS + col] = acc;
        }
    }
    __syncthreads();

    // 6. chunk-start references: Qt -> q e^{g}; Kh -> k e^{g_last - g}
    for (int i = tid; i < C * DK; i += NT) {
        const int r = i / DK, c = i % DK;
        Qt[r * KS + c] *= ERho[(r >> 4) * DK + c];
        Kh[r * KS + c] *= DRho[(r >> 4) * DK + c];
    }
    // 7. U = U' - W S0 (each thread owns rows rg*8.. of column e)
    const int e = tid & 31, grp = tid >> 5;
#pragma unroll 1
    for (int rr = 0; rr < 8; ++rr) {
        const int r = grp * 8 + rr;
        float acc = X[r * XS + DK + e];
        for (int c = 0; c < DK; ++c) acc = fmaf(-X[r * XS + c], S[c * DVB + e], acc);
        X[r * XS + DK + e] = acc;
    }
    __syncthreads();

    // 8. O = (q e^g) S0 + P U
#pragma unroll 1
    for (int rr = 0; rr < 8; ++rr) {
        const int r = grp * 8 + rr;
        if (r >= Lc) continue;
        float acc = 0.f;
        for (int c = 0; c < DK; ++c) acc = fmaf(Qt[r * KS + c], S[c * DVB + e], acc);
        for (int j = 0; j <= r; ++j) acc = fmaf(P[r * AS + j], X[j * XS + DK + e], acc);
        const int64_t oi = ((t0 + r) * H + h) * (int64_t)DV + dv0 + e;
        if (a.gate) acc *= ld_in<BF16>(a.gate, oi);  // output gate
        st_out<BF16>(a.out, oi, acc);
    }
    __syncthreads();

    // 9. S = Diag(e^{g_last}) S0 + (k e^{g_last - g})^T U
    constexpr int CPG = DK / 8;
#pragma unroll 1
    for (int cc = 0; cc < CPG; ++cc) {
        const int c = grp * CPG + cc;
        float acc = Gam[c] * S[c * DVB + e];
        for (int r = 0; r < C; ++r) acc = fmaf(Kh[r * KS + c], X[r * XS + DK + e], acc);
        S[c * DVB + e] = acc;
    }
    __syncthreads();
}

template <bool BF16, int DK>
__global__ void __launch_bounds__(NT, 1) kda_ffma_kernel(FwdArgs a) {
    using L = Smem<DK>;
    extern __shared__ float sm[];
    const int tid = threadIdx.x;
    const int n = blockIdx.x / a.H, h = blockIdx.x % a.H;
    const int dv0 = blockIdx.y * DVB;
    const int H = a.H, DV = a.dv;
    int64_t lo, hi;
    if (a.cu) {
        lo = a.cu[n];
        hi = a.cu[n + 1];
    } else {
        lo = (int64_t)n * a.T;
        hi = lo + a.T;
    }
    float* S = sm + L::ss;
    const int64_t sbase = ((int64_t)n * H + h) * DK * (int64_t)DV + dv0;
    for (int i = tid; i < DK * DVB; i += NT) {
        const int c = i / DVB, e = i % DVB;
        S[i] = a.s0 ? a.s0[sbase + (int64_t)c * DV + e] : 0.f;
    }
    __syncthreads();
    for (int64_t t0 = lo; t0 < hi; t0 += C) {
        const int Lc = (int)(hi - t0 < C ? hi - t0 : C);
        chunk_step<BF16, DK>(a, sm, t0, Lc, h, dv0);
        const int64_t pos = t0 + Lc - lo;  // tokens of the sequence done so far
        if (a.snap_pool && pos % a.snap_interval == 0 && pos / a.snap_interval <= a.snap_max) {
            const int slot = a.snap_slots[(int64_t)n * a.snap_max + pos / a.snap_interval - 1];
            if (slot >= a.snap_num_slots) {
                if (tid == 0) atomicCAS(a.status, 0, ERR_BAD_SLOT);
            } else if (slot >= 0) {
                float* sp = a.snap_pool + ((int64_t)slot * H + h) * DK * (int64_t)DV + dv0;
                for (int i = tid; i < DK * DVB; i += NT) {
                    const int c = i / DVB, e = i % DVB;
                    sp[(int64_t)c * DV + e] = S[i];
                }
            }
        }
    }
    if (a.s_final) {
        for (int i = tid; i < DK * DVB; i += NT) {
            const int c = i / DVB, e = i % DVB;
            a.s_final[sbase + (int64_t)c * DV + e] = S[i];
        }
    }
}

template <bool BF16, int DK>
cudaError_t launch_t(const FwdArgs& a, cudaStream_t stream) {
    using L = Smem<DK>;
    auto kern = kda_ffma_kernel<BF16, DK>;
    static bool attr_set[kMaxDevices] = {};  // per template instance and device
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices || !attr_set[dev]) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes);
        if (err != cudaSuccess) return err;
        if (dev < kMaxDevices) attr_set[dev] = true;
    }
    dim3 grid((unsigned)(a.N * a.H), (unsigned)(a.dv / DVB));
    profile_mark(SLOT_FFMA, true, stream);
    kern<<<grid, NT, L::bytes, stream>>>(a);
    profile_mark(SLOT_FFMA, false, stream);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffma(const FwdArgs& a, cudaStream_t stream, int* launches) {
    if (a.N * (int64_t)a.H == 0) return cudaSuccess;
    *launches += 1;
    if (a.bf16) {
        return a.dk == 128 ? launch_t<true, 128>(a, stream) : launch_t<true, 64>(a, stream);
    }
    return a.dk == 128 ? launch_t<false, 128>(a, stream) : launch_t<false, 64>(a, stream);
}

}  // namespace kda
