// kda_decode.cu -- a few new tokens per sequence on a resident KDA state.
//
// The per-token rewrite of the state (aiblin.ru, "Kimi K3 -- открытая модель,
// которая обошла закрытых лидеров рынка", section "Как хранить миллион токенов в
// памяти": partial erase, then write, with write strength beta and forget gate
// alpha clamped to [e^-5, 1]) applied to T_new = 1..16 tokens that follow a state
// kept between calls -- the step a decoder or a speculative-decoding verifier
// takes.  Per token, for every state column:
//     S <- Diag(alpha_t) S;  p = S^T k_t;  S <- S + beta_t k_t (v_t - p)^T;  o_t = S^T q_t
// The state is read once and written once; the path is bound by that traffic
// (64 KB of fp32 state per head and direction at d = 128).
//
// One CTA per (sequence, head, 64 state columns) with d_k * 64 / 32 threads;
// each thread keeps an 8-row x 4-column tile of the state in registers for all
// the tokens.  The lanes of a warp lie across 256-byte row pieces, so every
// state access is a coalesced float4 per lane.  Per token, each thread reads its rows'
// (alpha, k, q) as broadcast float4s from shared memory; the two reductions
// over d_k (S^T k and S^T q) combine per-row-group partial sums through shared
// memory.  An optional output gate (precomputed by the caller) multiplies o
// before it is stored.  The token inputs arrive by cp.async, 4 tokens per
// block (2 for fp32 inputs) and two blocks in flight, issued before the state
// loads so that both latencies overlap.
// Optionally the state after every token is written out (a verifier that
// accepts only a prefix of the drafted tokens rolls back to one of them), and
// sequences may address their state through a slot table into a state pool.
#include <cuda_bf16.h>

#include "kda_internal.h"

namespace kda {
namespace {

template <bool BF16>
__device__ __forceinline__ void st_x(void* p, int64_t i, float x) {
    if constexpr (BF16)
        reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
    else
        reinterpret_cast<float*>(p)[i] = x;
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(
                     (uint32_t)__cvta_generic_to_shared(dst)),
                 "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;\n" ::: "memory"); }

template <bool BF16>
__device__ __forceinline__ float raw_x(const unsigned char* p, int i) {
    if constexpr (BF16)
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    else
        return reinterpret_cast<const float*>(p)[i];
}

// A CTA owns DVC = 64 columns of one head's state (grid.y = d_v / 64): half a
// d_v = 128 state, so that four CTAs fit an SM and one's memory phases overlap
// another's arithmetic.
template <bool BF16, int DK, int DVC>
struct DecodeShape {
    static constexpr int CW = DVC / 4;    // lanes across the CTA's columns of one row (4 each)
    static constexpr int RGS = DK / 8;    // row groups of 8 rows
    static constexpr int NTH = RGS * CW;  // threads: d_k * d_v / 32
    static constexpr int TB = BF16 ? 4 : 2;  // tokens per staged block (static shared memory)
};

template <bool BF16, int DK, int DVC>
__global__ void __launch_bounds__(DecodeShape<BF16, DK, DVC>::NTH,
                                  1024 / DecodeShape<BF16, DK, DVC>::NTH)
    decode_kernel(DecodeArgs a) {
    using Sh = DecodeShape<BF16, DK, DVC>;
    constexpr int CW = Sh::CW, RGS = Sh::RGS, NTH = Sh::NTH, TB = Sh::TB;
    constexpr int ES = BF16 ? 2 : 4;  // bytes per q/k/v element
    // raw bytes of one token as it arrives: k | q | v | log_alpha [| gate], in
    // 16-byte chunks
    constexpr int CK = DK * ES / 16, CV = DVC * ES / 16, CL = DK * 4 / 16;
    constexpr int CH = 2 * CK + CV + CL;
    constexpr int RAWB = (CH + CV) * 16;
    // Raw token blocks arrive by cp.async, two blocks in flight; each block is
    // then widened to fp32: tok[t][r] = {alpha_r, k_r, q_r, 0} with
    // alpha = exp(clamp(log_alpha)), read by a warp as one broadcast float4.
    __shared__ __align__(16) unsigned char raw[2][TB][RAWB];
    __shared__ float raw_beta[2][TB];
    __shared__ __align__(16) float4 tok[TB][DK];
    __shared__ float vs[TB][DVC];
    __shared__ float gs[TB][DVC];  // output gate (when given)
    __shared__ float bs[TB];
    __shared__ __align__(16) float red[2][RGS][DVC];  // per-row-group partial sums
    __shared__ __align__(16) float us[DVC];          // u = beta (v - S^T k) of the token
    const int tid = threadIdx.x;
    const int rgrp = tid / CW, cq = tid % CW;  // rows 8 rgrp .. +7, columns 4 cq .. +3
    const int nh = blockIdx.x, n = nh / a.H, h = nh % a.H, H = a.H, T = a.T;
    const int DV = a.dv, c_off = DVC * blockIdx.y;  // row length; this CTA's first column
    int slot = n;
    if (a.slots) {
        slot = a.slots[n];
        if (slot == -1) return;  // padding entry: nothing is read or written
        if (slot < 0 || slot >= a.num_slots) {
            if (tid == 0) atomicCAS(a.status, 0, ERR_BAD_SLOT);
            return;
        }
    }
    const int nblk = (T + TB - 1) / TB;
    const int ch = CH + (a.gate ? CV : 0);  // chunks per token
    // issue the raw copies of token block b into buffer b & 1 (one commit group)
    auto issue = [&](int b) {
        const int t0 = b * TB, nt = min(TB, T - t0);
        for (int x = tid; x < nt * ch; x += NTH) {
            const int t = x / ch, c = x - t * ch;
            const int64_t row = ((int64_t)n * T + t0 + t) * H + h;
            const unsigned char* src;
            if (c < CK)
                src = (const unsigned char*)a.k + (row * DK) * ES + c * 16;
            else if (c < 2 * CK)
                src = (const unsigned char*)a.q + (row * DK) * ES + (c - CK) * 16;
            else if (c < 2 * CK + CV)
                src = (const unsigned char*)a.v + (row * DV + c_off) * ES + (c - 2 * CK) * 16;
            else if (c < CH)
                src = (const unsigned char*)(a.log_alpha + row * DK) + (c - 2 * CK - CV) * 16;
            else
                src = (const unsigned char*)a.gate + (row * DV + c_off) * ES + (c - CH) * 16;
            cp_async16(&raw[b & 1][t][c * 16], src);
        }
        if (tid < nt) cp_async4(&raw_beta[b & 1][tid], a.beta + ((int64_t)n * T + t0 + tid) * H + h);
    };
    if (nblk > 0) issue(0);
    cp_async_commit();
    if (nblk > 1) issue(1);
    cp_async_commit();

    // the thread's 8 x 4 tile of the state; a warp covers whole 512-byte rows
    float* st = a.state + ((int64_t)slot * H + h) * DK * DV + (int64_t)(8 * rgrp) * DV + c_off + 4 * cq;
    float4 s[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i] = *reinterpret_cast<const float4*>(st + i * DV);

    for (int b = 0; b < nblk; ++b) {
        const int t0 = b * TB, nt = min(TB, T - t0), buf = b & 1;
        cp_async_wait_1();  // block b has landed (block b+1 may still be in flight)
        __syncthreads();
        const int per_tok = DK + (a.gate ? 2 : 1) * DVC;
        for (int x = tid; x < nt * per_tok; x += NTH) {
            const int t = x / per_tok, e = x - t * per_tok;
            const unsigned char* r = raw[buf][t];
            if (e < DK) {
                const float la = reinterpret_cast<const float*>(r + (2 * CK + CV) * 16)[e];
                tok[t][e] = make_float4(expf(fminf(fmaxf(la, -5.f), 0.f)), raw_x<BF16>(r, e),
                                        raw_x<BF16>(r + CK * 16, e), 0.f);
            } else if (e < DK + DVC) {
                vs[t][e - DK] = raw_x<BF16>(r + 2 * CK * 16, e - DK);
            } else {
                gs[t][e - DK - DVC] = raw_x<BF16>(r + CH * 16, e - DK - DVC);
            }
        }
        if (tid < nt) bs[tid] = raw_beta[buf][tid];
        __syncthreads();  // raw[buf] consumed; tok/vs/bs ready
        if (b + 2 < nblk) issue(b + 2);
        cp_async_commit();
        // decay of token t, then its partial p = S^T k over the thread's 8 rows -> red[0]
        auto decay_p = [&](int t) {
            const float4* tk = tok[t] + 8 * rgrp;
            float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 x = tk[i];
                s[i].x *= x.x;
                s[i].y *= x.x;
                s[i].z *= x.x;
                s[i].w *= x.x;
                p.x = fmaf(s[i].x, x.y, p.x);
                p.y = fmaf(s[i].y, x.y, p.y);
                p.z = fmaf(s[i].z, x.y, p.z);
                p.w = fmaf(s[i].w, x.y, p.w);
            }
            *reinterpret_cast<float4*>(&red[0][rgrp][4 * cq]) = p;
        };
        // o of token t from the row-group partials in red[1] (threads tid < d_v)
        auto out_o = [&](int t) {
            float acc = 0.f;
#pragma unroll
            for (int g = 0; g < RGS; ++g) acc += red[1][g][tid];
            const int64_t oi = (((int64_t)n * T + t0 + t) * H + h) * DV + c_off + tid;
            if (a.gate) acc *= gs[t][tid];  // output gate
            st_x<BF16>(a.out, oi, acc);
        };
        // Two barriers per token: token t's rank-1 update and partial o share a phase
        // with token t+1's decay and partial p, and o(t) is reduced beside u(t+1).
        decay_p(0);
        for (int t = 0; t < nt; ++t) {
            __syncthreads();  // red[0] (p of t) and red[1] (o of t-1) complete
            if (tid < DVC) {
                float acc = 0.f;
#pragma unroll
                for (int g = 0; g < RGS; ++g) acc += red[0][g][tid];
                us[tid] = bs[t] * (vs[t][tid] - acc);
                if (t > 0) out_o(t - 1);
            }
            __syncthreads();  // us complete; red[0], red[1] consumed
            // rank-1 update, then partial o = S^T q -> red[1]
            const float4* tk = tok[t] + 8 * rgrp;
            const float4 u = *reinterpret_cast<const float4*>(&us[4 * cq]);
            float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 x = tk[i];
                s[i].x = fmaf(x.y, u.x, s[i].x);
                s[i].y = fmaf(x.y, u.y, s[i].y);
                s[i].z = fmaf(x.y, u.z, s[i].z);
                s[i].w = fmaf(x.y, u.w, s[i].w);
                o.x = fmaf(s[i].x, x.z, o.x);
                o.y = fmaf(s[i].y, x.z, o.y);
                o.z = fmaf(s[i].z, x.z, o.z);
                o.w = fmaf(s[i].w, x.z, o.w);
            }
            *reinterpret_cast<float4*>(&red[1][rgrp][4 * cq]) = o;
            if (a.token_states) {  // the state after token t0 + t
                float* ts = a.token_states + (((int64_t)n * T + t0 + t) * H + h) * DK * DV +
                            (int64_t)(8 * rgrp) * DV + c_off + 4 * cq;
#pragma unroll
                for (int i = 0; i < 8; ++i) *reinterpret_cast<float4*>(ts + i * DV) = s[i];
            }
            if (t + 1 < nt) decay_p(t + 1);
        }
        __syncthreads();  // red[1] holds the partials of the block's last token
        if (tid < DVC) out_o(nt - 1);
        // the next block's staging begins with a barrier, after which red, us and the
        // staged vectors may be rewritten
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) *reinterpret_cast<float4*>(st + i * DV) = s[i];
}

template <bool BF16, int DK>
cudaError_t launch_t(const DecodeArgs& a, cudaStream_t stream) {
    profile_mark(SLOT_DECODE, true, stream);
    decode_kernel<BF16, DK, 64><<<dim3((unsigned)(a.N * a.H), (unsigned)(a.dv / 64)),
                                  DecodeShape<BF16, DK, 64>::NTH, 0, stream>>>(a);
    profile_mark(SLOT_DECODE, false, stream);
    return cudaGetLastError();
}

template <bool BF16>
cudaError_t launch_dims(const DecodeArgs& a, cudaStream_t stream) {
    return a.dk == 128 ? launch_t<BF16, 128>(a, stream) : launch_t<BF16, 64>(a, stream);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream, int* launches) {
    if ((int64_t)a.N * a.H == 0) return cudaSuccess;
    *launches += 1;
    return a.bf16 ? launch_dims<true>(a, stream) : launch_dims<false>(a, stream);
}

}  // namespace kda
