// kda_cp.cu -- chains of segment transitions: the exchange step of context
// parallelism, and the composition of a sequence's segment transitions.
//
// aiblin.ru, "Kimi K3 -- открытая модель, которая обошла закрытых лидеров
// рынка", section "Как распараллелили последовательное обновление": a segment
// of the delta rule acts on its incoming state as an affine map, a local state
// plus a token-dependent transition matrix (S_out = M S_in + B), so the pieces of
// a long sequence can be computed independently -- on one GPU, or one piece per
// GPU -- and the true incoming states recovered afterwards by a prefix scan over
// the pieces' (M, B) after one all-gather.
//
// Transitions are kept transposed, as the tensor-core kernels produce them:
// entry [2][128][128] = B^T (d_v x d_k), then M^T (d_k x d_k), so that
// S^T_out = S^T_in M^T + B^T.  A chain step is X^T <- X^T M_j^T + A_j, on fp32
// CUDA cores:
//   composing:  X^T = [B_tot^T; M_tot^T] (256 x 128) from [0; I], A_j = [B_j^T; 0]
//               (then S_out = M_tot S_in + B_tot for the whole chain);
//   applying:   X^T = S^T (128 x 128) from S_in^T, A_j = B_j^T.
// One CTA owns 16 rows of X^T for one (sequence, head); M_j^T (64 KB) is staged
// in shared memory, the next one prefetched into registers during the product.
#include "kda_internal.h"

namespace kda {
namespace {

constexpr int D = 128;
constexpr int CHAIN_SMEM = 2 * D * D * 4 + 16 * D * 4;

__global__ void __launch_bounds__(256) chain_kernel(ChainArgs a) {
    extern __shared__ float4 chain_smem4[];
    float* Ms = reinterpret_cast<float*>(chain_smem4);  // [2][128][128]
    float* X = Ms + 2 * D * D;                         // [16][128]
    const int b = blockIdx.x, h = blockIdx.y, e0 = 16 * blockIdx.z, H = a.H;
    const int tid = threadIdx.x, el = tid >> 4, cg = tid & 15;
    int64_t base;  // index (in transitions) of the chain's first entry
    int64_t step;  // distance between consecutive entries
    int32_t J;
    if (a.compose) {
        const int32_t nu = *a.n_units;
        const int32_t u0 = a.off[b], u1 = min(a.off[b + 1], nu);
        J = u1 > u0 ? u1 - u0 : 0;
        base = (int64_t)u0 * H + h;
        step = H;
    } else {
        J = a.count;
        base = (int64_t)b * H + h;
        step = (int64_t)a.B * H;
    }
    for (int x = tid; x < 16 * D; x += 256) {
        const int r = x / D, c = x % D, gr = e0 + r;
        float v;
        if (a.compose)
            v = (gr >= D && c == gr - D) ? 1.f : 0.f;  // [0; I]
        else
            v = a.s0 ? a.s0[(((int64_t)b * H + h) * D + c) * D + gr] : 0.f;  // S^T
        X[r * D + c] = v;
    }
    float4 pre[16];
    auto load_m = [&](int32_t j) {
        const float4* Mt = reinterpret_cast<const float4*>(a.trans + (base + j * step) * 2 * D * D + D * D);
#pragma unroll
        for (int i = 0; i < 16; ++i) pre[i] = __ldg(Mt + tid + 256 * i);
    };
    auto store_m = [&](int buf) {
        float4* dst = reinterpret_cast<float4*>(Ms + buf * D * D);
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[tid + 256 * i] = pre[i];
    };
    if (J > 0) {
        load_m(0);
        store_m(0);
    }
    __syncthreads();
    const int gr = e0 + el;
    for (int32_t j = 0; j < J; ++j) {
        const int buf = j & 1;
        if (j + 1 < J) load_m(j + 1);
        float acc[8];
        if (gr < D) {
            const float* Bt = a.trans + (base + j * step) * 2 * D * D;
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = __ldg(Bt + (int64_t)gr * D + cg + 16 * i);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        }
        const float* M = Ms + buf * D * D;
#pragma unroll 4
        for (int c = 0; c < D; ++c) {
            const float xv = X[el * D + c];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = fmaf(xv, M[c * D + cg + 16 * i], acc[i]);
        }
        __syncthreads();  // everyone is done reading X and M[buf]
#pragma unroll
        for (int i = 0; i < 8; ++i) X[el * D + cg + 16 * i] = acc[i];
        if (j + 1 < J) store_m(buf ^ 1);
        __syncthreads();
    }
    // results
    if (a.compose) {
        float* dst = a.out + ((int64_t)b * H + h) * 2 * D * D + (int64_t)gr * D;
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[cg + 16 * i] = X[el * D + cg + 16 * i];
    } else {
        float* dst = a.out + ((int64_t)b * H + h) * D * D + gr;
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[(int64_t)(cg + 16 * i) * D] = X[el * D + cg + 16 * i];
    }
}

}  // namespace

cudaError_t launch_chain(const ChainArgs& c, cudaStream_t stream, int* launches) {
    if ((int64_t)c.B * c.H == 0) return cudaSuccess;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= kMaxDevices || !attr_set[dev]) {
        err = cudaFuncSetAttribute(chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   CHAIN_SMEM);
        if (err != cudaSuccess) return err;
        if (dev < kMaxDevices) attr_set[dev] = true;
    }
    const dim3 grid((unsigned)c.B, (unsigned)c.H, (unsigned)((c.compose ? 2 * D : D) / 16));
    profile_mark(SLOT_CHAIN, true, stream);
    chain_kernel<<<grid, 256, CHAIN_SMEM, stream>>>(c);
    profile_mark(SLOT_CHAIN, false, stream);
    *launches += 1;
    return cudaGetLastError();
}

}  // namespace kda
