// Internal declarations shared by the C-ABI layer and the kernels of libkda.so.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr int kChunk = 64;       // tokens per chunk
constexpr int kMaxDevices = 64;  // size of per-device attribute caches

// Everything a forward launch needs, already validated on the host.
struct FwdArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* log_alpha;
    const float* beta;
    const float* s0;         // [N,H,dk,dv] or nullptr
    const int32_t* cu;       // [N+1] device, or nullptr (then sequence n = [n*T, (n+1)*T))
    void* out;
    float* s_final;          // [N,H,dk,dv] or nullptr
    int32_t B, T, H, dk, dv, N;
    int32_t bf16;            // q/k/v/out are bf16 (else fp32)
};

// CUDA-core chunkwise path (exact fp32 arithmetic on fp32 or bf16 inputs).
cudaError_t launch_ffma(const FwdArgs& a, cudaStream_t stream, int* launches);

}  // namespace kda
