// kda_api.cu -- the C ABI of libkda.so (declared in include/kda.h).
//
// Host-side work only: argument validation (before any launch), choice of the
// kernel family, stream-ordered temporaries, and the host-buffer wrapper.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "kda.h"
#include "kda_internal.h"

namespace {

thread_local char g_last_error[512] = "";
thread_local int32_t g_last_launches = 0;
thread_local const char* g_last_path = "";

kda_status fail(kda_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

kda_status cuda_fail(cudaError_t e, const char* what) {
    return fail(KDA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

struct Range {
    uintptr_t lo, hi;  // [lo, hi)
    const char* name;
};

bool overlaps(const Range& a, const Range& b) {
    return a.lo < a.hi && b.lo < b.hi && a.lo < b.hi && b.lo < a.hi;
}

// Returns true when the pointer is usable by kernels on the current device.
bool device_accessible(const void* p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged ||
           (at.type == cudaMemoryTypeHost && at.devicePointer != nullptr);
}

kda_status validate(const void* q, const void* k, const void* v, const float* la,
                    const float* beta, const float* s0, const int32_t* cu, int32_t chunk,
                    const void* out, const float* sf, const kda_dims* d, bool device_ptrs,
                    kda::FwdArgs* a) {
    if (!d) return fail(KDA_ERR_INVALID_ARG, "dims is NULL");
    if (d->B < 1 || d->T < 0 || d->H < 1)
        return fail(KDA_ERR_INVALID_ARG, "need B >= 1, T >= 0, H >= 1 (got B=%d T=%d H=%d)",
                    d->B, d->T, d->H);
    if (d->qkv_dtype != KDA_F32 && d->qkv_dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "qkv_dtype must be KDA_F32 or KDA_BF16");
    if ((d->d_k != 64 && d->d_k != 128) || (d->d_v != 64 && d->d_v != 128))
        return fail(KDA_ERR_UNSUPPORTED, "d_k and d_v must be 64 or 128 (got %d, %d)", d->d_k,
                    d->d_v);
    if (chunk != kda::kChunk)
        return fail(KDA_ERR_UNSUPPORTED, "chunk must be %d (got %d)", kda::kChunk, chunk);
    int64_t N = d->B;
    if (cu) {
        if (d->B != 1) return fail(KDA_ERR_INVALID_ARG, "packed input (cu_seqlens) needs B == 1");
        if (d->num_seqs < 1) return fail(KDA_ERR_INVALID_ARG, "num_seqs must be >= 1");
        N = d->num_seqs;
    }
    const int64_t tokens = (int64_t)d->B * d->T;
    const int64_t e_in = d->qkv_dtype == KDA_BF16 ? 2 : 4;
    const int64_t nqk = tokens * d->H * d->d_k, nv = tokens * d->H * d->d_v;
    const int64_t nst = N * d->H * d->d_k * d->d_v;
    if (tokens > 0 && (!q || !k || !v || !la || !beta || !out))
        return fail(KDA_ERR_INVALID_ARG, "q, k, v, log_alpha, beta and out must be non-NULL");
    const void* ptrs[] = {q, k, v, la, beta, s0, cu, out, sf};
    const char* names[] = {"q", "k", "v", "log_alpha", "beta", "initial_state", "cu_seqlens",
                           "out", "final_state"};
    for (int i = 0; i < 9; ++i) {
        if (ptrs[i] && ((uintptr_t)ptrs[i] & 15u) && i != 6)
            return fail(KDA_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
        if (i == 6 && ptrs[i] && ((uintptr_t)ptrs[i] & 3u))
            return fail(KDA_ERR_MISALIGNED, "cu_seqlens is not 4-byte aligned");
    }
    const Range in[] = {
        {(uintptr_t)q, (uintptr_t)q + (q ? nqk * e_in : 0), "q"},
        {(uintptr_t)k, (uintptr_t)k + (k ? nqk * e_in : 0), "k"},
        {(uintptr_t)v, (uintptr_t)v + (v ? nv * e_in : 0), "v"},
        {(uintptr_t)la, (uintptr_t)la + (la ? nqk * 4 : 0), "log_alpha"},
        {(uintptr_t)beta, (uintptr_t)beta + (beta ? tokens * d->H * 4 : 0), "beta"},
        {(uintptr_t)s0, (uintptr_t)s0 + (s0 ? nst * 4 : 0), "initial_state"},
        {(uintptr_t)cu, (uintptr_t)cu + (cu ? (N + 1) * 4 : 0), "cu_seqlens"},
    };
    const Range ro = {(uintptr_t)out, (uintptr_t)out + (out ? nv * e_in : 0), "out"};
    const Range rs = {(uintptr_t)sf, (uintptr_t)sf + (sf ? nst * 4 : 0), "final_state"};
    for (const Range& r : in) {
        if (overlaps(ro, r)) return fail(KDA_ERR_ALIAS, "out overlaps %s", r.name);
        if (overlaps(rs, r) && !(r.lo == rs.lo && r.hi == rs.hi && r.name[0] == 'i'))
            return fail(KDA_ERR_ALIAS, "final_state overlaps %s", r.name);
    }
    if (overlaps(ro, rs)) return fail(KDA_ERR_ALIAS, "out overlaps final_state");
    if (device_ptrs) {
        for (int i = 0; i < 9; ++i)
            if (ptrs[i] && !device_accessible(ptrs[i]))
                return fail(KDA_ERR_INVALID_ARG, "%s is not device-accessible memory", names[i]);
    }
    a->q = q;
    a->k = k;
    a->v = v;
    a->log_alpha = la;
    a->beta = beta;
    a->s0 = s0;
    a->cu = cu;
    a->out = const_cast<void*>(out);
    a->s_final = const_cast<float*>(sf);
    a->B = d->B;
    a->T = d->T;
    a->H = d->H;
    a->dk = d->d_k;
    a->dv = d->d_v;
    a->N = (int32_t)N;
    a->bf16 = d->qkv_dtype == KDA_BF16;
    return KDA_OK;
}

kda_status run(const kda::FwdArgs& a, cudaStream_t stream) {
    int launches = 0;
    g_last_path = "ffma";
    cudaError_t e = kda::launch_ffma(a, stream, &launches);
    g_last_launches = launches;
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return KDA_OK;
}

}  // namespace

extern "C" {

kda_status kda_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                   const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                   int32_t chunk, void* out, float* final_state, const kda_dims* dims,
                   void* stream) {
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    kda::FwdArgs a;
    kda_status s = validate(q, k, v, log_alpha, beta, initial_state, cu_seqlens, chunk, out,
                            final_state, dims, true, &a);
    if (s != KDA_OK) return s;
    return run(a, (cudaStream_t)stream);
}

kda_status kda_fwd_host(const void* q, const void* k, const void* v, const float* log_alpha,
                        const float* beta, const float* initial_state,
                        const int32_t* cu_seqlens, int32_t chunk, void* out,
                        float* final_state, const kda_dims* dims, void* stream_) {
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    kda::FwdArgs a;
    kda_status s = validate(q, k, v, log_alpha, beta, initial_state, cu_seqlens, chunk, out,
                            final_state, dims, false, &a);
    if (s != KDA_OK) return s;
    cudaStream_t stream = (cudaStream_t)stream_;
    const int64_t tokens = (int64_t)a.B * a.T;
    const int64_t e_in = a.bf16 ? 2 : 4;
    const size_t bqk = (size_t)(tokens * a.H * a.dk * e_in), bv = (size_t)(tokens * a.H * a.dv * e_in);
    const size_t bla = (size_t)(tokens * a.H * a.dk * 4), bbe = (size_t)(tokens * a.H * 4);
    const size_t bst = (size_t)a.N * a.H * a.dk * a.dv * 4, bcu = cu_seqlens ? (size_t)(a.N + 1) * 4 : 0;
    // one pool allocation carved into 16-byte aligned pieces
    const size_t sizes[] = {bqk, bqk, bv, bla, bbe, initial_state ? bst : 0, bcu, bv,
                            final_state ? bst : 0};
    size_t off[9], total = 0;
    for (int i = 0; i < 9; ++i) {
        off[i] = total;
        total += (sizes[i] + 255) & ~(size_t)255;
    }
    char* base = nullptr;
    cudaError_t e = cudaSuccess;
    if (total) {
        e = cudaMallocAsync((void**)&base, total, stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync");
    }
    const void* src[] = {q, k, v, log_alpha, beta, initial_state, cu_seqlens};
    for (int i = 0; i < 7 && e == cudaSuccess; ++i)
        if (sizes[i] && src[i])
            e = cudaMemcpyAsync(base + off[i], src[i], sizes[i], cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) {
        cudaFreeAsync(base, stream);
        return cuda_fail(e, "host-to-device copy");
    }
    kda::FwdArgs d = a;
    d.q = base + off[0];
    d.k = base + off[1];
    d.v = base + off[2];
    d.log_alpha = (const float*)(base + off[3]);
    d.beta = (const float*)(base + off[4]);
    d.s0 = initial_state ? (const float*)(base + off[5]) : nullptr;
    d.cu = cu_seqlens ? (const int32_t*)(base + off[6]) : nullptr;
    d.out = base + off[7];
    d.s_final = final_state ? (float*)(base + off[8]) : nullptr;
    s = run(d, stream);
    if (s == KDA_OK) {
        if (sizes[7]) e = cudaMemcpyAsync(out, d.out, sizes[7], cudaMemcpyDeviceToHost, stream);
        if (e == cudaSuccess && final_state)
            e = cudaMemcpyAsync(final_state, d.s_final, sizes[8], cudaMemcpyDeviceToHost, stream);
    }
    if (base) cudaFreeAsync(base, stream);
    cudaError_t e2 = cudaStreamSynchronize(stream);
    if (s != KDA_OK) return s;
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
    if (e2 != cudaSuccess) return cuda_fail(e2, "stream synchronize");
    return KDA_OK;
}

const char* kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_MISALIGNED: return "KDA_ERR_MISALIGNED";
        case KDA_ERR_ALIAS: return "KDA_ERR_ALIAS";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_DEVICE_TIMEOUT: return "KDA_ERR_DEVICE_TIMEOUT";
    }
    return "KDA_ERR_UNKNOWN";
}

const char* kda_last_error(void) { return g_last_error; }

int32_t kda_last_launch_count(void) { return g_last_launches; }

const char* kda_last_path(void) { return g_last_path; }

}  // extern "C"
