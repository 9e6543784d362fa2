// kda_api.cu -- the C ABI of libkda.so (declared in include/kda.h).
//
// Host-side work only: argument validation (before any launch), choice of the
// kernel family, stream-ordered temporaries, and the host-buffer wrapper.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <mutex>
#include <vector>

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

kda_status check_accessible(const void* const* ptrs, const char* const* names, int n) {
    for (int i = 0; i < n; ++i)
        if (ptrs[i] && !device_accessible(ptrs[i]))
            return fail(KDA_ERR_INVALID_ARG, "%s is not device-accessible memory", names[i]);
    return KDA_OK;
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
        kda_status st = check_accessible(ptrs, names, 9);
        if (st != KDA_OK) return st;
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

// Library-owned stream-ordered pool per device.  Freed blocks stay reserved in
// the pool (release threshold = max), so repeated calls do not re-map memory.
cudaError_t get_pool(cudaMemPool_t* pool) {
    static cudaMemPool_t pools[kda::kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kda::kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!pools[dev]) {
        cudaMemPoolProps props;
        memset(&props, 0, sizeof props);
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        e = cudaMemPoolCreate(&pools[dev], &props);
        if (e != cudaSuccess) return e;
        uint64_t thr = UINT64_MAX;
        e = cudaMemPoolSetAttribute(pools[dev], cudaMemPoolAttrReleaseThreshold, &thr);
        if (e != cudaSuccess) return e;
    }
    *pool = pools[dev];
    return cudaSuccess;
}

cudaError_t pool_alloc(void** p, size_t bytes, cudaStream_t stream) {
    cudaMemPool_t pool;
    cudaError_t e = get_pool(&pool);
    if (e != cudaSuccess) return e;
    return cudaMallocFromPoolAsync(p, bytes, pool, stream);
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n;
}

// Segment plan: enough (segment, head) units for about two waves of CTAs.
kda::TcPlan plan_segments(const kda::FwdArgs& a) {
    constexpr int C = kda::kChunk;
    const int64_t nch_seq_max = ((int64_t)a.T + C - 1) / C;  // chunks of the longest possible sequence
    const int64_t nch_total = a.cu ? nch_seq_max + a.N : (int64_t)a.B * nch_seq_max;
    const int64_t target = 2LL * sm_count();
    int64_t seg;
    if (!a.cu) {
        const int64_t G = std::max<int64_t>(1, llround((double)target / ((double)a.B * a.H)));
        seg = (nch_seq_max + G - 1) / G;
    } else {
        seg = (nch_total * a.H + target - 1) / target;
    }
    seg = std::max<int64_t>(seg, 8);
    // test hook: force the segment length (in chunks)
    if (const char* env = getenv("KDA_SEG_CHUNKS")) {
        const long v = atol(env);
        if (v > 0) seg = v;
    }
    kda::TcPlan p;
    p.segmented = seg < nch_seq_max;
    if (!p.segmented) seg = std::max<int64_t>(nch_seq_max, 1);
    p.seg_chunks = (int)std::min<int64_t>(seg, 1 << 30);
    p.max_units = (int)(p.segmented ? (nch_total + seg - 1) / seg + a.N : a.N);
    p.total_chunks = nch_total;
    return p;
}

kda_status run_tc(const kda::FwdArgs& a, cudaStream_t stream, int* launches) {
    const kda::TcPlan p = plan_segments(a);
    const size_t st = (size_t)128 * 128 * sizeof(float);
    const size_t b_segs = ((size_t)p.max_units * sizeof(kda::SegEntry) + 255) & ~(size_t)255;
    const size_t b_off = ((size_t)(a.N + 1) * 4 + 4 + 255) & ~(size_t)255;
    const size_t b_trans = p.segmented ? (size_t)p.max_units * a.H * 2 * st : 0;
    const size_t b_sin = p.segmented ? (size_t)p.max_units * a.H * st : 0;
    // chunk cache of the segmented plan: kCacheEntryBytes per chunk and head
    const size_t b_cache = p.segmented ? (size_t)p.total_chunks * a.H * kda::kCacheEntryBytes : 0;
#ifdef KDA_DEBUG
    // debug builds: a guard band before the first buffer and after every buffer
    constexpr size_t G = kda::kGuardBytes;
#else
    constexpr size_t G = 0;
#endif
    char* base = nullptr;
    cudaError_t e = pool_alloc((void**)&base, G + b_segs + G + b_off + G + b_trans + G + b_sin + G +
                                                  b_cache + G, stream);
    if (e != cudaSuccess) return cuda_fail(e, "workspace allocation");
    char* ws = base + G;
    const size_t o_off = b_segs + G, o_trans = o_off + b_off + G, o_sin = o_trans + b_trans + G,
                 o_cache = o_sin + b_sin + G;
#ifdef KDA_DEBUG
    kda::GuardBands guards{};
    for (char* g : {base, ws + b_segs, ws + o_off + b_off, ws + o_trans + b_trans, ws + o_sin + b_sin,
                    ws + o_cache + b_cache}) {
        guards.band[guards.n++] = (const uint32_t*)g;
        if ((e = cudaMemsetAsync(g, 0xA5, G, stream)) != cudaSuccess) {
            cudaFreeAsync(base, stream);
            return cuda_fail(e, "guard band fill");
        }
    }
#endif
    kda::TcArgs t{};
    t.q = a.q;
    t.k = a.k;
    t.v = a.v;
    t.log_alpha = a.log_alpha;
    t.beta = a.beta;
    t.s0 = a.s0;
    t.cu = a.cu;
    t.out = a.out;
    t.s_final = a.s_final;
    t.gate = a.gate;
    t.snap_slots = a.snap_slots;
    t.snap_pool = a.snap_pool;
    t.snap_interval = a.snap_interval;
    t.snap_max = a.snap_max;
    t.snap_num_slots = a.snap_num_slots;
    t.B = a.B;
    t.T = a.T;
    t.H = a.H;
    t.N = a.N;
    t.segs = (kda::SegEntry*)ws;
    t.seg_off = (int32_t*)(ws + o_off);
    t.n_units = t.seg_off + a.N + 1;
    t.trans = p.segmented ? (float*)(ws + o_trans) : nullptr;
    t.sin = p.segmented ? (float*)(ws + o_sin) : nullptr;
    if (p.segmented) {  // pass 1 runs over every segment and leaves the chunk cache for pass 3
        t.cache = (uint8_t*)(ws + o_cache);
        t.total_chunks = p.total_chunks;
        t.trans_all = 1;
    }
    e = kda::launch_tc(t, p, stream, launches);
#ifdef KDA_DEBUG
    if (e == cudaSuccess) e = kda::launch_guard_check(guards, stream);
#endif
    cudaFreeAsync(base, stream);
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return KDA_OK;
}

kda_status run(const kda::FwdArgs& a, cudaStream_t stream) {
    int launches = 0;
    if ((int64_t)a.N * a.H == 0) return KDA_OK;
    kda_status s = KDA_OK;
    if (a.bf16 && a.dk == 128 && a.dv == 128) {
        g_last_path = "tc";
        s = run_tc(a, stream, &launches);
    } else {
        g_last_path = "ffma";
        cudaError_t e = kda::launch_ffma(a, stream, &launches);
        if (e != cudaSuccess) s = cuda_fail(e, "kernel launch");
    }
    g_last_launches = launches;
    return s;
}

// ---------------------------------------------------------------- launch timing
struct Profiler {
    std::mutex mu;
    std::atomic<bool> on{false};
    struct Mark {
        int slot;
        cudaEvent_t a, b;
    };
    std::vector<Mark> pending;
    std::vector<cudaEvent_t> free_events;
    cudaEvent_t open_ev[kda::NUM_SLOTS] = {};
    double total_ms[kda::NUM_SLOTS] = {};
    int64_t count[kda::NUM_SLOTS] = {};

    cudaEvent_t get_event() {
        if (!free_events.empty()) {
            cudaEvent_t e = free_events.back();
            free_events.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        cudaEventCreate(&e);
        return e;
    }
};
Profiler& profiler() {
    static Profiler p;
    return p;
}

// ---------------------------------------------------------------- no-allocation scratch
// Device scratch for kda_fwd_noalloc: a fixed array inside the library image.
// The driver reserves it on every device the library is loaded on, for the
// life of the process.  In host code `g_noalloc_scratch` only names the
// symbol; its device address comes from cudaGetSymbolAddress, taken once per
// device (with that device current) by noalloc_scratch().
constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

cudaError_t noalloc_scratch(char** ptr) {
    static void* addr[kda::kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= kda::kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *ptr = (char*)addr[dev];
    return cudaSuccess;
}

// Bytes of scratch the tensor-core path needs for a segment plan.
size_t tc_scratch_bytes(const kda::FwdArgs& a, const kda::TcPlan& p, size_t* b_segs,
                        size_t* b_off, size_t* b_trans) {
    const size_t st = (size_t)128 * 128 * sizeof(float);
    *b_segs = ((size_t)p.max_units * sizeof(kda::SegEntry) + 255) & ~(size_t)255;
    *b_off = ((size_t)(a.N + 1) * 4 + 4 + 255) & ~(size_t)255;
    *b_trans = p.segmented ? (size_t)p.max_units * a.H * 2 * st : 0;
    const size_t b_sin = p.segmented ? (size_t)p.max_units * a.H * st : 0;
    return *b_segs + *b_off + *b_trans + b_sin;
}

// Workspace of a span (segment table, per-segment transitions and incoming
// states, chunk cache) for the segment plan of the dims: offsets into one buffer.
struct SpanWs {
    kda::TcPlan p;
    size_t segs, off, trans, sin, cache, total;
};

SpanWs span_layout(const kda::FwdArgs& a) {
    SpanWs w;
    w.p = plan_segments(a);
    const size_t st = (size_t)128 * 128 * sizeof(float);
    size_t o = 0;
    auto take = [&](size_t b) {
        const size_t at = o;
        o += (b + 255) & ~(size_t)255;
        return at;
    };
    w.segs = take((size_t)w.p.max_units * sizeof(kda::SegEntry));
    w.off = take((size_t)(a.N + 1) * 4 + 4);
    w.trans = take((size_t)w.p.max_units * a.H * 2 * st);
    w.sin = take((size_t)w.p.max_units * a.H * st);
    w.cache = take((size_t)w.p.total_chunks * a.H * kda::kCacheEntryBytes);
    w.total = o;
    return w;
}

kda::TcArgs span_args(const kda::FwdArgs& a, const SpanWs& w, char* ws) {
    kda::TcArgs t{};
    t.q = a.q;
    t.k = a.k;
    t.v = a.v;
    t.log_alpha = a.log_alpha;
    t.beta = a.beta;
    t.B = a.B;
    t.T = a.T;
    t.H = a.H;
    t.N = a.N;
    t.segs = (kda::SegEntry*)(ws + w.segs);
    t.seg_off = (int32_t*)(ws + w.off);
    t.n_units = t.seg_off + a.N + 1;
    t.trans = (float*)(ws + w.trans);
    t.sin = (float*)(ws + w.sin);
    t.cache = (uint8_t*)(ws + w.cache);
    t.total_chunks = w.p.total_chunks;
    t.trans_all = 1;
    return t;
}

kda_status check_workspace(const void* ws, size_t bytes, size_t need) {
    if (!ws) return fail(KDA_ERR_INVALID_ARG, "workspace is NULL");
    if ((uintptr_t)ws & 255u) return fail(KDA_ERR_MISALIGNED, "workspace is not 256-byte aligned");
    if (bytes < need)
        return fail(KDA_ERR_INVALID_ARG, "workspace holds %zu bytes, the span needs %zu", bytes, need);
    return KDA_OK;
}

// Arguments of a span transition (k, v, log_alpha, beta; bf16, d = 128, no cu_seqlens);
// need_q: q too (checked like the other inputs).
kda_status validate_span_inputs(const void* q, const void* k, const void* v, const float* log_alpha,
                                const float* beta, const kda_dims* d, const float* trans,
                                bool need_q, kda::FwdArgs* a, size_t trans_bytes = 0,
                                const char* trans_name = "trans") {
    if (!d) return fail(KDA_ERR_INVALID_ARG, "dims is NULL");
    if (d->B < 1 || d->T < 0 || d->H < 1)
        return fail(KDA_ERR_INVALID_ARG, "need B >= 1, T >= 0, H >= 1 (got B=%d T=%d H=%d)",
                    d->B, d->T, d->H);
    if (d->qkv_dtype != KDA_F32 && d->qkv_dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "qkv_dtype must be KDA_F32 or KDA_BF16");
    if (d->d_k != 128 || d->d_v != 128 || d->qkv_dtype != KDA_BF16)
        return fail(KDA_ERR_UNSUPPORTED, "span transitions need bf16 k/v with d_k = d_v = 128");
    const int64_t tokens = (int64_t)d->B * d->T;
    if (!trans) return fail(KDA_ERR_INVALID_ARG, "%s must be non-NULL", trans_name);
    if (tokens > 0 && (!k || !v || !log_alpha || !beta || (need_q && !q)))
        return fail(KDA_ERR_INVALID_ARG, need_q ? "q, k, v, log_alpha and beta must be non-NULL"
                                                : "k, v, log_alpha and beta must be non-NULL");
    if (!need_q) q = nullptr;
    const void* ptrs[] = {q, k, v, log_alpha, beta, trans};
    const char* names[] = {"q", "k", "v", "log_alpha", "beta", trans_name};
    for (int i = 0; i < 6; ++i)
        if (ptrs[i] && ((uintptr_t)ptrs[i] & 15u))
            return fail(KDA_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    const int64_t n = tokens * d->H * 128;
    const Range in[] = {{(uintptr_t)q, (uintptr_t)q + (q ? n * 2 : 0), "q"},
                        {(uintptr_t)k, (uintptr_t)k + (k ? n * 2 : 0), "k"},
                        {(uintptr_t)v, (uintptr_t)v + (v ? n * 2 : 0), "v"},
                        {(uintptr_t)log_alpha, (uintptr_t)log_alpha + (log_alpha ? n * 4 : 0),
                         "log_alpha"},
                        {(uintptr_t)beta, (uintptr_t)beta + (beta ? tokens * d->H * 4 : 0), "beta"}};
    if (!trans_bytes) trans_bytes = (size_t)d->B * d->H * 2 * 128 * 128 * 4;
    const Range rt = {(uintptr_t)trans, (uintptr_t)trans + trans_bytes, trans_name};
    for (const Range& r : in)
        if (overlaps(rt, r)) return fail(KDA_ERR_ALIAS, "%s overlaps %s", trans_name, r.name);
    a->q = q;
    a->k = k;
    a->v = v;
    a->log_alpha = log_alpha;
    a->beta = beta;
    a->s0 = nullptr;
    a->cu = nullptr;
    a->out = nullptr;
    a->s_final = nullptr;
    a->B = d->B;
    a->T = d->T;
    a->H = d->H;
    a->dk = 128;
    a->dv = 128;
    a->N = d->B;
    a->bf16 = 1;
    return KDA_OK;
}

}  // namespace

void kda::profile_mark(int slot, bool begin, cudaStream_t stream) {
    Profiler& P = profiler();
    if (!P.on.load(std::memory_order_relaxed)) return;
    std::lock_guard<std::mutex> lock(P.mu);
    cudaEvent_t e = P.get_event();
    if (!e) return;
    cudaEventRecord(e, stream);
    if (begin) {
        P.open_ev[slot] = e;
    } else if (P.open_ev[slot]) {
        P.pending.push_back({slot, P.open_ev[slot], e});
        P.open_ev[slot] = nullptr;
    }
}

extern "C" {

kda_status kda_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                   const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                   int32_t chunk, void* out, float* final_state, const kda_dims* dims,
                   void* stream) {
    kda::NvtxRange nvtx_range("kda_fwd");
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    kda::FwdArgs a;
    kda_status s = validate(q, k, v, log_alpha, beta, initial_state, cu_seqlens, chunk, out,
                            final_state, dims, true, &a);
    if (s != KDA_OK) return s;
    return run(a, (cudaStream_t)stream);
}

// Checks the optional parts of a forward call against the validated dims and
// the call's other buffers, and records them in `a`.  Argument checks first,
// then whether every pointer is device memory (as in kda_fwd).
static kda_status apply_opts(const kda_fwd_opts* opts, const void* q, const void* k, const void* v,
                             const float* log_alpha, const float* beta, const float* initial_state,
                             const int32_t* cu_seqlens, const void* out, const float* final_state,
                             kda::FwdArgs* pa) {
    kda::FwdArgs& a = *pa;
    const kda_fwd_opts none = {nullptr, nullptr, nullptr, nullptr};
    if (!opts) opts = &none;
    const kda_snap_spec* snap = opts->snap;
    if (snap) {
        if (snap->interval <= 0 || snap->interval % kda::kChunk)
            return fail(KDA_ERR_INVALID_ARG, "snapshot interval must be a positive multiple of %d "
                        "(got %d)", kda::kChunk, snap->interval);
        if (snap->max_snaps < 0 || snap->num_slots < 0)
            return fail(KDA_ERR_INVALID_ARG, "max_snaps and num_slots must be >= 0");
        if (snap->max_snaps == 0 || snap->num_slots == 0) snap = nullptr;  // nothing requested
    }
    const void* gate = opts->out_gate;
    const int32_t* snap_slots = snap ? opts->snap_slots : nullptr;
    float* snap_pool = snap ? opts->snap_pool : nullptr;
    if (snap && (!snap_slots || !snap_pool))
        return fail(KDA_ERR_INVALID_ARG, "snap_slots and snap_pool must be non-NULL");
    if (gate && ((uintptr_t)gate & 15u)) return fail(KDA_ERR_MISALIGNED, "out_gate is not 16-byte aligned");
    if (snap_slots && ((uintptr_t)snap_slots & 3u))
        return fail(KDA_ERR_MISALIGNED, "snap_slots is not 4-byte aligned");
    if (snap_pool && ((uintptr_t)snap_pool & 15u))
        return fail(KDA_ERR_MISALIGNED, "snap_pool is not 16-byte aligned");
    const int64_t tokens = (int64_t)a.B * a.T, e_in = a.bf16 ? 2 : 4;
    const int64_t dd = (int64_t)a.dk * a.dv, nst = (int64_t)a.N * a.H * dd * 4;
    const Range r_gate = {(uintptr_t)gate, (uintptr_t)gate + (gate ? tokens * a.H * a.dv * e_in : 0),
                          "out_gate"};
    const Range r_pool = {(uintptr_t)snap_pool,
                          (uintptr_t)snap_pool + (snap_pool ? (uintptr_t)snap->num_slots * a.H * dd * 4 : 0),
                          "snap_pool"};
    const Range r_slots = {(uintptr_t)snap_slots,
                           (uintptr_t)snap_slots + (snap_slots ? (uintptr_t)a.N * snap->max_snaps * 4 : 0),
                           "snap_slots"};
    const Range r_out = {(uintptr_t)out, (uintptr_t)out + (out ? tokens * a.H * a.dv * e_in : 0), "out"};
    const Range r_fin = {(uintptr_t)final_state, (uintptr_t)final_state + (final_state ? nst : 0),
                         "final_state"};
    const Range inputs[] = {
        {(uintptr_t)q, (uintptr_t)q + (q ? tokens * a.H * a.dk * e_in : 0), "q"},
        {(uintptr_t)k, (uintptr_t)k + (k ? tokens * a.H * a.dk * e_in : 0), "k"},
        {(uintptr_t)v, (uintptr_t)v + (v ? tokens * a.H * a.dv * e_in : 0), "v"},
        {(uintptr_t)log_alpha, (uintptr_t)log_alpha + (log_alpha ? tokens * a.H * a.dk * 4 : 0),
         "log_alpha"},
        {(uintptr_t)beta, (uintptr_t)beta + (beta ? tokens * a.H * 4 : 0), "beta"},
        {(uintptr_t)initial_state, (uintptr_t)initial_state + (initial_state ? nst : 0),
         "initial_state"},
        {(uintptr_t)cu_seqlens, (uintptr_t)cu_seqlens + (cu_seqlens ? (a.N + 1) * 4 : 0),
         "cu_seqlens"},
        r_gate, r_slots,
    };
    // the written buffers (out, final_state: checked by validate; snap_pool) overlap no input
    for (const Range& r : inputs) {
        if (overlaps(r_pool, r)) return fail(KDA_ERR_ALIAS, "snap_pool overlaps %s", r.name);
        if (&r >= &inputs[7] && (overlaps(r_out, r) || overlaps(r_fin, r)))
            return fail(KDA_ERR_ALIAS, "%s overlaps an output", r.name);
    }
    if (overlaps(r_pool, r_out) || overlaps(r_pool, r_fin))
        return fail(KDA_ERR_ALIAS, "snap_pool overlaps an output");
    const void* ptrs[] = {q, k, v, log_alpha, beta, initial_state, cu_seqlens, out, final_state,
                          gate, snap_slots, snap_pool};
    const char* names[] = {"q", "k", "v", "log_alpha", "beta", "initial_state", "cu_seqlens",
                           "out", "final_state", "out_gate", "snap_slots", "snap_pool"};
    kda_status s = check_accessible(ptrs, names, 12);
    if (s != KDA_OK) return s;
    a.gate = gate;
    if (snap) {
        a.snap_slots = snap_slots;
        a.snap_pool = snap_pool;
        a.snap_interval = snap->interval;
        a.snap_max = snap->max_snaps;
        a.snap_num_slots = snap->num_slots;
        cudaError_t e = kda::status_word(&a.status);
        if (e != cudaSuccess) return cuda_fail(e, "device status word");
    }
    return KDA_OK;
}

kda_status kda_fwd_ex(const void* q, const void* k, const void* v, const float* log_alpha,
                      const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                      int32_t chunk, void* out, float* final_state, const kda_dims* dims,
                      const kda_fwd_opts* opts, void* stream) {
    kda::NvtxRange nvtx_range("kda_fwd_ex");
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    kda::FwdArgs a;
    kda_status s = validate(q, k, v, log_alpha, beta, initial_state, cu_seqlens, chunk, out,
                            final_state, dims, false, &a);
    if (s != KDA_OK) return s;
    s = apply_opts(opts, q, k, v, log_alpha, beta, initial_state, cu_seqlens, out, final_state, &a);
    if (s != KDA_OK) return s;
    return run(a, (cudaStream_t)stream);
}

kda_status kda_fwd_snap(const void* q, const void* k, const void* v, const float* log_alpha,
                        const float* beta, const float* initial_state,
                        const int32_t* cu_seqlens, int32_t chunk, void* out, float* final_state,
                        const kda_dims* dims, const kda_snap_spec* snap,
                        const int32_t* snap_slots, float* snap_pool, void* stream) {
    kda::NvtxRange nvtx_range("kda_fwd_snap");
    if (!snap) {
        g_last_error[0] = 0;
        g_last_launches = 0;
        g_last_path = "";
        return fail(KDA_ERR_INVALID_ARG, "snap is NULL");
    }
    const kda_fwd_opts o = {nullptr, snap, snap_slots, snap_pool};
    return kda_fwd_ex(q, k, v, log_alpha, beta, initial_state, cu_seqlens, chunk, out, final_state,
                      dims, &o, stream);
}

// Tokens per span of kda_fwd_host's pipelined path, or 0 for the one-call path: one
// sequence (B = 1, no cu_seqlens) longer than one span is cut into spans of whole chunks.
int64_t host_span_tokens(const kda::FwdArgs& a) {
    if (a.cu || a.B != 1) return 0;
    int64_t span = 131072;
    if (const char* env = getenv("KDA_HOST_SPAN_TOKENS")) {  // test hook
        const long v = atol(env);
        if (v > 0) span = v;
    }
    span = (span + kda::kChunk - 1) / kda::kChunk * kda::kChunk;
    return a.T > span ? span : 0;
}

kda_status kda_fwd_host(const void* q, const void* k, const void* v, const float* log_alpha,
                        const float* beta, const float* initial_state,
                        const int32_t* cu_seqlens, int32_t chunk, void* out,
                        float* final_state, const kda_dims* dims, void* stream_) {
    kda::NvtxRange nvtx_range("kda_fwd_host");
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
    const int64_t span = host_span_tokens(a);
    // one pool allocation carved into 256-byte aligned pieces (the last: the state passed
    // between spans)
    const size_t sizes[] = {bqk, bqk, bv, bla, bbe, initial_state ? bst : 0, bcu, bv,
                            final_state ? bst : 0, span ? bst : 0};
    size_t off[10], total = 0;
    for (int i = 0; i < 10; ++i) {
        off[i] = total;
        total += (sizes[i] + 255) & ~(size_t)255;
    }
    char* base = nullptr;
    cudaError_t e = cudaSuccess;
    if (total) {
        e = pool_alloc((void**)&base, total, stream);
        if (e != cudaSuccess) return cuda_fail(e, "device buffer allocation");
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
    const void* src[] = {q, k, v, log_alpha, beta, initial_state, cu_seqlens};
    if (!span) {  // copy in, one forward call, copy out, all on the caller's stream
        for (int i = 0; i < 7 && e == cudaSuccess; ++i)
            if (sizes[i] && src[i])
                e = cudaMemcpyAsync(base + off[i], src[i], sizes[i], cudaMemcpyHostToDevice, stream);
        if (e != cudaSuccess) {
            cudaFreeAsync(base, stream);
            return cuda_fail(e, "host-to-device copy");
        }
        s = run(d, stream);
        if (s == KDA_OK) {
            if (sizes[7]) e = cudaMemcpyAsync(out, d.out, sizes[7], cudaMemcpyDeviceToHost, stream);
            if (e == cudaSuccess && final_state)
                e = cudaMemcpyAsync(final_state, d.s_final, sizes[8], cudaMemcpyDeviceToHost, stream);
        }
    } else {
        // The sequence in spans: span r's inputs come in on `cin` while earlier spans are
        // computed on `cmp` (one forward call per span, each starting from the state the
        // previous one ended with, held in one buffer that every call reads before it
        // writes it) and earlier outputs go back on `cout`, so the two copy directions
        // overlap.  The caller's stream waits for all three at the end.
        const int64_t n_spans = (a.T + span - 1) / span;
        const int64_t row_in = a.H * a.dk * e_in, row_v = a.H * a.dv * e_in;
        const int64_t row_la = a.H * a.dk * 4, row_be = a.H * 4;
        float* st = (float*)(base + off[9]);
        cudaStream_t cin = nullptr, cmp = nullptr, cout_ = nullptr;
        cudaEvent_t ev_start = nullptr, ev_end = nullptr;
        e = cudaStreamCreateWithFlags(&cin, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&cmp, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&cout_, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_end, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventRecord(ev_start, stream);  // after the allocation
        for (cudaStream_t x : {cin, cmp, cout_})
            if (e == cudaSuccess) e = cudaStreamWaitEvent(x, ev_start, 0);
        if (e == cudaSuccess && initial_state)
            e = cudaMemcpyAsync(base + off[5], initial_state, bst, cudaMemcpyHostToDevice, cin);
        int launches = 0;
        for (int64_t r = 0; r < n_spans && e == cudaSuccess && s == KDA_OK; ++r) {
            const int64_t t0 = r * span, L = std::min<int64_t>(span, a.T - t0);
            const size_t pieces[5][2] = {{off[0] + t0 * row_in, (size_t)(L * row_in)},
                                         {off[1] + t0 * row_in, (size_t)(L * row_in)},
                                         {off[2] + t0 * row_v, (size_t)(L * row_v)},
                                         {off[3] + t0 * row_la, (size_t)(L * row_la)},
                                         {off[4] + t0 * row_be, (size_t)(L * row_be)}};
            const int64_t src_off[5] = {t0 * row_in, t0 * row_in, t0 * row_v, t0 * row_la, t0 * row_be};
            for (int i = 0; i < 5 && e == cudaSuccess; ++i)
                e = cudaMemcpyAsync(base + pieces[i][0], (const char*)src[i] + src_off[i], pieces[i][1],
                                    cudaMemcpyHostToDevice, cin);
            cudaEvent_t ev_in = nullptr, ev_done = nullptr;
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_in, cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_done, cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventRecord(ev_in, cin);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(cmp, ev_in, 0);
            if (e == cudaSuccess) {
                kda::FwdArgs dr = d;
                dr.T = (int32_t)L;
                dr.q = base + pieces[0][0];
                dr.k = base + pieces[1][0];
                dr.v = base + pieces[2][0];
                dr.log_alpha = (const float*)(base + pieces[3][0]);
                dr.beta = (const float*)(base + pieces[4][0]);
                dr.out = base + off[7] + t0 * row_v;
                dr.s0 = r == 0 ? d.s0 : st;
                dr.s_final = (r == n_spans - 1 && d.s_final) ? d.s_final : st;
                s = run(dr, cmp);
                launches += g_last_launches;
            }
            if (e == cudaSuccess && s == KDA_OK) e = cudaEventRecord(ev_done, cmp);
            if (e == cudaSuccess && s == KDA_OK) e = cudaStreamWaitEvent(cout_, ev_done, 0);
            if (e == cudaSuccess && s == KDA_OK)
                e = cudaMemcpyAsync((char*)out + t0 * row_v, base + off[7] + t0 * row_v, (size_t)(L * row_v),
                                    cudaMemcpyDeviceToHost, cout_);
            if (ev_in) cudaEventDestroy(ev_in);  // released once the work recorded on it is done
            if (ev_done) cudaEventDestroy(ev_done);
        }
        if (e == cudaSuccess && s == KDA_OK && final_state)
            e = cudaMemcpyAsync(final_state, d.s_final, bst, cudaMemcpyDeviceToHost, cout_);
        // join: the caller's stream waits for every stream that ran (copies in flight on a
        // failed path are drained by the synchronisations below)
        for (cudaStream_t x : {cin, cmp, cout_}) {
            if (!x) continue;
            if (ev_end && cudaEventRecord(ev_end, x) == cudaSuccess) cudaStreamWaitEvent(stream, ev_end, 0);
            cudaStreamSynchronize(x);
        }
        for (cudaStream_t x : {cin, cmp, cout_})
            if (x) cudaStreamDestroy(x);
        if (ev_start) cudaEventDestroy(ev_start);
        if (ev_end) cudaEventDestroy(ev_end);
        g_last_path = a.bf16 && a.dk == 128 && a.dv == 128 ? "tc" : "ffma";
        g_last_launches = launches;
    }
    if (base) cudaFreeAsync(base, stream);
    cudaError_t e2 = cudaStreamSynchronize(stream);
    if (s != KDA_OK) return s;
    if (e != cudaSuccess) return cuda_fail(e, "copy or stream operation");
    if (e2 != cudaSuccess) return cuda_fail(e2, "stream synchronize");
    return KDA_OK;
}

kda_status kda_fwd_noalloc(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* initial_state,
                           const int32_t* cu_seqlens, int32_t chunk, void* out,
                           float* final_state, const kda_dims* dims, void* stream_) {
    kda::NvtxRange nvtx_range("kda_fwd_noalloc");
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    kda::FwdArgs a;
    kda_status s = validate(q, k, v, log_alpha, beta, initial_state, cu_seqlens, chunk, out,
                            final_state, dims, true, &a);
    if (s != KDA_OK) return s;
    cudaStream_t stream = (cudaStream_t)stream_;
    if ((int64_t)a.N * a.H == 0) return KDA_OK;
    int launches = 0;
    if (!(a.bf16 && a.dk == 128 && a.dv == 128)) {
        // the CUDA-core path keeps everything on chip: no scratch at all
        g_last_path = "ffma";
        cudaError_t e = kda::launch_ffma(a, stream, &launches);
        g_last_launches = launches;
        return e == cudaSuccess ? KDA_OK : cuda_fail(e, "kernel launch");
    }
    // Segment plan of kda_fwd, with longer segments until the scratch fits.
    kda::TcPlan p = plan_segments(a);
    size_t b_segs, b_off, b_trans;
    size_t need = tc_scratch_bytes(a, p, &b_segs, &b_off, &b_trans);
    while (need > kNoAllocScratchBytes && p.segmented) {
        const int64_t nch_seq_max = ((int64_t)a.T + kda::kChunk - 1) / kda::kChunk;
        const int64_t nch_total = a.cu ? nch_seq_max + a.N : (int64_t)a.B * nch_seq_max;
        const int64_t seg = (int64_t)p.seg_chunks * 2;
        p.segmented = seg < nch_seq_max;
        p.seg_chunks = (int)std::min<int64_t>(p.segmented ? seg : std::max<int64_t>(nch_seq_max, 1),
                                              1 << 30);
        p.max_units = (int)(p.segmented ? (nch_total + p.seg_chunks - 1) / p.seg_chunks + a.N : a.N);
        need = tc_scratch_bytes(a, p, &b_segs, &b_off, &b_trans);
    }
    if (need > kNoAllocScratchBytes)
        return fail(KDA_ERR_UNSUPPORTED,
                    "kda_fwd_noalloc: %d sequences need %zu bytes of scratch, more than the "
                    "fixed %zu-byte array",
                    a.N, need, kNoAllocScratchBytes);
    char* ws = nullptr;
    cudaError_t e = noalloc_scratch(&ws);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-allocation scratch)");
    // Nothing in the scratch needs to start at zero: the segment-table kernel
    // writes every entry that is read later, pass 1 writes every transition the
    // scan reads, and the scan writes every incoming state pass 3 reads.
    kda::TcArgs t{};
    t.q = a.q;
    t.k = a.k;
    t.v = a.v;
    t.log_alpha = a.log_alpha;
    t.beta = a.beta;
    t.s0 = a.s0;
    t.cu = a.cu;
    t.out = a.out;
    t.s_final = a.s_final;
    t.gate = a.gate;
    t.snap_slots = a.snap_slots;
    t.snap_pool = a.snap_pool;
    t.snap_interval = a.snap_interval;
    t.snap_max = a.snap_max;
    t.snap_num_slots = a.snap_num_slots;
    t.B = a.B;
    t.T = a.T;
    t.H = a.H;
    t.N = a.N;
    t.segs = (kda::SegEntry*)ws;
    t.seg_off = (int32_t*)(ws + b_segs);
    t.n_units = t.seg_off + a.N + 1;
    t.trans = p.segmented ? (float*)(ws + b_segs + b_off) : nullptr;
    t.sin = p.segmented ? (float*)(ws + b_segs + b_off + b_trans) : nullptr;
    g_last_path = "tc";
    e = kda::launch_tc(t, p, stream, &launches);
    g_last_launches = launches;
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return KDA_OK;
}

kda_status kda_transition(const void* k, const void* v, const float* log_alpha,
                          const float* beta, const kda_dims* d, float* trans, void* stream) {
    kda::NvtxRange nvtx_range("kda_transition");
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    kda::FwdArgs a;
    kda_status st = validate_span_inputs(nullptr, k, v, log_alpha, beta, d, trans, false, &a);
    if (st != KDA_OK) return st;
    const void* ptrs[] = {k, v, log_alpha, beta, trans};
    const char* names[] = {"k", "v", "log_alpha", "beta", "trans"};
    st = check_accessible(ptrs, names, 5);
    if (st != KDA_OK) return st;
    const kda::TcPlan p = plan_segments(a);
    const size_t b_segs = ((size_t)p.max_units * sizeof(kda::SegEntry) + 255) & ~(size_t)255;
    const size_t b_off = ((size_t)(a.N + 1) * 4 + 4 + 255) & ~(size_t)255;
    const size_t b_trans = (size_t)p.max_units * a.H * 2 * 128 * 128 * sizeof(float);
    cudaStream_t cs = (cudaStream_t)stream;
    char* ws = nullptr;
    cudaError_t e = pool_alloc((void**)&ws, b_segs + b_off + b_trans, cs);
    if (e != cudaSuccess) return cuda_fail(e, "workspace allocation");
    kda::TcArgs t{};
    t.k = k;
    t.v = v;
    t.log_alpha = log_alpha;
    t.beta = beta;
    t.B = a.B;
    t.T = a.T;
    t.H = a.H;
    t.N = a.N;
    t.segs = (kda::SegEntry*)ws;
    t.seg_off = (int32_t*)(ws + b_segs);
    t.n_units = t.seg_off + a.N + 1;
    t.trans = (float*)(ws + b_segs + b_off);
    int launches = 0;
    g_last_path = "tc";
    e = kda::launch_transition(t, p, trans, cs, &launches);
    cudaFreeAsync(ws, cs);
    g_last_launches = launches;
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return KDA_OK;
}

size_t kda_span_workspace_bytes(const kda_dims* d) {
    if (!d || d->B < 1 || d->T < 0 || d->H < 1) return 0;
    kda::FwdArgs a;
    a.B = d->B;
    a.T = d->T;
    a.H = d->H;
    a.dk = a.dv = 128;
    a.N = d->B;
    a.cu = nullptr;
    return span_layout(a).total;
}

kda_status kda_span_transition(const void* q, const void* k, const void* v, const float* log_alpha,
                               const float* beta, const kda_dims* d, void* workspace,
                               size_t workspace_bytes, float* trans, void* stream) {
    kda::NvtxRange nvtx_range("kda_span_transition");
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    kda::FwdArgs a;
    kda_status st = validate_span_inputs(q, k, v, log_alpha, beta, d, trans, true, &a);
    if (st != KDA_OK) return st;
    const SpanWs w = span_layout(a);
    st = check_workspace(workspace, workspace_bytes, w.total);
    if (st != KDA_OK) return st;
    const int64_t tokens = (int64_t)a.B * a.T, n = tokens * a.H * 128;
    const Range rw = {(uintptr_t)workspace, (uintptr_t)workspace + w.total, "workspace"};
    const Range other[] = {{(uintptr_t)q, (uintptr_t)q + (q ? n * 2 : 0), "q"},
                           {(uintptr_t)k, (uintptr_t)k + (k ? n * 2 : 0), "k"},
                           {(uintptr_t)v, (uintptr_t)v + (v ? n * 2 : 0), "v"},
                           {(uintptr_t)log_alpha, (uintptr_t)log_alpha + (log_alpha ? n * 4 : 0),
                            "log_alpha"},
                           {(uintptr_t)beta, (uintptr_t)beta + (beta ? tokens * a.H * 4 : 0), "beta"},
                           {(uintptr_t)trans, (uintptr_t)trans + (uintptr_t)a.B * a.H * 2 * 128 * 128 * 4,
                            "trans"}};
    for (const Range& r : other)
        if (overlaps(rw, r)) return fail(KDA_ERR_ALIAS, "workspace overlaps %s", r.name);
    const void* wp[] = {q, k, v, log_alpha, beta, trans, workspace};
    const char* wn[] = {"q", "k", "v", "log_alpha", "beta", "trans", "workspace"};
    st = check_accessible(wp, wn, 7);
    if (st != KDA_OK) return st;
    kda::TcArgs t = span_args(a, w, (char*)workspace);
    int launches = 0;
    g_last_path = "tc";
    cudaError_t e = kda::launch_transition(t, w.p, trans, (cudaStream_t)stream, &launches);
    g_last_launches = launches;
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return KDA_OK;
}

kda_status kda_span_forward_ex(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta,
                               const float* initial_state, void* out, float* final_state,
                               const kda_dims* d, const void* workspace, size_t workspace_bytes,
                               const kda_fwd_opts* opts, void* stream) {
    kda::NvtxRange nvtx_range("kda_span_forward_ex");
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    kda::FwdArgs a;
    kda_status st = validate(q, k, v, log_alpha, beta, initial_state, nullptr, kda::kChunk, out,
                             final_state, d, false, &a);
    if (st != KDA_OK) return st;
    if (!(a.bf16 && a.dk == 128 && a.dv == 128))
        return fail(KDA_ERR_UNSUPPORTED, "kda_span_forward needs bf16 q/k/v with d_k = d_v = 128");
    const SpanWs w = span_layout(a);
    st = check_workspace(workspace, workspace_bytes, w.total);
    if (st != KDA_OK) return st;
    const int64_t tokens = (int64_t)a.B * a.T;
    const Range rw = {(uintptr_t)workspace, (uintptr_t)workspace + w.total, "workspace"};
    const Range outs[] = {{(uintptr_t)out, (uintptr_t)out + (out ? tokens * a.H * a.dv * 2 : 0), "out"},
                          {(uintptr_t)final_state,
                           (uintptr_t)final_state + (final_state ? (uintptr_t)a.N * a.H * 128 * 128 * 4 : 0),
                           "final_state"}};
    for (const Range& r : outs)
        if (overlaps(rw, r)) return fail(KDA_ERR_ALIAS, "workspace overlaps %s", r.name);
    if (opts && opts->snap && opts->snap_pool) {
        const kda_snap_spec* sp = opts->snap;
        const Range rp = {(uintptr_t)opts->snap_pool,
                          (uintptr_t)opts->snap_pool + (uintptr_t)std::max(sp->num_slots, 0) * a.H * 128 * 128 * 4,
                          "snap_pool"};
        if (overlaps(rw, rp)) return fail(KDA_ERR_ALIAS, "workspace overlaps snap_pool");
    }
    // option checks and the device-memory check of every caller buffer
    st = apply_opts(opts, q, k, v, log_alpha, beta, initial_state, nullptr, out, final_state, &a);
    if (st != KDA_OK) return st;
    const void* wp[] = {workspace};
    const char* wn[] = {"workspace"};
    st = check_accessible(wp, wn, 1);
    if (st != KDA_OK) return st;
    if ((int64_t)a.N * a.H == 0) return KDA_OK;
    kda::TcArgs t = span_args(a, w, (char*)workspace);
    t.q = q;
    t.s0 = initial_state;
    t.out = out;
    t.s_final = final_state;
    t.gate = a.gate;
    t.snap_slots = a.snap_slots;
    t.snap_pool = a.snap_pool;
    t.snap_interval = a.snap_interval;
    t.snap_max = a.snap_max;
    t.snap_num_slots = a.snap_num_slots;
    int launches = 0;
    g_last_path = "tc";
    cudaError_t e = kda::launch_tc(t, w.p, (cudaStream_t)stream, &launches, /*from_span=*/true);
    g_last_launches = launches;
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return KDA_OK;
}

kda_status kda_span_forward(const void* q, const void* k, const void* v, const float* log_alpha,
                            const float* beta, const float* initial_state, void* out,
                            float* final_state, const kda_dims* d, const void* workspace,
                            size_t workspace_bytes, void* stream) {
    return kda_span_forward_ex(q, k, v, log_alpha, beta, initial_state, out, final_state, d,
                               workspace, workspace_bytes, nullptr, stream);
}

kda_status kda_chunk_operands(const void* q, const void* k, const void* v, const float* log_alpha,
                              const float* beta, const kda_dims* d, void* images, void* stream) {
    kda::NvtxRange nvtx_range("kda_chunk_operands");
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    if (!d) return fail(KDA_ERR_INVALID_ARG, "dims is NULL");
    const int64_t nch = d->T > 0 ? ((int64_t)d->T + kda::kChunk - 1) / kda::kChunk : 0;
    const size_t bytes = (size_t)std::max<int64_t>(d->B, 0) * nch * std::max(d->H, 0) *
                         kda::kChunkImageBytes;
    kda::FwdArgs a;
    kda_status st = validate_span_inputs(q, k, v, log_alpha, beta, d, (const float*)images, true, &a,
                                         std::max<size_t>(bytes, 1), "images");
    if (st != KDA_OK) return st;
    const void* wp[] = {q, k, v, log_alpha, beta, images};
    const char* wn[] = {"q", "k", "v", "log_alpha", "beta", "images"};
    st = check_accessible(wp, wn, 6);
    if (st != KDA_OK) return st;
    if (nch == 0) return KDA_OK;
    // one segment per sequence: chunk c of sequence b is entry b * nch + c
    kda::TcPlan p;
    p.seg_chunks = (int)std::min<int64_t>(nch, 1 << 30);
    p.segmented = false;
    p.max_units = a.N;
    p.total_chunks = (int64_t)a.B * nch;
    const size_t b_segs = ((size_t)p.max_units * sizeof(kda::SegEntry) + 255) & ~(size_t)255;
    const size_t b_off = ((size_t)(a.N + 1) * 4 + 4 + 255) & ~(size_t)255;
    cudaStream_t cs = (cudaStream_t)stream;
    char* ws = nullptr;
    cudaError_t e = pool_alloc((void**)&ws, b_segs + b_off, cs);
    if (e != cudaSuccess) return cuda_fail(e, "workspace allocation");
    kda::TcArgs t{};
    t.q = q;
    t.k = k;
    t.v = v;
    t.log_alpha = log_alpha;
    t.beta = beta;
    t.B = a.B;
    t.T = a.T;
    t.H = a.H;
    t.N = a.N;
    t.segs = (kda::SegEntry*)ws;
    t.seg_off = (int32_t*)(ws + b_segs);
    t.n_units = t.seg_off + a.N + 1;
    t.dump = (uint8_t*)images;
    t.total_chunks = p.total_chunks;
    int launches = 0;
    g_last_path = "tc";
    e = kda::launch_dump(t, p, cs, &launches);
    cudaFreeAsync(ws, cs);
    g_last_launches = launches;
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return KDA_OK;
}

kda_status kda_apply_transitions(const float* trans, int32_t count, int32_t B, int32_t H,
                                 const float* initial_state, float* state_out, void* stream) {
    kda::NvtxRange nvtx_range("kda_apply_transitions");
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    if (count < 0 || B < 1 || H < 1)
        return fail(KDA_ERR_INVALID_ARG, "need count >= 0, B >= 1, H >= 1 (got %d, %d, %d)",
                    count, B, H);
    if (!state_out) return fail(KDA_ERR_INVALID_ARG, "state_out must be non-NULL");
    if (count > 0 && !trans) return fail(KDA_ERR_INVALID_ARG, "trans must be non-NULL");
    const void* ptrs[] = {trans, initial_state, state_out};
    const char* names[] = {"trans", "initial_state", "state_out"};
    for (int i = 0; i < 3; ++i)
        if (ptrs[i] && ((uintptr_t)ptrs[i] & 15u))
            return fail(KDA_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
    const uintptr_t st_bytes = (uintptr_t)B * H * 128 * 128 * 4;
    const Range rt = {(uintptr_t)trans, (uintptr_t)trans + (trans ? (uintptr_t)count * 2 * st_bytes : 0),
                      "trans"};
    const Range r0 = {(uintptr_t)initial_state, (uintptr_t)initial_state + (initial_state ? st_bytes : 0),
                      "initial_state"};
    const Range ro = {(uintptr_t)state_out, (uintptr_t)state_out + st_bytes, "state_out"};
    if (overlaps(ro, rt)) return fail(KDA_ERR_ALIAS, "state_out overlaps trans");
    if (overlaps(ro, r0) && !(ro.lo == r0.lo))
        return fail(KDA_ERR_ALIAS, "state_out partly overlaps initial_state");
    kda_status st = check_accessible(ptrs, names, 3);
    if (st != KDA_OK) return st;
    kda::ChainArgs c;
    c.trans = trans;
    c.off = nullptr;
    c.n_units = nullptr;
    c.count = count;
    c.B = B;
    c.H = H;
    c.s0 = initial_state;
    c.out = state_out;
    c.compose = 0;
    int launches = 0;
    g_last_path = "chain";
    cudaError_t e = kda::launch_chain(c, (cudaStream_t)stream, &launches);
    g_last_launches = launches;
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return KDA_OK;
}

kda_status kda_decode(const void* q, const void* k, const void* v, const float* log_alpha,
                      const float* beta, float* state, const int32_t* slots, void* out,
                      const void* out_gate, float* token_states, const kda_decode_dims* d,
                      void* stream) {
    kda::NvtxRange nvtx_range("kda_decode");
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    if (!d) return fail(KDA_ERR_INVALID_ARG, "dims is NULL");
    if (d->N < 0 || d->T < 0 || d->H < 1)
        return fail(KDA_ERR_INVALID_ARG, "need N >= 0, T >= 0, H >= 1 (got N=%d T=%d H=%d)", d->N,
                    d->T, d->H);
    if (d->qkv_dtype != KDA_F32 && d->qkv_dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "qkv_dtype must be KDA_F32 or KDA_BF16");
    if ((d->d_k != 64 && d->d_k != 128) || (d->d_v != 64 && d->d_v != 128))
        return fail(KDA_ERR_UNSUPPORTED, "d_k and d_v must be 64 or 128 (got %d, %d)", d->d_k,
                    d->d_v);
    if (slots && d->num_slots < 1)
        return fail(KDA_ERR_INVALID_ARG, "num_slots must be >= 1 with a slot table");
    const int64_t S = slots ? d->num_slots : d->N;
    const int64_t tokens = (int64_t)d->N * d->T;
    const int64_t e_in = d->qkv_dtype == KDA_BF16 ? 2 : 4;
    const int64_t nqk = tokens * d->H * d->d_k, nv = tokens * d->H * d->d_v;
    const int64_t dd = (int64_t)d->d_k * d->d_v;
    if ((int64_t)d->N * d->H == 0) return KDA_OK;
    if ((int64_t)d->N * d->H > INT32_MAX)
        return fail(KDA_ERR_UNSUPPORTED, "N * H = %lld exceeds 2^31 - 1",
                    (long long)d->N * d->H);
    if (!state) return fail(KDA_ERR_INVALID_ARG, "state must be non-NULL");
    if (tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !out))
        return fail(KDA_ERR_INVALID_ARG, "q, k, v, log_alpha, beta and out must be non-NULL");
    const void* ptrs[] = {q, k, v, log_alpha, beta, state, slots, out, token_states, out_gate};
    const char* names[] = {"q", "k", "v", "log_alpha", "beta", "state", "slots", "out",
                           "token_states", "out_gate"};
    for (int i = 0; i < 10; ++i) {
        if (ptrs[i] && ((uintptr_t)ptrs[i] & 15u) && i != 6)
            return fail(KDA_ERR_MISALIGNED, "%s is not 16-byte aligned", names[i]);
        if (i == 6 && ptrs[i] && ((uintptr_t)ptrs[i] & 3u))
            return fail(KDA_ERR_MISALIGNED, "slots is not 4-byte aligned");
    }
    const int64_t bytes[] = {nqk * e_in, nqk * e_in, nv * e_in, nqk * 4, tokens * d->H * 4,
                             S * d->H * dd * 4, (int64_t)d->N * 4, nv * e_in,
                             tokens * d->H * dd * 4, nv * e_in};
    Range r[10];
    for (int i = 0; i < 10; ++i)
        r[i] = {(uintptr_t)ptrs[i], (uintptr_t)ptrs[i] + (ptrs[i] ? bytes[i] : 0), names[i]};
    // written buffers (state, out, token_states) overlap nothing else
    for (int w : {5, 7, 8})
        for (int i = 0; i < 10; ++i)
            if (i != w && overlaps(r[w], r[i]))
                return fail(KDA_ERR_ALIAS, "%s overlaps %s", names[w], names[i]);
    kda_status st = check_accessible(ptrs, names, 10);
    if (st != KDA_OK) return st;
    kda::DecodeArgs a;
    a.q = q;
    a.k = k;
    a.v = v;
    a.log_alpha = log_alpha;
    a.beta = beta;
    a.state = state;
    a.slots = slots;
    a.out = out;
    a.gate = out_gate;
    a.token_states = token_states;
    a.N = d->N;
    a.T = d->T;
    a.H = d->H;
    a.dk = d->d_k;
    a.dv = d->d_v;
    a.num_slots = (int32_t)S;
    a.bf16 = d->qkv_dtype == KDA_BF16;
    cudaError_t e = kda::status_word(&a.status);
    if (e != cudaSuccess) return cuda_fail(e, "device status word");
    int launches = 0;
    g_last_path = "decode";
    e = kda::launch_decode(a, (cudaStream_t)stream, &launches);
    g_last_launches = launches;
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
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

void kda_profile_enable(int32_t on) { profiler().on.store(on != 0); }

kda_status kda_profile_read(double* total_ms, int64_t* launches, int32_t n) {
    g_last_error[0] = 0;
    Profiler& P = profiler();
    std::lock_guard<std::mutex> lock(P.mu);
    cudaError_t err = cudaSuccess;
    for (const Profiler::Mark& m : P.pending) {
        float ms = 0.f;
        cudaError_t e = cudaEventSynchronize(m.b);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, m.a, m.b);
        if (e != cudaSuccess) err = e;
        P.total_ms[m.slot] += ms;
        P.count[m.slot] += 1;
        P.free_events.push_back(m.a);
        P.free_events.push_back(m.b);
    }
    P.pending.clear();
    for (int i = 0; i < kda::NUM_SLOTS && i < n; ++i) {
        if (total_ms) total_ms[i] = P.total_ms[i];
        if (launches) launches[i] = P.count[i];
        P.total_ms[i] = 0.0;
        P.count[i] = 0;
    }
    if (err != cudaSuccess) return cuda_fail(err, "profile event");
    return KDA_OK;
}

const char* kda_profile_slot_name(int32_t slot) {
    static const char* names[] = {"seg_setup", "tc_pass1_transitions", "seg_scan",
                                  "tc_pass3_forward", "ffma_forward", "decode_step",
                                  "transition_chain"};
    return (slot >= 0 && slot < kda::NUM_SLOTS) ? names[slot] : "";
}

kda_status kda_selftest_wait(uint64_t timeout_ns, int32_t arrive, void* stream) {
    g_last_error[0] = 0;
    g_last_launches = 0;
    g_last_path = "";
    if (timeout_ns < 1000 || timeout_ns > 100000000ull)
        return fail(KDA_ERR_INVALID_ARG, "timeout_ns must lie in [1e3, 1e8] (got %llu)",
                    (unsigned long long)timeout_ns);
    cudaError_t e = kda::launch_wait_probe(timeout_ns, arrive != 0, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    g_last_launches = 1;
    return KDA_OK;
}

kda_status kda_check_device(void* stream) {
    g_last_error[0] = 0;
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    int code = 0;
    e = kda::tc_take_status(&code);
    if (e != cudaSuccess) return cuda_fail(e, "device status read");
    if (code == kda::ERR_WAIT_TIMEOUT) return fail(KDA_ERR_DEVICE_TIMEOUT, "a bounded device wait gave up");
    if (code == kda::ERR_SEG_OVERFLOW)
        return fail(KDA_ERR_INVALID_ARG, "segment table overflow: malformed cu_seqlens");
    if (code == kda::ERR_BAD_SLOT)
        return fail(KDA_ERR_INVALID_ARG, "a decode slot index lies outside the state pool");
    if ((code & 0xff) == kda::ERR_DEBUG_INDEX)
        return fail(KDA_ERR_CUDA, "debug build: a device index check failed (kda_tc.cu line %d)",
                    code >> 8);
    if ((code & 0xff) == kda::ERR_DEBUG_GUARD)
        return fail(KDA_ERR_CUDA, "debug build: guard band %d of the kda_fwd workspace was overwritten",
                    code >> 8);
    if (code) return fail(KDA_ERR_CUDA, "device status %d", code);
    return KDA_OK;
}

}  // extern "C"
