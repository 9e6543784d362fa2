/*
 * kda.h -- C ABI of libkda.so: the Kimi Delta Attention (KDA) chunked forward
 * pass on NVIDIA B200 (sm_100a).
 *
 * The operation (aiblin.ru, "Kimi K3 -- открытая модель, которая обошла
 * закрытых лидеров рынка", section "Как хранить миллион токенов в памяти"):
 * a fixed-size state S (d_k x d_v, fp32) replaces the KV cache and is rewritten
 * at every token -- part of the old content is erased, then new content is
 * written with strength beta in (0,1); a per-channel forget coefficient alpha,
 * clamped to [e^-5, 1], decays the old content.  Read as
 *
 *     alpha_t = exp(clamp(log_alpha_t, -5, 0))                (d_k vector)
 *     S_t     = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t     = S_t^T q_t
 *
 * The library evaluates it chunkwise (section "Как распараллелили
 * последовательное обновление" of the same page): all tokens of a 64-token
 * chunk in parallel, then the state passed from chunk to chunk; long sequences
 * are additionally cut into segments whose state transitions (a local state
 * plus a d_k x d_k transition matrix, S_out = M S_in + B) are computed in
 * parallel on one GPU and chained by a scan.  No q scaling, no k
 * normalisation, no beta or gate activation happens inside: the caller passes
 * k, beta and log_alpha as the recurrence consumes them (log_alpha is clamped
 * inside).
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes.  Every argument error is detected on the host before any
 * launch; such a call writes nothing. */
typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,    /* null/negative/inconsistent argument, host pointer where a
                                   device pointer is required, bad cu_seqlens length        */
    KDA_ERR_UNSUPPORTED = 2,    /* valid but not implemented: d_k/d_v not in {64,128}, chunk != 64 */
    KDA_ERR_MISALIGNED = 3,     /* a tensor pointer is not 16-byte aligned                   */
    KDA_ERR_ALIAS = 4,          /* out or final_state overlaps an input (final_state ==
                                   initial_state exactly is allowed)                         */
    KDA_ERR_CUDA = 5,           /* a CUDA runtime call or kernel launch failed               */
    KDA_ERR_DEVICE_TIMEOUT = 6  /* a bounded inter-block wait on the device gave up; the
                                   outputs of that call are undefined                        */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1 } kda_dtype;

/* Shapes.  Without cu_seqlens: B sequences of T tokens each (N = B).
 * With cu_seqlens: B must be 1, T is the packed token count and
 * N = num_seqs sequences are given by cu_seqlens. */
typedef struct {
    int32_t B;          /* batch (>= 1; 1 when packed)                          */
    int32_t T;          /* tokens per sequence, or packed total (>= 0)          */
    int32_t H;          /* heads (>= 1)                                         */
    int32_t d_k;        /* key/query channels: 64 or 128                        */
    int32_t d_v;        /* value channels: 64 or 128                            */
    int32_t num_seqs;   /* N when cu_seqlens != NULL (>= 1); ignored otherwise  */
    int32_t qkv_dtype;  /* kda_dtype of q, k, v and out                          */
} kda_dims;

/*
 * kda_fwd -- chunked KDA forward on device buffers, asynchronous on `stream`.
 *
 * All tensors are dense, row-major (last index fastest), 16-byte aligned,
 * device-resident, owned by the caller:
 *   q            [B, T, H, d_k]   qkv_dtype
 *   k            [B, T, H, d_k]   qkv_dtype
 *   v            [B, T, H, d_v]   qkv_dtype
 *   log_alpha    [B, T, H, d_k]   fp32, clamped to [-5, 0] inside
 *   beta         [B, T, H]        fp32, used as given
 *   initial_state[N, H, d_k, d_v] fp32, or NULL for a zero state
 *   cu_seqlens   [N + 1]          int32 on the device, or NULL (then N = B);
 *                                 cu[0] = 0, non-decreasing, cu[N] = T.  The
 *                                 library does not read it on the host: a
 *                                 malformed table is undefined behaviour.
 *   chunk        tokens per chunk; must be 64
 *   out          [B, T, H, d_v]   qkv_dtype (bf16 rounded to nearest even)
 *   final_state  [N, H, d_k, d_v] fp32, or NULL; may be the same pointer as
 *                                 initial_state (read before written)
 *   stream       a cudaStream_t (NULL = legacy default stream)
 *
 * The state restarts at every sequence start (from initial_state[n] or zero)
 * and a chunk never straddles two sequences.  A zero-length sequence gives
 * final_state[n] = initial_state[n].
 *
 * Temporary device memory (the segment table, and for long sequences the
 * segment transitions and incoming states, 192 KiB per segment and head, and a
 * cache of every chunk's operands of the output pass, which the transition pass
 * prepares: about 1030 bytes per token and head) is taken stream-ordered
 * (cudaMallocFromPoolAsync / cudaFreeAsync on `stream`) from a memory pool the
 * library creates once per device and keeps for the life of the process; freed
 * blocks stay reserved in that pool for the next call.  Nothing else persists between calls apart from
 * cached kernel attributes and the device status word (kda_check_device).
 * Errors: see kda_status; a kernel fault surfaces at the caller's next
 * synchronisation, as with any CUDA launch.
 */
kda_status kda_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                   const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                   int32_t chunk, void* out, float* final_state, const kda_dims* dims,
                   void* stream);

/* Where kda_fwd_snap / kda_fwd_ex write state snapshots. */
typedef struct {
    int32_t interval;   /* tokens between snapshots: a positive multiple of 64 (chunk) */
    int32_t max_snaps;  /* snapshots per sequence the slot table has room for (>= 0)  */
    int32_t num_slots;  /* rows of the snapshot pool (>= 0)                           */
} kda_snap_spec;

/*
 * kda_fwd_snap -- kda_fwd that also writes the state at chunk boundaries, for
 * a prefix cache.
 *
 * KDA places new demands on prefix caching, and its authors released an
 * implementation of it for a public serving engine (habr.com article 1063882
 * on the Kimi K3 technical report, the paragraph on KDA and AttnRes).  A
 * cached prefix of a linear-attention layer is a state, not a list of keys and
 * values, so a request that shares a prefix resumes from the state at its end.
 * This call writes such states while it runs the forward pass.
 *
 * Arguments and results of kda_fwd, plus:
 *   snap        interval, max_snaps, num_slots (above)
 *   snap_slots  [N, max_snaps] int32 on the device: snapshot j of sequence n,
 *               the state after its first (j+1)*interval tokens (so only for
 *               (j+1)*interval <= length of the sequence), is written to row
 *               snap_slots[n*max_snaps + j] of snap_pool when that entry is
 *               >= 0; entries < 0 request nothing.  An entry >= num_slots
 *               skips that snapshot and sets the device status word
 *               (kda_check_device: KDA_ERR_INVALID_ARG).  Two requested
 *               snapshots must not name the same row.
 *   snap_pool   [num_slots, H, d_k, d_v] fp32 on the device, 16-byte
 *               aligned; rows not named are left as they were.  It may not
 *               overlap any other buffer.
 * A snapshot is the state after those tokens: the final_state kda_fwd
 * returns for the sequence cut there (bit for bit when neither call splits
 * the sequence into segments, else up to rounding), and kda_fwd continued
 * from it reproduces the rest of the sequence.  Writing snapshots changes no
 * other result.  max_snaps == 0 or num_slots == 0 is a plain kda_fwd.
 * Temporary memory: as kda_fwd.
 */
kda_status kda_fwd_snap(const void* q, const void* k, const void* v, const float* log_alpha,
                        const float* beta, const float* initial_state,
                        const int32_t* cu_seqlens, int32_t chunk, void* out, float* final_state,
                        const kda_dims* dims, const kda_snap_spec* snap,
                        const int32_t* snap_slots, float* snap_pool, void* stream);

/* Optional parts of a forward call (kda_fwd_ex). */
typedef struct {
    const void* out_gate;         /* [B, T, H, d_v] qkv_dtype, or NULL              */
    const kda_snap_spec* snap;    /* NULL: no snapshots                             */
    const int32_t* snap_slots;    /* as in kda_fwd_snap (used when snap != NULL)    */
    float* snap_pool;             /* as in kda_fwd_snap (used when snap != NULL)    */
} kda_fwd_opts;

/*
 * kda_fwd_ex -- kda_fwd with the optional parts of a KDA layer's forward.
 *
 * out_gate: the gate that follows the attention in KDA blocks (aiblin.ru page
 * named at the top, in its description of the layer stack: after the
 * attention a further filter decides which share of the retrieved information
 * passes on to the model's main stream, in the Gated MLA blocks and in the
 * KDA blocks alike).  The caller computes the gate (its projection and
 * activation are outside this library) and passes its values; the library
 * multiplies them into the output before the single rounding to qkv_dtype:
 *     out[t, h, c] = o[t, h, c] * out_gate[t, h, c]
 * Same layout as out, 16-byte aligned, device memory; it may not overlap out
 * or final_state.  The gate does not enter the state.
 * snap, snap_slots, snap_pool: prefix-cache snapshots exactly as in
 * kda_fwd_snap.  opts == NULL (or all members NULL) is a plain kda_fwd.
 */
kda_status kda_fwd_ex(const void* q, const void* k, const void* v, const float* log_alpha,
                      const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                      int32_t chunk, void* out, float* final_state, const kda_dims* dims,
                      const kda_fwd_opts* opts, void* stream);

/*
 * kda_fwd_host -- the same computation on HOST buffers (same shapes/layouts;
 * cu_seqlens is a host array here).  Copies the inputs to the device (one
 * cudaMemcpyAsync per tensor; pinned host memory makes them asynchronous),
 * runs kda_fwd on `stream`, copies out/final_state back and synchronises the
 * stream before returning.  Device buffers come from the stream-ordered pool.
 *
 * One sequence longer than 131 072 tokens (B = 1, cu_seqlens NULL) is run as
 * a pipeline of spans of that many tokens: the state after span r is exact
 * (fp32) and depends on spans 0..r only, so span r's outputs are copied back
 * while later spans are still being copied in.  The call creates three
 * streams for this (copy in, compute, copy out), which wait for `stream`
 * first and which `stream` waits for at the end.  Results are those of
 * kda_fwd called span by span with the state carried between the calls; they
 * agree with one kda_fwd over the whole sequence within rounding (the spans
 * change where the tensor-core path cuts the sequence into segments).
 */
kda_status kda_fwd_host(const void* q, const void* k, const void* v, const float* log_alpha,
                        const float* beta, const float* initial_state,
                        const int32_t* cu_seqlens, int32_t chunk, void* out,
                        float* final_state, const kda_dims* dims, void* stream);

/*
 * kda_fwd_noalloc -- kda_fwd for callers that cannot allocate device memory.
 *
 * (The pages describe no such entry point; it is an addition of this library.)
 * Some callers must not allocate on the call path: a serving loop whose device
 * memory is reserved up front by another allocator, a process whose memory
 * budget leaves nothing to grow a pool, or code that cannot afford the latency
 * or implicit synchronisation an allocation may bring.  kda_fwd takes its
 * temporaries from a stream-ordered pool; this entry point takes them instead
 * from a fixed 32 MiB scratch array compiled into the library, which every GPU
 * that loads the library holds until the process exits.  It calls no
 * cudaMalloc, cudaFree or allocating library routine.
 *
 * Arguments, layouts, ownership and results are those of kda_fwd.  The segment
 * split of long sequences is coarsened (longer segments) until its temporaries
 * fit in the array; a call whose segment table alone does not fit (about a
 * million sequences) returns KDA_ERR_UNSUPPORTED and launches nothing.
 *
 * Every call shares the one array, which keeps the previous call's contents
 * (nothing in it has to start at zero).  Calls whose kernels overlap on the GPU
 * -- on two streams, or from two host threads -- race on the array: order them
 * on one stream or synchronise between them.  The first call on a device looks
 * up the array's device address (cudaGetSymbolAddress, with that device
 * current); make that first call before any stream capture on the device.
 */
kda_status kda_fwd_noalloc(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, const float* initial_state,
                           const int32_t* cu_seqlens, int32_t chunk, void* out,
                           float* final_state, const kda_dims* dims, void* stream);

/* Shapes of a decode / verify step. */
typedef struct {
    int32_t N;          /* sequences in the step (>= 0)                             */
    int32_t T;          /* new tokens per sequence (>= 0; meant for 1..16)          */
    int32_t H;          /* heads (>= 1)                                             */
    int32_t d_k;        /* 64 or 128                                                */
    int32_t d_v;        /* 64 or 128                                                */
    int32_t num_slots;  /* rows of the state pool when slots != NULL (>= 1); else N */
    int32_t qkv_dtype;  /* kda_dtype of q, k, v and out                             */
} kda_decode_dims;

/*
 * kda_decode -- a few new tokens per sequence on a resident state, in place.
 *
 * The same recurrence as kda_fwd (section "Как хранить миллион токенов в
 * памяти" of the page named at the top), evaluated token by token as in
 * generation: a decoder passes T = 1; a speculative-decoding verifier passes
 * the T drafted tokens at once (the same page, in its account of the training
 * pipeline, describes an auxiliary draft model whose proposed tokens the main
 * model confirms in batches).  Equal to
 * kda_fwd on the same tokens with initial_state = final_state = state, but
 * without a 64-token chunk per call: the work is one read and one write of the
 * state (64 KiB of fp32 per head at d_k = d_v = 128) plus the tokens.
 *
 * Tensors are dense, row-major, 16-byte aligned, device-resident, owned by
 * the caller:
 *   q, k         [N, T, H, d_k]   qkv_dtype
 *   v            [N, T, H, d_v]   qkv_dtype
 *   log_alpha    [N, T, H, d_k]   fp32, clamped to [-5, 0] inside
 *   beta         [N, T, H]        fp32, used as given
 *   state        [S, H, d_k, d_v] fp32 (S = num_slots with slots, else N):
 *                                 read, then overwritten with the state after
 *                                 the T tokens
 *   slots        [N] int32 on the device, or NULL (sequence n uses state row
 *                n).  Row slots[n] of the pool holds sequence n's state; -1
 *                marks a padding entry, which reads and writes nothing (its
 *                out rows are left as they were).  Other values outside
 *                [0, num_slots) skip the sequence the same way and set the
 *                device status word (kda_check_device: KDA_ERR_INVALID_ARG).
 *                Two sequences must not name the same slot.
 *   out          [N, T, H, d_v]   qkv_dtype (bf16 rounded to nearest even)
 *   out_gate     [N, T, H, d_v]   qkv_dtype, or NULL: output gate, as in
 *                                 kda_fwd_ex (out = o * out_gate)
 *   token_states [N, T, H, d_k, d_v] fp32, or NULL: the state after each of
 *                the T tokens, so that a verifier that accepts only the first
 *                m tokens can continue from token_states[n][m-1]
 *
 * No buffer may overlap another.  Allocates nothing; one kernel launch.
 */
kda_status kda_decode(const void* q, const void* k, const void* v, const float* log_alpha,
                      const float* beta, float* state, const int32_t* slots, void* out,
                      const void* out_gate, float* token_states, const kda_decode_dims* dims,
                      void* stream);

/*
 * kda_transition -- the affine map each sequence applies to its state.
 *
 * The chunk-parallel section of the page named at the top: a span of tokens
 * acts on the state that enters it as S_out = M S_in + B, with B the span's
 * local state (from a zero incoming state) and M a token-dependent d_k x d_k
 * transition matrix, so spans can be processed independently and chained
 * afterwards.  This entry point returns (M, B) for each of the B sequences of
 * [B, T, H, *] k, v, log_alpha, beta (no cu_seqlens; q is not needed); with
 * kda_apply_transitions it is the exchange step of context parallelism, where
 * each GPU holds one span of a long sequence.
 *
 *   k, v       [B, T, H, 128] bf16;  log_alpha [B, T, H, 128] fp32;  beta [B, T, H]
 *   trans      [B, H, 2, 128, 128] fp32, written: trans[b][h][0] = B^T (d_v x d_k),
 *              trans[b][h][1] = M^T (d_k x d_k), i.e. S_out^T = S_in^T M^T + B^T
 * Only bf16 with d_k = d_v = 128 (KDA_ERR_UNSUPPORTED otherwise).  Long spans
 * are cut into segments whose transitions are computed in parallel and then
 * composed in fp32.  Temporary memory as kda_fwd.  trans may not overlap an
 * input.
 */
kda_status kda_transition(const void* k, const void* v, const float* log_alpha,
                          const float* beta, const kda_dims* dims, float* trans, void* stream);

/*
 * kda_apply_transitions -- the state after a chain of spans.
 *
 *   trans          [count, B, H, 2, 128, 128] fp32: transitions of consecutive
 *                  spans (as kda_transition writes them), span 0 first
 *   initial_state  [B, H, 128, 128] fp32 (d_k x d_v), or NULL for zero
 *   state_out      [B, H, 128, 128] fp32, written with the state after the
 *                  `count` spans: S <- M_j S + B_j for j = 0 .. count-1 (fp32).
 *                  count = 0 copies initial_state (or writes zero).  It may be
 *                  the same buffer as initial_state, not otherwise overlap it,
 *                  and may not overlap trans.
 * With the spans of a sequence spread over ranks, rank r passes the gathered
 * transitions of ranks 0 .. r-1 and gets its incoming state.
 */
kda_status kda_apply_transitions(const float* trans, int32_t count, int32_t B, int32_t H,
                                 const float* initial_state, float* state_out, void* stream);

/*
 * Context-parallel spans with shared work.  A rank that holds one span of B
 * sequences first computes the span's transition (to exchange), then -- once it
 * knows its incoming state -- the span's forward pass.  Both need the same
 * per-segment transitions and per-chunk operands, so the transition call can
 * leave them in a caller-owned workspace for the forward call, which then runs
 * only the segment scan and the output pass.
 *
 * kda_span_workspace_bytes: bytes of that workspace for these dims (B, T, H;
 *   d_k = d_v = 128, bf16, no cu_seqlens); 0 for invalid dims.
 * kda_span_transition: kda_transition that also fills `workspace` (device,
 *   256-byte aligned, at least kda_span_workspace_bytes, not overlapping any
 *   argument) with the segment table, the segment transitions and, for a span
 *   cut into segments, every chunk's operands of the output pass (W, the decayed
 *   keys, the gated queries, the intra-chunk query-key matrix, T diag(beta) and
 *   the chunk decay: about 1030 bytes per token and head).  It takes the span's q
 *   as well (same layout as k).
 * kda_span_forward: kda_fwd on the same span (same k, v, log_alpha, beta and
 *   dims; q, initial_state, out, final_state as in kda_fwd) that takes the
 *   workspace's contents instead of recomputing them.  It computes exactly as
 *   kda_fwd does on the span, so the results are equal bit for bit.
 *   If the workspace was not filled by kda_span_transition on the same inputs
 *   the results are undefined.  It reads the workspace only, so one transition
 *   may serve several forward calls (e.g. retries).
 * kda_span_forward_ex: kda_span_forward with the options of kda_fwd_ex (output
 *   gate, prefix-cache snapshots), checked as there; the workspace may not
 *   overlap snap_pool either.  Snapshot positions count tokens from the start
 *   of the span, so a rank whose span starts at a multiple of the interval
 *   takes snapshots at the same sequence positions as a whole-sequence call.
 *   opts == NULL is kda_span_forward.
 */
size_t kda_span_workspace_bytes(const kda_dims* dims);
kda_status kda_span_transition(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta, const kda_dims* dims,
                               void* workspace, size_t workspace_bytes, float* trans, void* stream);
kda_status kda_span_forward(const void* q, const void* k, const void* v, const float* log_alpha,
                            const float* beta, const float* initial_state, void* out,
                            float* final_state, const kda_dims* dims, const void* workspace,
                            size_t workspace_bytes, void* stream);
kda_status kda_span_forward_ex(const void* q, const void* k, const void* v,
                               const float* log_alpha, const float* beta,
                               const float* initial_state, void* out, float* final_state,
                               const kda_dims* dims, const void* workspace, size_t workspace_bytes,
                               const kda_fwd_opts* opts, void* stream);

/*
 * kda_chunk_operands -- diagnostic: the chunkwise operands of the forward pass.
 *
 * The per-chunk quantities of the chunkwise form (section "Как распараллелили
 * последовательное обновление" of the page named at the top: all tokens of a chunk
 * at once, then the state handed on), exactly as the tensor-core forward pass
 * computes them and hands them to its state products, written out so they can be
 * checked one by one.  For B sequences of T tokens (q, k, v, log_alpha, beta as in
 * kda_fwd; bf16, d_k = d_v = 128, no cu_seqlens), chunk c of sequence b and head h
 * (c < ceil(T/64)) gets entry (b * ceil(T/64) + c) * H + h of `images`, 74 240 bytes
 * of bf16 operand images in their shared-memory layouts (128-byte swizzle: in a
 * K-major tile of R rows, element (r, k) sits at byte (k / 64) R 128 + (r / 8) 1024 +
 * (r % 8) 128 + (((k % 64) / 8) ^ (r % 8)) 16 + (k % 8) 2; an MN-major tile of K rows
 * is the same with (r, k) -> (k, mn)), with g the in-chunk cumulative clamped
 * log-gate and T = (I + A)^-1 as in the chunkwise form:
 *   [0, 16384)       W^T, W = T diag(beta) (K e^g): MN-major, K rows = channels
 *   [16384, 32768)   U'^T, U' = T diag(beta) V: [128][64], the 16-byte piece p of
 *                    row e at e 128 + ((p ^ (e % 8)) 16)
 *   [32768, 49152)   K_dec = K e^(g_last - g): MN-major, K rows = tokens
 *   [49152, 65536)   Q~ = Q e^g: K-major, 64 rows
 *   [65536, 73728)   P = lower-inclusive (Q e^g)(K e^-g)^T: K-major 64 x 64
 *   [73728, 74240)   gamma = e^(g_last), fp32 [128]
 * Rows past a sequence's end are those of identity steps.  images: device,
 * 16-byte aligned, B ceil(T/64) H 74240 bytes, not overlapping an input.
 * Temporary memory as kda_fwd.  Only the operands; no state chain runs.
 */
kda_status kda_chunk_operands(const void* q, const void* k, const void* v,
                              const float* log_alpha, const float* beta, const kda_dims* dims,
                              void* images, void* stream);

/* Static description of a status code. */
const char* kda_status_string(kda_status s);

/* Detail of the last error raised on the calling host thread ("" if none). */
const char* kda_last_error(void);

/* Number of kernel launches the last kda_fwd / kda_decode call on this host
 * thread issued. */
int32_t kda_last_launch_count(void);

/* Kernel family the last call on this host thread used: "ffma" (fp32
 * CUDA-core path), "tc" (tcgen05 tensor-core path), "decode" (kda_decode),
 * "chain" (kda_apply_transitions) or "" (no launch). */
const char* kda_last_path(void);

/* Synchronises `stream`, then reads and clears the current device's status
 * word, which kernels set when a bounded wait gives up (KDA_ERR_DEVICE_TIMEOUT),
 * the device-built segment table would overflow because cu_seqlens is malformed,
 * or a kda_decode slot index lay outside the state pool (both KDA_ERR_INVALID_ARG).
 * In a library built with -DKDA_DEBUG the kernels also check the indices they take
 * from device-built tables before using them; a failed check reports KDA_ERR_CUDA
 * with the source line in kda_last_error().  KDA_OK when none of these happened
 * since the last check. */
kda_status kda_check_device(void* stream);

/*
 * kda_selftest_wait -- exercises the failure path of the kernels' bounded waits.
 *
 * (No counterpart on the pages; a test aid of this library.)  Every wait of the
 * tensor-core kernels on an mbarrier (a tensor-core product, a TMA copy, the other
 * warp group's hand-off) is bounded in wall time; when the bound passes, the
 * kernel records KDA_ERR_DEVICE_TIMEOUT in the device status word and returns
 * instead of spinning.  This launches one thread that waits through that same
 * code on an mbarrier of arrival count 1: with arrive != 0 it arrives first and
 * the wait completes at once; with arrive == 0 nothing ever arrives, so the wait
 * gives up after timeout_ns nanoseconds (1e3 .. 1e8, else KDA_ERR_INVALID_ARG)
 * and the next kda_check_device reports KDA_ERR_DEVICE_TIMEOUT.  Nothing else is
 * in flight in that kernel, so the context stays usable.  Asynchronous on stream.
 */
kda_status kda_selftest_wait(uint64_t timeout_ns, int32_t arrive, void* stream);

/* Optional launch timing (off by default).  While enabled, every kda_fwd and
 * kda_decode call records a CUDA event on its stream before and after each
 * internal kernel launch.  kda_profile_read synchronises those events, writes for each of the
 * first n kernel slots the summed duration in milliseconds and the number of
 * launches since the previous read, then resets the sums.  Slots: 0 segment
 * table, 1 pass 1 (segment transitions), 2 segment scan, 3 pass 3 (forward),
 * 4 CUDA-core forward, 5 decode step, 6 transition chain;
 * kda_profile_slot_name gives their names. */
void kda_profile_enable(int32_t on);
kda_status kda_profile_read(double* total_ms, int64_t* launches, int32_t n);
const char* kda_profile_slot_name(int32_t slot);

#ifdef __cplusplus
}
#endif
#endif /* KDA_H_ */
