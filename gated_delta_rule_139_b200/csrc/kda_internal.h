// Internal declarations shared by the C-ABI layer and the kernels of libkda.so.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

namespace kda {

constexpr int kChunk = 64;       // tokens per chunk
constexpr int kMaxDevices = 64;  // size of per-device attribute caches

// NVTX range over a host scope (header-only NVTX 3: a no-op unless a profiler is
// attached), so a timeline shows which public call and which pass issued a kernel.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

// Kernel slots of the optional per-launch timing (kda_profile_*).
enum KernelSlot : int { SLOT_SETUP = 0, SLOT_PASS1 = 1, SLOT_SCAN = 2, SLOT_PASS3 = 3, SLOT_FFMA = 4,
                        SLOT_DECODE = 5, SLOT_CHAIN = 6, NUM_SLOTS = 7 };

// Device status codes (first error wins; read and cleared by kda_check_device).
// ERR_DEBUG_INDEX (KDA_DEBUG builds only) carries the failing check's source line
// in the bits above the low byte, ERR_DEBUG_GUARD (likewise) the overwritten guard
// band's index.
enum DeviceStatus : int { ERR_WAIT_TIMEOUT = 1, ERR_SEG_OVERFLOW = 2, ERR_BAD_SLOT = 3,
                          ERR_DEBUG_INDEX = 4, ERR_DEBUG_GUARD = 5 };

// Guard bands of the debug build's kda_fwd workspace: kGuardBytes of kGuardWord
// before and after each of its buffers, checked after the launches.
constexpr size_t kGuardBytes = 4096;
constexpr uint32_t kGuardWord = 0xA5A5A5A5u;
constexpr int kMaxGuards = 8;
struct GuardBands {
    const uint32_t* band[kMaxGuards];
    int n;
};
// Checks every band (kGuardBytes each) on the device; an overwritten band i records
// ERR_DEBUG_GUARD | (i << 8) in the status word.  Not counted as a launch.
cudaError_t launch_guard_check(const GuardBands& g, cudaStream_t stream);
// Device address of the current device's status word.
cudaError_t status_word(int** p);
// Records a CUDA event on `stream` before (begin=true) or after a launch of
// `slot` when timing is enabled; no-op otherwise.
void profile_mark(int slot, bool begin, cudaStream_t stream);

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
    const void* gate = nullptr;  // optional output gate [B, T, H, dv] (dtype of out): out = o * gate
    // optional state snapshots (kda_fwd_snap): snapshot j of sequence n, the
    // state after its first (j+1)*snap_interval tokens, goes to pool row
    // snap_slots[n*snap_max + j] when that entry is >= 0
    const int32_t* snap_slots = nullptr;  // [N, snap_max] device
    float* snap_pool = nullptr;           // [snap_num_slots, H, dk, dv]
    int32_t snap_interval = 0, snap_max = 0, snap_num_slots = 0;
    int* status = nullptr;                // device status word (set when snapshots are on)
};

// CUDA-core chunkwise path (exact fp32 arithmetic on fp32 or bf16 inputs).
cudaError_t launch_ffma(const FwdArgs& a, cudaStream_t stream, int* launches);

// One segment of one sequence: tokens [t_begin, t_end), whole chunks except
// possibly the sequence's last.
struct SegEntry {
    int64_t t_begin, t_end;
    int32_t n;       // sequence
    int32_t j;       // segment index inside the sequence
    int32_t last;    // 1 for the sequence's last segment
    int32_t pad;
    int64_t c_base;  // index of the segment's first chunk among all chunks of all sequences
};

// Tensor-core path arguments: the validated forward arguments plus workspace.
struct TcArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* log_alpha;
    const float* beta;
    const float* s0;
    const int32_t* cu;
    void* out;
    float* s_final;
    int32_t B, T, H, N;
    SegEntry* segs;     // [max_units]
    int32_t* seg_off;   // [N+1]: first unit of each sequence
    int32_t* n_units;   // [1]
    float* trans;       // [max_units, H, 2, 128, 128]: B^T then M^T of each segment
    float* sin;         // [max_units, H, 128, 128]: S_in^T of each segment
    const void* gate = nullptr;  // optional output gate, as in FwdArgs
    int32_t trans_all = 0;       // pass 1 also for each sequence's last segment
    uint8_t* dump = nullptr;     // operand dump: [total_chunks][H][kChunkImageBytes] (launch_dump)
    uint8_t* cache = nullptr;    // chunk cache: [total_chunks][H][kCacheEntryBytes] (pass 1 writes,
                                 // pass 3 reads); nullptr: pass 3 recomputes every chunk's operands
    int64_t total_chunks = 0;    // chunks the dump / cache holds per head
    // optional state snapshots, as in FwdArgs
    const int32_t* snap_slots = nullptr;
    float* snap_pool = nullptr;
    int32_t snap_interval = 0, snap_max = 0, snap_num_slots = 0;
};

// Bytes of one chunk's operand images as the operand dump writes them (per chunk
// and head): the bf16 images of W^T, U'^T, K_dec, Q~ (16 KB each), P (8 KB) and
// the fp32 chunk decay gamma (512 B).
constexpr size_t kChunkImageBytes = 74240;
// Bytes of one chunk's entry in the chunk cache that pass 1 leaves for pass 3 (per
// chunk and head): W^T, K_dec, Q~ (16 KB each), P, T diag(beta) (8 KB each), gamma.
constexpr size_t kCacheEntryBytes = 66048;

// TMA descriptors of the q, k, v, out, gate (bf16) and log_alpha (fp32)
// tensors, viewed as [T, H, 128]; passed as a grid constant.
struct TcMaps {
    CUtensorMap q, k, v, la, out, gate;
    CUtensorMap beta;  // [T][H] fp32, box (4 heads, 64 tokens); only when H % 4 == 0
    int beta_tma;      // the beta map is set
};

struct TcPlan {
    int seg_chunks;        // chunks per segment
    int max_units;         // upper bound on the number of segments over all sequences
    bool segmented;        // some sequence may have more than one segment
    int64_t total_chunks;  // upper bound on the chunks of all sequences (ceil(T/64) + N packed)
};

// bf16 q/k/v with d_k = d_v = 128: tcgen05 tensor-core path.  from_span: the
// segment table and the transitions of this plan are already in a's workspace
// (left by launch_transition), so only the scan and pass 3 run.
cudaError_t launch_tc(const TcArgs& a, const TcPlan& p, cudaStream_t stream, int* launches,
                      bool from_span = false);
// Every chunk's operand images (kChunkImageBytes each) into a.dump: the segment
// table, then the forward pass's chunk-local work with a chain that only copies.
cudaError_t launch_dump(const TcArgs& a, const TcPlan& p, cudaStream_t stream, int* launches);

// Chain of affine state maps S -> M S + B, in the transposed layout of the
// library's transitions (entry [2][128][128]: B^T, then M^T; S^T_out = S^T_in M^T
// + B^T), evaluated on fp32 CUDA cores.
//   compose = 1: for each sequence b, compose its units off[b] .. off[b+1]-1 of
//                `trans` ([units][H][2][128][128]) into one transition, written to
//                out[b][h] in the same layout.
//   compose = 0: apply the first `count` transitions of `trans`
//                ([count][B][H][2][128][128]) to s0 ([B][H][128][128], or zero),
//                writing the resulting state to out ([B][H][128][128], natural
//                d_k x d_v layout).
struct ChainArgs {
    const float* trans;
    const int32_t* off;      // compose: [B+1] first unit of each sequence
    const int32_t* n_units;  // compose: number of valid units
    int32_t count;           // apply: transitions to apply
    int32_t B, H;
    const float* s0;         // apply: initial state or nullptr
    float* out;
    int32_t compose;
};
cudaError_t launch_chain(const ChainArgs& c, cudaStream_t stream, int* launches);

// Transition of every sequence (S_out = M S_in + B over all its tokens): the
// segment table, pass 1 over all segments, then their composition into out
// ([N][H][2][128][128]: B^T, M^T).  Uses a.trans as the per-segment workspace.
cudaError_t launch_transition(const TcArgs& a, const TcPlan& p, float* out, cudaStream_t stream,
                              int* launches);
size_t tc_smem_bytes();
// The bounded-wait self-test kernel (kda_selftest_wait).
cudaError_t launch_wait_probe(uint64_t timeout_ns, int arrive, cudaStream_t stream);
// Reads and clears the current device's status word (0 = no device-side error).
cudaError_t tc_take_status(int* code);

// Decode / multi-token verify step on a resident state (validated on the host).
struct DecodeArgs {
    const void* q;             // [N, T, H, dk]
    const void* k;             // [N, T, H, dk]
    const void* v;             // [N, T, H, dv]
    const float* log_alpha;    // [N, T, H, dk]
    const float* beta;         // [N, T, H]
    float* state;              // [num_slots, H, dk, dv], read and written in place
    const int32_t* slots;      // [N] state row of each sequence (-1 = skip), or nullptr
    void* out;                 // [N, T, H, dv]
    const void* gate;          // [N, T, H, dv] output gate (dtype of out), or nullptr
    float* token_states;       // [N, T, H, dk, dv] or nullptr
    int* status;               // device status word
    int32_t N, T, H, dk, dv, num_slots;
    int32_t bf16;
};
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream, int* launches);

}  // namespace kda
