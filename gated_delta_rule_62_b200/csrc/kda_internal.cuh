// Internal declarations shared by the libkda translation units (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "host_plan.h"
#include "kda.h"

// ---- optional NVTX ranges (build with -DKDA_NVTX): one named range per library call, so a
// profiler's timeline shows which entry point enqueued which kernels. Off by default: no cost.
#ifdef KDA_NVTX
#include <nvtx3/nvToolsExt.h>
namespace kda {
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
}  // namespace kda
#define KDA_RANGE(name) ::kda::NvtxRange kda_nvtx_range_(name)
#else
#define KDA_RANGE(name) ((void)0)
#endif

namespace kda {

// Sets a kernel's dynamic shared-memory limit on the current device, once per device (the
// attribute belongs to that device's context, so each GPU a process uses needs its own call).
inline cudaError_t set_smem_limit_once(PerDeviceOnce<> &once, const void *func, int bytes) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int r = once.run(dev, [&] {
        return (int)cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    });
    return r == PerDeviceOnce<>::kBadDevice ? cudaErrorInvalidDevice : static_cast<cudaError_t>(r);
}

// ---- element access for the two input dtypes -------------------------------------------
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// ---- where a sequence's states live ------------------------------------------------------
// Entry n of initial_state / final_state ([N, H, d_k, d_v]); or, with slot tables, slot
// init_slot[n] / final_slot[n] of one pool ([slots, H, d_k, d_v]), -1 meaning none. A slot outside
// [-1, slots) counts as -1 and sets kStatusBadSlot in the device status word.
constexpr int32_t kStatusTimeout = 1, kStatusBadSlot = 2, kStatusBadAccept = 4, kStatusBounds = 8;

// ---- debug builds (-DKDA_DEBUG): every global access at a computed address is checked against
// the byte range of the buffer it belongs to. An access outside it is skipped, and the first one
// is recorded in the device status word: bit kStatusBounds, then word 1 = the access site, words
// 2-3 = the offending address. No trap, no assert: the kernel keeps running and the host reads
// the record (kda_read_device_status -> KDA_ERR_INTERNAL). Release builds compile the checks away.
struct BufRange {
    uintptr_t lo = 0, hi = 0;  // [lo, hi); empty: not checked
};
struct DebugRanges {
    BufRange out, init, fin, beta, ws;  // outputs, initial / final states, beta, workspace
};
__host__ __device__ inline BufRange buf_range(const void *p, uint64_t bytes) {
    BufRange r;
    r.lo = reinterpret_cast<uintptr_t>(p);
    r.hi = p ? r.lo + bytes : 0;
    return r;
}
#ifdef KDA_DEBUG
static __device__ __noinline__ bool debug_access_ok(int32_t *status, const BufRange &r, const void *p,
                                             uint32_t bytes, int site) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    if (r.hi == r.lo || (a >= r.lo && a + bytes <= r.hi)) return true;
    if (status && !(atomicOr(status, kStatusBounds) & kStatusBounds)) {
        status[1] = site;
        reinterpret_cast<unsigned long long *>(status)[1] = (unsigned long long)a;
    }
    return false;
}
#define KDA_ACCESS_OK(status, range, ptr, bytes, site) \
    ::kda::debug_access_ok((status), (range), (ptr), (bytes), (site))
#else
#define KDA_ACCESS_OK(status, range, ptr, bytes, site) true
#endif
struct StateSlots {
    const int32_t *init_slot = nullptr, *final_slot = nullptr;  // device tables (or null)
    int64_t slots = 0;
    int32_t *status = nullptr;  // device status word (may be null)
};
__device__ __forceinline__ int64_t state_slot(const int32_t *tab, int n, const StateSlots &ss) {
    if (!tab) return n;
    const int32_t s = tab[n];
    if (s < -1 || (int64_t)s >= ss.slots) {
        if (ss.status) atomicOr(ss.status, kStatusBadSlot);
        return -1;
    }
    return s;
}
// Head h's [d_k, d_v] block of sequence n's initial / final state, or null for none.
__device__ __forceinline__ const float *init_state_block(const float *base, int n, int H, int h,
                                                         size_t elems, const StateSlots &ss) {
    if (!base) return nullptr;
    const int64_t s = state_slot(ss.init_slot, n, ss);
    return s < 0 ? nullptr : base + ((size_t)s * H + h) * elems;
}
__device__ __forceinline__ float *final_state_block(float *base, int n, int H, int h, size_t elems,
                                                    const StateSlots &ss) {
    if (!base) return nullptr;
    const int64_t s = state_slot(ss.final_slot, n, ss);
    return s < 0 ? nullptr : base + ((size_t)s * H + h) * elems;
}

// ---- the KDA layer's elementwise prologue (kda_prefill_prologue) -------------------------
// Raw q, k rows are L2-normalised, raw gates g give log alpha = -scale softplus(g), raw logits b
// give beta = sigmoid(b), as the kernels load them.
struct Prologue {
    uint32_t flags = 0;
    float gate_scale = 1.f;
};
constexpr float kL2NormEps = 1e-6f;
// -scale softplus(g), softplus(g) = max(g, 0) + log(1 + e^-|g|) (no overflow for any g)
__device__ __forceinline__ float gate_from_raw(float g, float scale) {
    return -scale * (fmaxf(g, 0.f) + __logf(1.f + __expf(-fabsf(g))));
}
__device__ __forceinline__ float beta_from_raw(float b) { return 1.f / (1.f + __expf(-b)); }

// ---- context parallelism: long sequences split into segments run as separate chains ------
// Device tables and buffers in the workspace (see kda_context.cu). A segment is a "virtual
// sequence" v with token offsets vcu[v], vcu[v + 1]; vinfo[v] = {sequence n, segment index g,
// segments of n, first chunk of its E tiles}. Segments g >= 1 start from a zero state; their
// consumers also carry the segment's transition product and emit, per chunk, E = P R: the
// chunk's output is its zero-start output plus E times the segment's true start state, which
// the scan kernel finds after all chains are done and the fix-up kernel applies.
struct SegPlan {
    int32_t *vcu = nullptr;       // [N_v + 1]
    int4 *vinfo = nullptr;        // [N_v]
    int32_t *vfirst = nullptr;    // [N] first segment of each sequence
    float *seg_state = nullptr;   // [N_v, H, d_k, d_v] fp32 end state of each segment's chain
    float *seg_trans = nullptr;   // [N_v, H, d_k, d_k] fp32 transition product of segments g >= 1
    uint8_t *s_start = nullptr;   // [N_v, H] 32 KB bf16 tiles: true start state of segments g >= 1
    uint8_t *e_tiles = nullptr;   // [E chunks, H] 16 KB bf16 tiles
    int32_t *e_live = nullptr;    // [N_v, H] chunks of a later segment whose E tile is live
    int32_t segments = 1, num_vseqs = 0, e_chunks = 0, max_chunks = 0;
};
constexpr uint32_t kSegStartTileBytes = 32768, kSegETileBytes = 16384;
// A later segment's transition product R (max |entry|) below this has decayed past any effect on
// the outputs: under the value contract (beta in [0, 1], unit keys) every chunk's transition is a
// contraction, so R only shrinks further, and the rest of the segment's E = P R and its share of
// the start state are below 128^2 * 2^-40 of the inputs' scale. Its chain and E tiles stop there.
constexpr float kSegDeadR = 9.094947e-13f;  // 2^-40

// ---- problem description passed from the API layer to the launchers --------------------
struct Problem {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    const float *initial_state;  // or the state pool (with slots)
    const int32_t *cu_seqlens;  // device
    int32_t num_seqs;
    int64_t total_tokens;
    int32_t H, dk, dv;
    kda_dtype_t dtype;
    void *out;
    float *final_state;          // or the state pool (with slots)
    StateSlots slots;
    Prologue pro;
    const SegPlan *seg = nullptr;  // context parallelism (split kernel only), or none
    DebugRanges dbg;               // buffer ranges for the debug build's access checks
};

// Each launcher enqueues its kernel(s) on `stream` and returns the launch's cudaError_t.
cudaError_t launch_prefill_recurrent(const Problem &p, cudaStream_t stream);

// Tensor-core chunk kernel: bf16 inputs with d_k = d_v = 128 and at least one token.
bool chunk_supported(const Problem &p);
size_t chunk_workspace_bytes(int32_t num_seqs);
// workspace: [0, 256) status word, then the longest-first sequence order (int32 each).
cudaError_t launch_prefill_chunk(const Problem &p, void *workspace, cudaStream_t stream,
                                 uint64_t timeout_ns);
cudaError_t launch_bounded_wait_probe(void *workspace, uint64_t timeout_ns, cudaStream_t stream);
cudaError_t launch_flag_wait_probe(void *workspace, uint64_t timeout_ns, cudaStream_t stream);

// Split-role chunk kernel (consumers run the state chain, producers the key-side half) for
// workloads with few (sequence, head) pairs; it needs a larger workspace (a ring of chunk images).
bool split_eligible(int64_t heads, kda_dtype_t dtype, int32_t dk, int32_t dv);
bool split_eligible_seqs(int32_t num_seqs);
size_t split_workspace_bytes(int64_t heads);
// Enqueues the split-role kernel; if its blocks cannot all be resident on this device, enqueues
// nothing, sets *not_coresident and returns cudaSuccess.
cudaError_t launch_prefill_split(const Problem &p, int32_t max_chunks, void *workspace,
                                 cudaStream_t stream, uint64_t timeout_ns, bool *not_coresident);

// Context parallelism (kda_context.cu): workspace bytes beyond the split kernel's for a plan, and
// the launches around the split kernel: the plan kernel before it, then the segment scan (true
// start and final states) and the output fix-up after it.
size_t seg_workspace_bytes(int32_t num_seqs, int32_t num_vseqs, int64_t e_chunks, int32_t H);
void seg_carve(SegPlan &sp, void *base, int32_t num_seqs, int32_t num_vseqs, int64_t e_chunks,
               int32_t H);
cudaError_t launch_seg_plan(const Problem &p, const SegPlan &sp, cudaStream_t stream);
cudaError_t launch_seg_scan_fixup(const Problem &p, const SegPlan &sp, int32_t *status,
                                  cudaStream_t stream, int32_t *launches);

// Records `msg` as the calling thread's kda_last_error() and returns `st`.
kda_status_t record_error(kda_status_t st, const char *msg);

// Upper bound on any single on-device wait before a kernel gives up (ns).
constexpr uint64_t kWaitTimeoutNs = 4000000000ull;

struct DecodeProblem {
    const void *q, *k, *v;
    const float *log_alpha, *beta;
    float *state;  // or the state pool (slots.init_slot == slots.final_slot: the slot table)
    int32_t num_seqs, H, dk, dv;
    kda_dtype_t dtype;
    void *out;
    StateSlots slots;
    DebugRanges dbg;
};
cudaError_t launch_decode(const DecodeProblem &p, cudaStream_t stream);

// Speculative decode: T draft tokens per sequence (rows n*T + t). With q set, the draft is
// verified (out and u_cache written); with accepted set, state n is first advanced by accepted[n]
// tokens of the previous draft (prev_k, prev_log_alpha, prev_u; rows n*T_prev + t) and stored.
struct VerifyProblem {
    const void *q, *k, *v;      // the draft to verify (q == null: commit only)
    const float *log_alpha, *beta;
    const void *prev_k;         // the accepted tokens to commit (accepted == null: none)
    const float *prev_log_alpha, *prev_u;
    const int32_t *accepted;    // device, [num_seqs]
    float *state;               // [num_seqs, ...] or, with slots, the pool
    int32_t num_seqs, T, T_prev, H, dk, dv;
    kda_dtype_t dtype;
    void *out;
    float *u_cache;
    StateSlots slots;
};
cudaError_t launch_verify(const VerifyProblem &p, cudaStream_t stream);

}  // namespace kda
