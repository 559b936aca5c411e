// Internal declarations shared by the libkda translation units (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "host_plan.h"
#include "kda.h"

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
constexpr int32_t kStatusTimeout = 1, kStatusBadSlot = 2, kStatusBadAccept = 4;
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
