// libkda C ABI: host-side validation, planning and dispatch to the kernels.
// Every argument error is caught here, before anything is enqueued.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <string>

#include "kda_internal.cuh"

namespace {

thread_local std::string g_last_error;
thread_local int32_t g_last_launches = 0;  // kernels enqueued by the thread's last successful call

kda_status_t fail(kda_status_t st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
kda_status_t fail(kda_status_t st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

kda_status_t ok() {
    g_last_error.clear();
    return KDA_OK;
}

// Success after enqueuing `n` of this library's kernels (memsets and copies are not counted).
kda_status_t launched(int32_t n) {
    g_last_launches = n;
    return ok();
}

kda_status_t cuda_fail(cudaError_t e, const char *where) {
    return fail(KDA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool supported_d(int32_t d) { return d == 32 || d == 64 || d == 128; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kStatusBytes = 256;
constexpr int32_t kMaxSegments = 64;

// Checks shared by the prefill entry points. On success returns KDA_OK.
kda_status_t check_prefill(const void *q, const void *k, const void *v, const float *log_alpha,
                           const float *beta, const float *initial_state,
                           const int32_t *cu_dev, const int32_t *cu_host, int32_t num_seqs,
                           int64_t total_tokens, int32_t H, int32_t d_k, int32_t d_v,
                           kda_dtype_t dtype, const void *out, const float *final_state) {
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARGUMENT, "dtype %d is not KDA_F32 or KDA_BF16", (int)dtype);
    if (H <= 0 || H > 65535) return fail(KDA_ERR_INVALID_ARGUMENT, "H=%d outside [1, 65535]", H);
    if (!supported_d(d_k) || !supported_d(d_v))
        return fail(KDA_ERR_INVALID_ARGUMENT, "d_k=%d, d_v=%d: each must be 32, 64 or 128", d_k, d_v);
    if (num_seqs < 0) return fail(KDA_ERR_INVALID_ARGUMENT, "num_seqs=%d < 0", num_seqs);
    if (total_tokens < 0 || total_tokens > INT32_MAX)
        return fail(KDA_ERR_INVALID_ARGUMENT, "total_tokens=%lld outside [0, 2^31)",
                    (long long)total_tokens);
    if (num_seqs == 0) {
        if (total_tokens != 0)
            return fail(KDA_ERR_INVALID_ARGUMENT, "num_seqs=0 but total_tokens=%lld",
                        (long long)total_tokens);
        return ok();
    }
    if (!cu_dev || !cu_host)
        return fail(KDA_ERR_INVALID_ARGUMENT, "cu_seqlens_dev and cu_seqlens_host are required");
    if (cu_host[0] != 0) return fail(KDA_ERR_INVALID_ARGUMENT, "cu_seqlens[0]=%d != 0", cu_host[0]);
    for (int32_t n = 0; n < num_seqs; ++n)
        if (cu_host[n + 1] < cu_host[n])
            return fail(KDA_ERR_INVALID_ARGUMENT, "cu_seqlens decreases at %d (%d -> %d)", n,
                        cu_host[n], cu_host[n + 1]);
    if ((int64_t)cu_host[num_seqs] != total_tokens)
        return fail(KDA_ERR_INVALID_ARGUMENT, "cu_seqlens[%d]=%d != total_tokens=%lld", num_seqs,
                    cu_host[num_seqs], (long long)total_tokens);
    if (total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta || !out))
        return fail(KDA_ERR_INVALID_ARGUMENT, "q, k, v, log_alpha, beta and out are required");
    const void *ptrs[] = {q, k, v, log_alpha, out, initial_state, final_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return fail(KDA_ERR_INVALID_ARGUMENT, "tensor pointer %p is not 16-byte aligned", p);
    if (out && (out == q || out == k || out == v))
        return fail(KDA_ERR_INVALID_ARGUMENT, "out must not alias q, k or v");
    return ok();
}

kda::Problem make_problem(const void *q, const void *k, const void *v, const float *log_alpha,
                          const float *beta, const float *initial_state, const int32_t *cu_dev,
                          int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                          int32_t d_v, kda_dtype_t dtype, void *out, float *final_state) {
    kda::Problem p;
    p.q = q; p.k = k; p.v = v;
    p.log_alpha = log_alpha; p.beta = beta;
    p.initial_state = initial_state;
    p.cu_seqlens = cu_dev;
    p.num_seqs = num_seqs; p.total_tokens = total_tokens;
    p.H = H; p.dk = d_k; p.dv = d_v; p.dtype = dtype;
    p.out = out; p.final_state = final_state;
    return p;
}

// Byte ranges of the problem's buffers, for the debug build's access checks (no effect otherwise).
void set_ranges(kda::Problem &p, const void *workspace, size_t workspace_bytes, int64_t state_entries) {
    const uint64_t esz = p.dtype == KDA_BF16 ? 2 : 4;
    const uint64_t sbytes = (uint64_t)state_entries * p.H * p.dk * p.dv * 4;
    p.dbg.out = kda::buf_range(p.out, (uint64_t)p.total_tokens * p.H * p.dv * esz);
    p.dbg.init = kda::buf_range(p.initial_state, sbytes);
    p.dbg.fin = kda::buf_range(p.final_state, sbytes);
    p.dbg.beta = kda::buf_range(p.beta, (uint64_t)p.total_tokens * p.H * 4);
    p.dbg.ws = kda::buf_range(workspace, workspace_bytes);
#ifdef KDA_DEBUG
    // Debug builds only: declare the output smaller than it is, so a test can see the checks
    // skip and report the writes past that point (the buffer itself is large enough for them).
    if (const char *e = getenv("KDA_DEBUG_SHRINK_OUT")) {
        const uint64_t b = strtoull(e, nullptr, 10);
        if (p.dbg.out.hi > p.dbg.out.lo + b) p.dbg.out.hi = p.dbg.out.lo + b;
    }
#endif
}

// Workspace check and kernel choice shared by kda_prefill and kda_prefill_slots.
kda_status_t run_prefill(kda::Problem &p, const int32_t *cu_seqlens_host, void *workspace,
                         size_t workspace_bytes, cudaStream_t s, const char *who) {
    // Any workspace of the minimum size is accepted; a larger one (as sized by
    // kda_prefill_workspace_size) lets few-head problems use the split-role kernel.
    const size_t need = kda::chunk_workspace_bytes(p.num_seqs);
    if (!workspace || workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARGUMENT, "workspace %p of %zu bytes < required %zu",
                    workspace, workspace_bytes, need);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(KDA_ERR_INVALID_ARGUMENT, "workspace is not 256-byte aligned");
    set_ranges(p, workspace, workspace_bytes, p.slots.init_slot ? p.slots.slots : p.num_seqs);
    cudaError_t e;
    int32_t max_chunks = 0;
    for (int32_t n = 0; n < p.num_seqs; ++n) {
        const int32_t c = (cu_seqlens_host[n + 1] - cu_seqlens_host[n] + 63) / 64;
        max_chunks = c > max_chunks ? c : max_chunks;
    }
    const int64_t heads = (int64_t)p.num_seqs * p.H;
    if (kda::chunk_supported(p) && max_chunks >= 2 && kda::split_eligible(heads, p.dtype, p.dk, p.dv) &&
        kda::split_eligible_seqs(p.num_seqs) &&
        workspace_bytes >= kda::split_workspace_bytes(heads)) {
        // few heads: consumer CTAs run the state chains, producer CTAs fill the other SMs
        bool not_coresident = false;
        e = kda::launch_prefill_split(p, max_chunks, workspace, s, kda::kWaitTimeoutNs, &not_coresident);
        if (e == cudaSuccess && not_coresident)  // nothing enqueued: the single-role kernel runs
            e = kda::launch_prefill_chunk(p, workspace, s, kda::kWaitTimeoutNs);
    } else if (kda::chunk_supported(p)) {
        // the planning kernel clears the status word
        e = kda::launch_prefill_chunk(p, workspace, s, kda::kWaitTimeoutNs);
    } else {
        e = cudaMemsetAsync(workspace, 0, kStatusBytes, s);
        p.slots.status = static_cast<int32_t *>(workspace);
        if (e == cudaSuccess) e = kda::launch_prefill_recurrent(p, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, who);
    return launched(kda::chunk_supported(p) ? 2 : 1);  // init/plan + chunk kernel, or token-serial
}

}  // namespace

namespace kda {
kda_status_t record_error(kda_status_t st, const char *msg) { return fail(st, "%s", msg); }
}  // namespace kda

extern "C" {

size_t kda_prefill_workspace_size(int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                                  int32_t d_v, kda_dtype_t dtype) {
    if (num_seqs < 0 || total_tokens < 0 || H <= 0 || !supported_d(d_k) || !supported_d(d_v) ||
        (dtype != KDA_F32 && dtype != KDA_BF16))
        return 0;
    // [0, 256): device status word; then the per-sequence schedule (int32 each). Few-head
    // problems also get room for the split-role kernel's ring of chunk images.
    const size_t fused = kda::chunk_workspace_bytes(num_seqs);
    const int64_t heads = (int64_t)num_seqs * H;
    if (kda::split_eligible(heads, dtype, d_k, d_v)) {
        const size_t split = kda::split_workspace_bytes(heads);
        return split > fused ? split : fused;
    }
    return fused;
}

kda_status_t kda_prefill(const void *q, const void *k, const void *v, const float *log_alpha,
                         const float *beta, const float *initial_state,
                         const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                         int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                         int32_t d_v, kda_dtype_t dtype, void *out, float *final_state,
                         void *workspace, size_t workspace_bytes, kda_stream_t stream) {
    KDA_RANGE("kda_prefill");
    kda_status_t st = check_prefill(q, k, v, log_alpha, beta, initial_state, cu_seqlens_dev,
                                    cu_seqlens_host, num_seqs, total_tokens, H, d_k, d_v, dtype,
                                    out, final_state);
    if (st != KDA_OK || num_seqs == 0) return st;
    kda::Problem p = make_problem(q, k, v, log_alpha, beta, initial_state, cu_seqlens_dev,
                                  num_seqs, total_tokens, H, d_k, d_v, dtype, out, final_state);
    return run_prefill(p, cu_seqlens_host, workspace, workspace_bytes,
                       reinterpret_cast<cudaStream_t>(stream), "kda_prefill: launch");
}

size_t kda_prefill_cp_workspace_size(int32_t num_seqs, const int32_t *cu_seqlens_host, int32_t H,
                                     int32_t d_k, int32_t d_v, kda_dtype_t dtype, int32_t segments) {
    if (num_seqs < 0 || H <= 0 || !supported_d(d_k) || !supported_d(d_v) ||
        (dtype != KDA_F32 && dtype != KDA_BF16) || segments < 1 || segments > kMaxSegments ||
        (num_seqs > 0 && !cu_seqlens_host))
        return 0;
    const int64_t total = num_seqs > 0 ? (int64_t)cu_seqlens_host[num_seqs] : 0;
    const size_t plain = kda_prefill_workspace_size(num_seqs, total, H, d_k, d_v, dtype);
    if (num_seqs == 0 || dtype != KDA_BF16 || d_k != 128 || d_v != 128 || segments == 1) return plain;
    const kda::SegTotals t = kda::seg_totals(cu_seqlens_host, num_seqs, segments);
    const size_t cp = kda::split_workspace_bytes((int64_t)t.num_vseqs * H) +
                      kda::seg_workspace_bytes(num_seqs, t.num_vseqs, t.e_chunks, H);
    return cp > plain ? cp : plain;
}

kda_status_t kda_prefill_cp(const void *q, const void *k, const void *v, const float *log_alpha,
                            const float *beta, const float *initial_state,
                            const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                            int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                            int32_t d_v, kda_dtype_t dtype, void *out, float *final_state,
                            int32_t segments, void *workspace, size_t workspace_bytes,
                            kda_stream_t stream) {
    KDA_RANGE("kda_prefill_cp");
    if (segments < 1 || segments > kMaxSegments)
        return fail(KDA_ERR_INVALID_ARGUMENT, "segments=%d outside [1, %d]", segments, kMaxSegments);
    kda_status_t st = check_prefill(q, k, v, log_alpha, beta, initial_state, cu_seqlens_dev,
                                    cu_seqlens_host, num_seqs, total_tokens, H, d_k, d_v, dtype,
                                    out, final_state);
    if (st != KDA_OK || num_seqs == 0) return st;
    kda::Problem p = make_problem(q, k, v, log_alpha, beta, initial_state, cu_seqlens_dev,
                                  num_seqs, total_tokens, H, d_k, d_v, dtype, out, final_state);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const kda::SegTotals t = kda::seg_totals(cu_seqlens_host, num_seqs, segments);
    if (!kda::chunk_supported(p) || t.num_vseqs == num_seqs)  // nothing to split: the plain prefill
        return run_prefill(p, cu_seqlens_host, workspace, workspace_bytes, s, "kda_prefill_cp: launch");
    const size_t split_bytes = kda::split_workspace_bytes((int64_t)t.num_vseqs * H);
    const size_t need = split_bytes + kda::seg_workspace_bytes(num_seqs, t.num_vseqs, t.e_chunks, H);
    if (!workspace || workspace_bytes < need)
        return fail(KDA_ERR_INVALID_ARGUMENT,
                    "workspace %p of %zu bytes < %zu required for %d segments (kda_prefill_cp_workspace_size)",
                    workspace, workspace_bytes, need, segments);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(KDA_ERR_INVALID_ARGUMENT, "workspace is not 256-byte aligned");
    set_ranges(p, workspace, workspace_bytes, num_seqs);
    kda::SegPlan sp;
    sp.segments = segments;
    sp.max_chunks = t.max_chunks;
    kda::seg_carve(sp, static_cast<uint8_t *>(workspace) + split_bytes, num_seqs, t.num_vseqs,
                   t.e_chunks, H);
    p.seg = &sp;
    cudaError_t e = kda::launch_seg_plan(p, sp, s);
    if (e != cudaSuccess) return cuda_fail(e, "kda_prefill_cp: plan");
    bool not_coresident = false;
    e = kda::launch_prefill_split(p, t.max_chunks, workspace, s, kda::kWaitTimeoutNs, &not_coresident);
    if (e != cudaSuccess) return cuda_fail(e, "kda_prefill_cp: launch");
    if (not_coresident) {  // too many chains to be resident at once: the plain prefill
        p.seg = nullptr;
        return run_prefill(p, cu_seqlens_host, workspace, workspace_bytes, s, "kda_prefill_cp: launch");
    }
    int32_t n = 3;  // plan, split init, split kernel
    e = kda::launch_seg_scan_fixup(p, sp, static_cast<int32_t *>(workspace), s, &n);
    if (e != cudaSuccess) return cuda_fail(e, "kda_prefill_cp: scan / fix-up");
    return launched(n);
}

kda_status_t kda_prefill_prologue(const void *q, const void *k, const void *v,
                                  const float *log_alpha, const float *beta,
                                  const float *initial_state, const int32_t *cu_seqlens_dev,
                                  const int32_t *cu_seqlens_host, int32_t num_seqs,
                                  int64_t total_tokens, int32_t H, int32_t d_k, int32_t d_v,
                                  kda_dtype_t dtype, void *out, float *final_state, void *workspace,
                                  size_t workspace_bytes, uint32_t prologue_flags, float gate_scale,
                                  kda_stream_t stream) {
    KDA_RANGE("kda_prefill_prologue");
    constexpr uint32_t kAll =
        KDA_PROLOGUE_QK_L2NORM | KDA_PROLOGUE_GATE_SOFTPLUS | KDA_PROLOGUE_BETA_SIGMOID;
    if (prologue_flags & ~kAll)
        return fail(KDA_ERR_INVALID_ARGUMENT, "prologue_flags 0x%x has unknown bits", prologue_flags);
    if ((prologue_flags & KDA_PROLOGUE_GATE_SOFTPLUS) && !(gate_scale > 0.f && gate_scale < INFINITY))
        return fail(KDA_ERR_INVALID_ARGUMENT, "gate_scale=%g must be finite and > 0", (double)gate_scale);
    kda_status_t st = check_prefill(q, k, v, log_alpha, beta, initial_state, cu_seqlens_dev,
                                    cu_seqlens_host, num_seqs, total_tokens, H, d_k, d_v, dtype,
                                    out, final_state);
    if (st != KDA_OK || num_seqs == 0) return st;
    kda::Problem p = make_problem(q, k, v, log_alpha, beta, initial_state, cu_seqlens_dev,
                                  num_seqs, total_tokens, H, d_k, d_v, dtype, out, final_state);
    p.pro.flags = prologue_flags;
    p.pro.gate_scale = gate_scale;
    return run_prefill(p, cu_seqlens_host, workspace, workspace_bytes,
                       reinterpret_cast<cudaStream_t>(stream), "kda_prefill_prologue: launch");
}

kda_status_t kda_prefill_slots(const void *q, const void *k, const void *v, const float *log_alpha,
                               const float *beta, float *state_pool, int64_t pool_slots,
                               const int32_t *init_slot_dev, const int32_t *final_slot_dev,
                               const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
                               int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k,
                               int32_t d_v, kda_dtype_t dtype, void *out, void *workspace,
                               size_t workspace_bytes, kda_stream_t stream) {
    KDA_RANGE("kda_prefill_slots");
    if (pool_slots < 0 || pool_slots > INT32_MAX)
        return fail(KDA_ERR_INVALID_ARGUMENT, "pool_slots=%lld outside [0, 2^31)", (long long)pool_slots);
    if (pool_slots > 0 && !state_pool)
        return fail(KDA_ERR_INVALID_ARGUMENT, "state_pool is NULL with pool_slots=%lld",
                    (long long)pool_slots);
    kda_status_t st = check_prefill(q, k, v, log_alpha, beta, state_pool, cu_seqlens_dev,
                                    cu_seqlens_host, num_seqs, total_tokens, H, d_k, d_v, dtype,
                                    out, state_pool);
    if (st != KDA_OK || num_seqs == 0) return st;
    if (!init_slot_dev || !final_slot_dev)
        return fail(KDA_ERR_INVALID_ARGUMENT, "init_slot_dev and final_slot_dev are required");
    if (state_pool && out == (void *)state_pool)
        return fail(KDA_ERR_INVALID_ARGUMENT, "out must not alias the state pool");
    kda::Problem p = make_problem(q, k, v, log_alpha, beta, state_pool, cu_seqlens_dev, num_seqs,
                                  total_tokens, H, d_k, d_v, dtype, out, state_pool);
    p.slots.init_slot = init_slot_dev;
    p.slots.final_slot = final_slot_dev;
    p.slots.slots = pool_slots;
    return run_prefill(p, cu_seqlens_host, workspace, workspace_bytes,
                       reinterpret_cast<cudaStream_t>(stream), "kda_prefill_slots: launch");
}

kda_status_t kda_prefill_recurrent(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta,
                                   const float *initial_state, const int32_t *cu_seqlens_dev,
                                   const int32_t *cu_seqlens_host, int32_t num_seqs,
                                   int64_t total_tokens, int32_t H, int32_t d_k, int32_t d_v,
                                   kda_dtype_t dtype, void *out, float *final_state,
                                   kda_stream_t stream) {
    KDA_RANGE("kda_prefill_recurrent");
    kda_status_t st = check_prefill(q, k, v, log_alpha, beta, initial_state, cu_seqlens_dev,
                                    cu_seqlens_host, num_seqs, total_tokens, H, d_k, d_v, dtype,
                                    out, final_state);
    if (st != KDA_OK || num_seqs == 0) return st;
    kda::Problem p = make_problem(q, k, v, log_alpha, beta, initial_state, cu_seqlens_dev,
                                  num_seqs, total_tokens, H, d_k, d_v, dtype, out, final_state);
    set_ranges(p, nullptr, 0, num_seqs);
    cudaError_t e = kda::launch_prefill_recurrent(p, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kda_prefill_recurrent: launch");
    return launched(1);
}

kda_status_t kda_decode_step(const void *q, const void *k, const void *v, const float *log_alpha,
                             const float *beta, float *state, int32_t num_seqs, int32_t H,
                             int32_t d_k, int32_t d_v, kda_dtype_t dtype, void *out,
                             void *workspace, size_t workspace_bytes, kda_stream_t stream) {
    KDA_RANGE("kda_decode_step");
    (void)workspace;
    (void)workspace_bytes;
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARGUMENT, "dtype %d is not KDA_F32 or KDA_BF16", (int)dtype);
    if (H <= 0) return fail(KDA_ERR_INVALID_ARGUMENT, "H=%d <= 0", H);
    if (!supported_d(d_k) || !supported_d(d_v))
        return fail(KDA_ERR_INVALID_ARGUMENT, "d_k=%d, d_v=%d: each must be 32, 64 or 128", d_k, d_v);
    if (num_seqs < 0) return fail(KDA_ERR_INVALID_ARGUMENT, "num_seqs=%d < 0", num_seqs);
    if ((int64_t)num_seqs * H > INT32_MAX)
        return fail(KDA_ERR_INVALID_ARGUMENT, "num_seqs * H exceeds 2^31 - 1");
    if (num_seqs == 0) return ok();
    if (!q || !k || !v || !log_alpha || !beta || !state || !out)
        return fail(KDA_ERR_INVALID_ARGUMENT, "q, k, v, log_alpha, beta, state and out are required");
    const void *ptrs[] = {q, k, v, log_alpha, state, out};
    for (const void *p : ptrs)
        if (!aligned16(p))
            return fail(KDA_ERR_INVALID_ARGUMENT, "tensor pointer %p is not 16-byte aligned", p);
    if (out == q || out == k || out == v || out == (void *)state)
        return fail(KDA_ERR_INVALID_ARGUMENT, "out must not alias an input or the state");
    kda::DecodeProblem p;
    p.q = q; p.k = k; p.v = v; p.log_alpha = log_alpha; p.beta = beta; p.state = state;
    p.num_seqs = num_seqs; p.H = H; p.dk = d_k; p.dv = d_v; p.dtype = dtype; p.out = out;
    const uint64_t esz = dtype == KDA_BF16 ? 2 : 4;
    p.dbg.out = kda::buf_range(out, (uint64_t)num_seqs * H * d_v * esz);
    p.dbg.init = p.dbg.fin = kda::buf_range(state, (uint64_t)num_seqs * H * d_k * d_v * 4);
    cudaError_t e = kda::launch_decode(p, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kda_decode_step: launch");
    return launched(1);
}

kda_status_t kda_decode_step_slots(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const float *beta, float *state_pool,
                                   int64_t pool_slots, const int32_t *slot_dev, int32_t num_seqs,
                                   int32_t H, int32_t d_k, int32_t d_v, kda_dtype_t dtype,
                                   void *out, void *workspace, size_t workspace_bytes,
                                   kda_stream_t stream) {
    KDA_RANGE("kda_decode_step_slots");
    if (pool_slots < 0 || pool_slots > INT32_MAX)
        return fail(KDA_ERR_INVALID_ARGUMENT, "pool_slots=%lld outside [0, 2^31)", (long long)pool_slots);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARGUMENT, "dtype %d is not KDA_F32 or KDA_BF16", (int)dtype);
    if (H <= 0) return fail(KDA_ERR_INVALID_ARGUMENT, "H=%d <= 0", H);
    if (!supported_d(d_k) || !supported_d(d_v))
        return fail(KDA_ERR_INVALID_ARGUMENT, "d_k=%d, d_v=%d: each must be 32, 64 or 128", d_k, d_v);
    if (num_seqs < 0) return fail(KDA_ERR_INVALID_ARGUMENT, "num_seqs=%d < 0", num_seqs);
    if ((int64_t)num_seqs * H > INT32_MAX)
        return fail(KDA_ERR_INVALID_ARGUMENT, "num_seqs * H exceeds 2^31 - 1");
    if (num_seqs == 0) return ok();
    if (!q || !k || !v || !log_alpha || !beta || !out || !slot_dev)
        return fail(KDA_ERR_INVALID_ARGUMENT, "q, k, v, log_alpha, beta, slot_dev and out are required");
    if (pool_slots > 0 && !state_pool)
        return fail(KDA_ERR_INVALID_ARGUMENT, "state_pool is NULL with pool_slots=%lld",
                    (long long)pool_slots);
    if (!workspace || workspace_bytes < kStatusBytes ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(KDA_ERR_INVALID_ARGUMENT, "a 256-byte aligned workspace of >= %zu bytes is required",
                    kStatusBytes);
    const void *ptrs[] = {q, k, v, log_alpha, state_pool, out};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr))
            return fail(KDA_ERR_INVALID_ARGUMENT, "tensor pointer %p is not 16-byte aligned", ptr);
    if (out == q || out == k || out == v || (state_pool && out == (void *)state_pool))
        return fail(KDA_ERR_INVALID_ARGUMENT, "out must not alias an input or the state pool");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    kda::DecodeProblem p;
    p.q = q; p.k = k; p.v = v; p.log_alpha = log_alpha; p.beta = beta; p.state = state_pool;
    p.num_seqs = num_seqs; p.H = H; p.dk = d_k; p.dv = d_v; p.dtype = dtype; p.out = out;
    p.slots.init_slot = p.slots.final_slot = slot_dev;
    p.slots.slots = pool_slots;
    p.slots.status = static_cast<int32_t *>(workspace);
    const uint64_t esz = dtype == KDA_BF16 ? 2 : 4;
    p.dbg.out = kda::buf_range(out, (uint64_t)num_seqs * H * d_v * esz);
    p.dbg.init = p.dbg.fin = kda::buf_range(state_pool, (uint64_t)pool_slots * H * d_k * d_v * 4);
    cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, s);
    if (e == cudaSuccess) e = kda::launch_decode(p, s);
    if (e != cudaSuccess) return cuda_fail(e, "kda_decode_step_slots: launch");
    return launched(1);
}

}  // extern "C"

namespace {

// Checks shared by kda_decode_verify and kda_decode_commit (shapes, pool, workspace).
kda_status_t check_verify(const char *who, const float *state, int64_t pool_slots,
                          const int32_t *slot_dev, int32_t num_seqs, int32_t T, int32_t H,
                          int32_t d_k, int32_t d_v, kda_dtype_t dtype, const void *workspace,
                          size_t workspace_bytes) {
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: dtype %d is not KDA_F32 or KDA_BF16", who, (int)dtype);
    if (H <= 0) return fail(KDA_ERR_INVALID_ARGUMENT, "%s: H=%d <= 0", who, H);
    if (!supported_d(d_k) || !supported_d(d_v))
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: d_k=%d, d_v=%d: each must be 32, 64 or 128", who,
                    d_k, d_v);
    if (T < 1 || T > KDA_MAX_DRAFT_TOKENS)
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: T=%d outside [1, %d]", who, T, KDA_MAX_DRAFT_TOKENS);
    if (num_seqs < 0) return fail(KDA_ERR_INVALID_ARGUMENT, "%s: num_seqs=%d < 0", who, num_seqs);
    if ((int64_t)num_seqs * T * H > INT32_MAX)
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: num_seqs * T * H exceeds 2^31 - 1", who);
    if (slot_dev && (pool_slots < 0 || pool_slots > INT32_MAX))
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: pool_slots=%lld outside [0, 2^31)", who,
                    (long long)pool_slots);
    if (num_seqs > 0 && !state && !(slot_dev && pool_slots == 0))
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: state is NULL", who);
    if (!workspace || workspace_bytes < kStatusBytes ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(KDA_ERR_INVALID_ARGUMENT,
                    "%s: a 256-byte aligned workspace of >= %zu bytes is required", who, kStatusBytes);
    if (state && !aligned16(state))
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: state %p is not 16-byte aligned", who,
                    (const void *)state);
    return ok();
}

// Pointer checks of the draft to verify (kda_decode_verify, kda_decode_commit_verify).
kda_status_t check_draft(const char *who, const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta, const float *state,
                         const void *out, const float *u_cache) {
    if (!q || !k || !v || !log_alpha || !beta || !out || !u_cache)
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: q, k, v, log_alpha, beta, out and u_cache are "
                    "required", who);
    const void *ptrs[] = {q, k, v, log_alpha, out, u_cache};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr))
            return fail(KDA_ERR_INVALID_ARGUMENT, "%s: tensor pointer %p is not 16-byte aligned", who, ptr);
    const void *outs[] = {out, u_cache};
    for (const void *o : outs)
        if (o == q || o == k || o == v || o == (const void *)log_alpha || o == (const void *)state)
            return fail(KDA_ERR_INVALID_ARGUMENT, "%s: out and u_cache must not alias an input or "
                        "the state", who);
    if (out == (const void *)u_cache)
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: out aliases u_cache", who);
    return ok();
}

// Pointer checks of the accepted tokens to commit (kda_decode_commit, kda_decode_commit_verify).
kda_status_t check_accepted(const char *who, const void *k, const float *log_alpha,
                            const float *u_cache, const int32_t *accepted_dev, const float *state) {
    if (!k || !log_alpha || !u_cache || !accepted_dev)
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: k, log_alpha, u_cache and accepted_dev are "
                    "required", who);
    if (!aligned16(k) || !aligned16(log_alpha) || !aligned16(u_cache))
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: k, log_alpha and u_cache must be 16-byte aligned",
                    who);
    if (state && (k == (const void *)state || log_alpha == state || u_cache == state))
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: an input aliases the state", who);
    return ok();
}

kda_status_t launch_spec(const char *who, kda::VerifyProblem &p, int64_t pool_slots,
                         const int32_t *slot_dev, void *workspace, cudaStream_t s) {
    p.slots.init_slot = p.slots.final_slot = slot_dev;
    p.slots.slots = pool_slots;
    p.slots.status = static_cast<int32_t *>(workspace);
    cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, s);
    if (e == cudaSuccess) e = kda::launch_verify(p, s);
    if (e != cudaSuccess) return cuda_fail(e, who);
    return launched(1);
}

}  // namespace

extern "C" {

kda_status_t kda_decode_verify(const void *q, const void *k, const void *v, const float *log_alpha,
                               const float *beta, const float *state, int64_t pool_slots,
                               const int32_t *slot_dev, int32_t num_seqs, int32_t T, int32_t H,
                               int32_t d_k, int32_t d_v, kda_dtype_t dtype, void *out,
                               float *u_cache, void *workspace, size_t workspace_bytes,
                               kda_stream_t stream) {
    KDA_RANGE("kda_decode_verify");
    const char *who = "kda_decode_verify";
    kda_status_t st = check_verify(who, state, pool_slots, slot_dev, num_seqs, T, H, d_k, d_v, dtype,
                                   workspace, workspace_bytes);
    if (st != KDA_OK || num_seqs == 0) return st;
    st = check_draft(who, q, k, v, log_alpha, beta, state, out, u_cache);
    if (st != KDA_OK) return st;
    kda::VerifyProblem p{};
    p.q = q; p.k = k; p.v = v; p.log_alpha = log_alpha; p.beta = beta;
    p.state = const_cast<float *>(state);  // only read without a commit
    p.num_seqs = num_seqs; p.T = T; p.H = H; p.dk = d_k; p.dv = d_v; p.dtype = dtype;
    p.out = out; p.u_cache = u_cache;
    return launch_spec(who, p, pool_slots, slot_dev, workspace, reinterpret_cast<cudaStream_t>(stream));
}

kda_status_t kda_decode_commit(const void *k, const float *log_alpha, const float *u_cache,
                               float *state, int64_t pool_slots, const int32_t *slot_dev,
                               const int32_t *accepted_dev, int32_t num_seqs, int32_t T, int32_t H,
                               int32_t d_k, int32_t d_v, kda_dtype_t dtype, void *workspace,
                               size_t workspace_bytes, kda_stream_t stream) {
    KDA_RANGE("kda_decode_commit");
    const char *who = "kda_decode_commit";
    kda_status_t st = check_verify(who, state, pool_slots, slot_dev, num_seqs, T, H, d_k, d_v, dtype,
                                   workspace, workspace_bytes);
    if (st != KDA_OK || num_seqs == 0) return st;
    st = check_accepted(who, k, log_alpha, u_cache, accepted_dev, state);
    if (st != KDA_OK) return st;
    kda::VerifyProblem p{};
    p.prev_k = k; p.prev_log_alpha = log_alpha; p.prev_u = u_cache; p.accepted = accepted_dev;
    p.state = state;
    p.num_seqs = num_seqs; p.T_prev = T; p.H = H; p.dk = d_k; p.dv = d_v; p.dtype = dtype;
    return launch_spec(who, p, pool_slots, slot_dev, workspace, reinterpret_cast<cudaStream_t>(stream));
}

kda_status_t kda_decode_commit_verify(const void *prev_k, const float *prev_log_alpha,
                                      const float *prev_u, const int32_t *accepted_dev,
                                      int32_t T_prev, const void *q, const void *k, const void *v,
                                      const float *log_alpha, const float *beta, float *state,
                                      int64_t pool_slots, const int32_t *slot_dev, int32_t num_seqs,
                                      int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                      kda_dtype_t dtype, void *out, float *u_cache,
                                      void *workspace, size_t workspace_bytes,
                                      kda_stream_t stream) {
    KDA_RANGE("kda_decode_commit_verify");
    const char *who = "kda_decode_commit_verify";
    kda_status_t st = check_verify(who, state, pool_slots, slot_dev, num_seqs, T, H, d_k, d_v, dtype,
                                   workspace, workspace_bytes);
    if (st != KDA_OK) return st;
    if (T_prev < 1 || T_prev > KDA_MAX_DRAFT_TOKENS)
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: T_prev=%d outside [1, %d]", who, T_prev,
                    KDA_MAX_DRAFT_TOKENS);
    if ((int64_t)num_seqs * T_prev * H > INT32_MAX)
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: num_seqs * T_prev * H exceeds 2^31 - 1", who);
    if (num_seqs == 0) return ok();
    st = check_draft(who, q, k, v, log_alpha, beta, state, out, u_cache);
    if (st == KDA_OK) st = check_accepted(who, prev_k, prev_log_alpha, prev_u, accepted_dev, state);
    if (st != KDA_OK) return st;
    if (u_cache == prev_u || out == (const void *)prev_u || out == prev_k || u_cache == prev_k ||
        out == (const void *)prev_log_alpha || u_cache == prev_log_alpha)
        return fail(KDA_ERR_INVALID_ARGUMENT, "%s: out and u_cache must not alias the previous "
                    "draft's k, log_alpha or u", who);
    kda::VerifyProblem p{};
    p.q = q; p.k = k; p.v = v; p.log_alpha = log_alpha; p.beta = beta;
    p.prev_k = prev_k; p.prev_log_alpha = prev_log_alpha; p.prev_u = prev_u; p.accepted = accepted_dev;
    p.state = state;
    p.num_seqs = num_seqs; p.T = T; p.T_prev = T_prev; p.H = H; p.dk = d_k; p.dv = d_v;
    p.dtype = dtype; p.out = out; p.u_cache = u_cache;
    return launch_spec(who, p, pool_slots, slot_dev, workspace, reinterpret_cast<cudaStream_t>(stream));
}

const char *kda_status_string(kda_status_t s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARGUMENT: return "KDA_ERR_INVALID_ARGUMENT";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        case KDA_ERR_INTERNAL: return "KDA_ERR_INTERNAL";
    }
    return "KDA_ERR_UNKNOWN";
}

const char *kda_last_error(void) { return g_last_error.c_str(); }

kda_status_t kda_read_device_status(const void *workspace, kda_stream_t stream) {
    if (!workspace) return fail(KDA_ERR_INVALID_ARGUMENT, "workspace is NULL");
    int32_t rec[4] = {0, 0, 0, 0};  // status word; with kStatusBounds: site, address
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(rec, workspace, sizeof rec, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "kda_read_device_status");
    const int32_t word = rec[0];
    if (word == 0) return ok();
    if (word & kda::kStatusBounds) {
        unsigned long long addr = 0;
        memcpy(&addr, rec + 2, sizeof addr);
        return fail(KDA_ERR_INTERNAL, "device status word 0x%x: the debug build caught an access "
                    "outside its buffer at site %d (address 0x%llx)", (unsigned)word, rec[1], addr);
    }
    if (word & (kda::kStatusBadSlot | kda::kStatusBadAccept))
        return fail(KDA_ERR_INVALID_ARGUMENT, "device status word 0x%x: a state slot outside "
                    "[-1, pool_slots) or an accepted count outside [0, T]", (unsigned)word);
    return fail(KDA_ERR_TIMEOUT, "device status word 0x%x: a bounded on-device wait gave up",
                (unsigned)word);
}

kda_status_t kda_selftest_bounded_wait(void *workspace, size_t workspace_bytes,
                                       uint64_t timeout_ns, kda_stream_t stream) {
    if (!workspace || workspace_bytes < kStatusBytes)
        return fail(KDA_ERR_INVALID_ARGUMENT, "workspace of at least %zu bytes is required",
                    kStatusBytes);
    if (timeout_ns == 0 || timeout_ns > 10000000000ull)
        return fail(KDA_ERR_INVALID_ARGUMENT, "timeout_ns must be in (0, 1e10]");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, s);
    if (e == cudaSuccess) e = kda::launch_bounded_wait_probe(workspace, timeout_ns, s);
    if (e != cudaSuccess) return cuda_fail(e, "kda_selftest_bounded_wait: launch");
    return launched(1);
}

kda_status_t kda_selftest_flag_wait(void *workspace, size_t workspace_bytes, uint64_t timeout_ns,
                                    kda_stream_t stream) {
    if (!workspace || workspace_bytes < kStatusBytes)
        return fail(KDA_ERR_INVALID_ARGUMENT, "workspace of at least %zu bytes is required",
                    kStatusBytes);
    if (timeout_ns == 0 || timeout_ns > 10000000000ull)
        return fail(KDA_ERR_INVALID_ARGUMENT, "timeout_ns must be in (0, 1e10]");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, s);
    if (e == cudaSuccess) e = kda::launch_flag_wait_probe(workspace, timeout_ns, s);
    if (e != cudaSuccess) return cuda_fail(e, "kda_selftest_flag_wait: launch");
    return launched(1);
}

int32_t kda_version(void) { return 100; }

int32_t kda_last_launch_count(void) { return g_last_launches; }

}  // extern "C"
