// kda_prefill_noalloc: the chunked prefill for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run a prefill: code
// inside a custom allocator or memory-pool callback, a serving loop whose device
// memory is carved up once at start-up and must not grow, or a host that forbids
// allocation on its hot path. kda_prefill needs a small caller-provided workspace
// (a status word and the longest-first sequence order); this entry point keeps
// that scratch in a fixed array in the library's own device memory instead.
//
// The scratch array below is loaded with the library: every GPU that loads
// libkda holds it (kNoallocScratchBytes) until the process exits. In host code
// its name is only a host-side stand-in for the symbol, not a device address, so
// the address is looked up with cudaGetSymbolAddress once per device (with that
// device current) and passed to the kernels as a plain pointer. That address is
// kept for the life of the process; a cudaDeviceReset unloads the library's
// device code and may move the array, so after a reset of a device this entry
// point must not be used on it again in the same process.
#include <cstdio>
#include <mutex>

#include "kda_internal.cuh"

namespace {

constexpr size_t kNoallocScratchBytes = 64 * 1024;
constexpr size_t kStatusBytes = 256;
// Sequences whose schedule fits behind the status word.
constexpr int32_t kNoallocMaxSeqs = (int32_t)((kNoallocScratchBytes - kStatusBytes) / sizeof(int32_t));

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, set up on first use.
cudaError_t scratch_on_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" KDA_API kda_status_t kda_prefill_noalloc(
    const void *q, const void *k, const void *v, const float *log_alpha, const float *beta,
    const float *initial_state, const int32_t *cu_seqlens_dev, const int32_t *cu_seqlens_host,
    int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k, int32_t d_v,
    kda_dtype_t dtype, void *out, float *final_state, kda_stream_t stream) {
    KDA_RANGE("kda_prefill_noalloc");
    if (num_seqs > kNoallocMaxSeqs) {
        char msg[160];
        snprintf(msg, sizeof msg, "kda_prefill_noalloc: num_seqs=%d exceeds the fixed scratch limit of %d",
                 num_seqs, kNoallocMaxSeqs);
        return kda::record_error(KDA_ERR_INVALID_ARGUMENT, msg);
    }
    void *scratch = nullptr;
    cudaError_t e = scratch_on_current_device(&scratch);
    if (e != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof msg, "kda_prefill_noalloc: scratch set-up (cudaGetSymbolAddress) failed: %s",
                 cudaGetErrorString(e));
        return kda::record_error(KDA_ERR_CUDA, msg);
    }
    // Same checks, planning and kernels as kda_prefill, with the fixed scratch as its workspace.
    // The planning kernel rewrites the status word and the whole schedule on every call.
    return kda_prefill(q, k, v, log_alpha, beta, initial_state, cu_seqlens_dev, cu_seqlens_host,
                       num_seqs, total_tokens, H, d_k, d_v, dtype, out, final_state, scratch,
                       kNoallocScratchBytes, stream);
}

// The status word of the last kda_prefill_noalloc on the current device sits at the start of the
// scratch array; read it the way kda_read_device_status reads a caller's workspace.
extern "C" KDA_API kda_status_t kda_prefill_noalloc_status(kda_stream_t stream) {
    void *scratch = nullptr;
    cudaError_t e = scratch_on_current_device(&scratch);
    if (e != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof msg, "kda_prefill_noalloc_status: scratch set-up (cudaGetSymbolAddress) failed: %s",
                 cudaGetErrorString(e));
        return kda::record_error(KDA_ERR_CUDA, msg);
    }
    return kda_read_device_status(scratch, stream);
}
