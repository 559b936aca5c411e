// Host-side bookkeeping and planning in plain C++ (no CUDA types), so it is unit-tested on the CPU.
//
// PerDeviceOnce: once-per-device set-up.
// Some CUDA state belongs to one device's context, not to the process: a kernel's
// cudaFuncAttributeMaxDynamicSharedMemorySize, or the device address of a __device__ array. A
// process-wide "done" flag would skip that set-up on the second GPU a process uses. PerDeviceOnce
// keeps one flag per device id: run(dev, f) calls f() (with that device current, which is the
// caller's job) until it returns 0 once for that device, then never again for it; a non-zero
// result is returned and not remembered, so a later call retries.
#pragma once

#include <mutex>

#ifdef __CUDACC__
#define KDA_HD __host__ __device__
#else
#define KDA_HD
#endif

namespace kda {

template <int MaxDevices = 64>
class PerDeviceOnce {
  public:
    static constexpr int kBadDevice = -1;

    // Result of f() on the call that ran it, 0 once set-up for `dev` has succeeded, or kBadDevice
    // for a device id outside [0, MaxDevices).
    template <class F>
    int run(int dev, F &&f) {
        if (dev < 0 || dev >= MaxDevices) return kBadDevice;
        std::lock_guard<std::mutex> lk(mutex_);
        if (done_[dev]) return 0;
        const int r = static_cast<int>(f());
        if (r == 0) done_[dev] = true;
        return r;
    }

    bool done(int dev) {
        if (dev < 0 || dev >= MaxDevices) return false;
        std::lock_guard<std::mutex> lk(mutex_);
        return done_[dev];
    }

  private:
    std::mutex mutex_;
    bool done_[MaxDevices] = {};
};

// The split-role prefill is one cooperative launch of per_sm thread blocks on each of `sms` SMs, of
// which `heads` run the state chains; it needs every block resident at once and at least as many
// producer blocks as consumers. False means: run the single-role chunk kernel instead.
inline bool split_coresident(int per_sm, int sms, long long heads) {
    return per_sm >= 1 && sms >= 1 && heads >= 1 && (long long)per_sm * sms >= 2 * heads;
}

// Context parallelism: a sequence of `chunks` 64-token chunks runs as seg_count(chunks, segments)
// segments (at least one, so an empty sequence still has a chain that carries its state), segment
// g covering chunks [seg_chunk_begin(chunks, G, g), seg_chunk_begin(chunks, G, g + 1)). The host
// plans with these and the device plan kernel derives the same table from them.
KDA_HD inline int seg_count(int chunks, int segments) {
    const int g = chunks < segments ? chunks : segments;
    return g < 1 ? 1 : g;
}
KDA_HD inline int seg_chunk_begin(int chunks, int G, int g) {
    return (int)((long long)g * chunks / G);
}

// Totals of a segmentation of num_seqs sequences (token offsets cu[0..num_seqs]): the segments
// (chains), the chunks of all segments after their sequence's first (one E tile per chunk and
// head), and the most chunks in one segment.
struct SegTotals {
    int num_vseqs = 0;
    long long e_chunks = 0;
    int max_chunks = 0;
};
inline SegTotals seg_totals(const int *cu, int num_seqs, int segments) {
    SegTotals t;
    for (int n = 0; n < num_seqs; ++n) {
        const int chunks = (cu[n + 1] - cu[n] + 63) / 64;
        const int G = seg_count(chunks, segments);
        t.num_vseqs += G;
        for (int g = 0; g < G; ++g) {
            const int len = seg_chunk_begin(chunks, G, g + 1) - seg_chunk_begin(chunks, G, g);
            if (g >= 1) t.e_chunks += len;
            if (len > t.max_chunks) t.max_chunks = len;
        }
    }
    return t;
}

}  // namespace kda
