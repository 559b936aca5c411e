// Split-role chunked prefill for workloads with few (sequence, head) pairs.
//
// The chunk algebra is that of kda_chunk.cu, regrouped so that the sequential state chain
// holds a single dependent MMA batch per chunk. With U = T'V - W S (T'V written U~):
//
//   S_next = diag(gamma) S + K^^T U = S + M S + K^^T U~,   M = diag(gamma - 1) - K^^T W,
//   O      = Q~ S + A U             = P S + A U~,          P = Q~ - A W.
//
// M, P and U~ depend only on the chunk's own q, k, v, gates and beta, so they are computed
// off the chain. One persistent cooperative launch fills the GPU:
//
//   producer CTAs (most SMs): for chunks ahead of the chain, chunk-major order: the gating,
//     A and L, T' = (I + L)^-1 diag(beta), W = T' K~, then U~ and -A W in one M=128 MMA
//     ([T'; 0] V + [0; A] (-W)) and -K^^T W in another, and from those U~, P and M as
//     ready-to-use shared-memory images (bf16) in a ring of RING slots per head in the
//     workspace (L2 resident). Each producer keeps two items in flight, so that one item's
//     MMAs run while the compute warps work on the other (see the producer).
//   consumer CTAs (one per head): the chain. Per chunk: S += M S_b + K^^T U~ (S_b = the
//     state's bf16 copy, fed from tensor memory), O = P S_b + A U~ behind it; the outputs leave
//     while the next chunk's chain runs. The fp32 state stays in TMEM for the whole sequence.
//
// Hand-off: a producer fills slot (head, c % RING) with bulk stores, then releases
// filled[slot] = c + 1; a consumer acquires it, copies the image into shared memory with a
// bulk copy, and releases its consumed counter = c + 1 once the copy has landed; the producer
// acquires the head's consumers' counters >= c - RING + 1 before reusing the slot. Producer
// items are ordered by chunk, and every producer works through its items in order, so the
// item a consumer waits for never waits on anything later: no cycle. Every spin and mbarrier
// wait is bounded; on timeout the status word is set and the CTA stops. The launch is
// cooperative, so all CTAs are resident together or the launch fails.
#include <cuda.h>

#include <mutex>

#include "kda_chunk_common.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace chunk;

// Ring depth, in chunks per head. 8 keeps the ring (22.5 MiB for 32 heads) resident in L2 next to
// the streaming inputs; with 16 it spilled (DRAM writes per 8192 x 32 launch: 58 -> 267 MB) for
// no gain in time.
constexpr int RING = 8;
// Chunk image (bytes), the same in a ring slot and in a consumer stage (bf16, 128-byte
// swizzled tiles):
//   [0, 32K)     M [c][c'] (K-major A operand, 128 rows, 64-column blocks of 16 KB)
//   [32K, 48K)   K^ [j][c] (MN-major A operand of K^^T U~, blocks of 8 KB)
//   [48K, 64K)   U~ [j][d] (MN-major B operand, blocks of 8 KB)
//   [64K, 80K)   P [i][c] (K-major A operand, 64 rows, blocks of 8 KB)
//   [80K, 88K)   A [i][j] (K-major A operand, 64 rows)
constexpr uint32_t SL_M = 0, SL_KH = 32768, SL_U = 49152, SL_P = 65536, SL_A = 81920;
constexpr uint32_t SLOT = 90112;
static_assert(SLOT % 1024 == 0, "slot layout");
// The ring moves with plain (1-D) bulk copies: a consumer loads a whole image in one copy, a
// producer stores it in six, one per contiguous piece of its shared memory. (One SM moves about
// 75 bytes per cycle from L2 into shared memory this way, and about 30 the other way; the 2-D
// tensor copies of 512-byte rows used before loaded at about a third of that.)

struct SplitParams {
    const int32_t *cu_seqlens;
    const float *beta;
    Prologue pro;
    const float *s0;  // initial states, or the state pool
    float *sT;        // final states, or the state pool
    __nv_bfloat16 *out;
    int32_t *status;
    StateSlots ss;
    uint8_t *ring;       // [heads][RING][SLOT]
    int32_t *filled;     // [heads][RING]
    int32_t *consumed;   // [heads]
    int32_t *next_item;  // producers' work counter (items k = chunk * heads + head, chunk-major)
    int32_t H, heads, max_chunks;
    uint64_t timeout_ns;
    // context parallelism (segments as separate chains), or all null
    const int4 *vinfo;   // [segments] {sequence, segment index, segments of the sequence, E offset}
    float *seg_state;    // [segments, H, D, D] each chain's end state (sequences of several segments)
    float *seg_trans;    // [segments, H, D, D] transition product of segments after the first
    uint8_t *e_tiles;    // [E chunks, H] E = P R tiles
    int32_t *e_live;     // [segments, H] chunks of a later segment whose E tile is live
    DebugRanges dbg;     // buffer ranges (checked by debug builds only)
};

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// shared -> global, tracked by the issuing thread's bulk async-group
__device__ __forceinline__ void bulk_store(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(smem_u32(src)),
                 "r"(bytes)
                 : "memory");
}
// Output element store with the streaming (evict-first) cache hint: outputs are not read again
// here, so they should not push the ring's images out of L2.
__device__ __forceinline__ void st_stream_bf16(__nv_bfloat16 *dst, float x) {
    __stcs(reinterpret_cast<unsigned short *>(dst), __bfloat16_as_ushort(__float2bfloat16_rn(x)));
}
// Waits until the committed TMA stores have finished reading shared memory / are complete.
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Every split CTA runs NTC compute threads (warps 0..15) plus two control warps: lane 0 of
// warp 16 issues the tensor-core MMAs (and, in a producer, the TMA loads); lane 0 of warp 17
// brings a consumer its chunk images, or takes a producer's finished images to the ring (slot
// wait, stores, hand-off flag). None of their waits stalls a compute warp. Sixteen compute warps
// (four per SM sub-partition) halve each phase's per-thread work against eight: the per-chunk work
// is latency-bound, not issue-bound.
constexpr int NTC = 2 * NT;    // compute threads: 16 warps
constexpr int NTS = NTC + 64;
constexpr int CTL = NTC;       // the MMA / control thread
constexpr int LDR = NTC + 32;  // the consumer's loader thread
constexpr int STR = NTC + 32;  // the producer's store thread
// Barrier of a producer's compute threads and its control warp (warps 0 .. 16), which leaves out
// the store thread's warp: its waits on the ring never hold up the others.
constexpr int NWORK = NTC + 32;
__device__ __forceinline__ void sync_work() { asm volatile("bar.sync 2, %0;" ::"n"(NWORK) : "memory"); }
__device__ __forceinline__ int sync_work_or(int pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 2, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "n"(NWORK)
        : "memory");
    return (int)r;
}

__device__ __forceinline__ uint32_t ld_volatile(const uint32_t *p) {
    return *reinterpret_cast<const volatile uint32_t *>(p);
}

// ---------------------------------------------------------------- consumer (state chain)
// One consumer per head. The state is kept transposed, S^T [d][c] (lane = value channel d), so its
// bf16 copy can feed the chain's MMA as an A operand straight from tensor memory:
//   S^T += S_b^T M^T + U~^T K^   (A = S_b^T in TMEM, B = M as stored; A = U~, B = K^ MN-major)
//   O    = P S_b + A U~          (M = 64 tokens; B = S_b^T [d][c], a K-major tile in shared memory)
// so the next chunk's chain waits neither for the output MMA nor for a shared-memory store.
namespace cons {
constexpr uint32_t STAGE0 = 0, STAGE1 = SLOT;
constexpr uint32_t MISC = 2 * SLOT;        // barriers, flags
constexpr uint32_t BYTES = MISC + 256;
// TMEM: S^T fp32 (128 columns), two bf16 copies S_b^T (64 columns each, used by alternate chunks),
// two output accumulators O^T (lane = value channel, column = token; 64 of 128 columns used).
constexpr uint32_t TM_S = 0, TM_SB0 = 128, TM_SB1 = 192, TM_O0 = 256, TM_O1 = 384, TM_COLS = 512;
}  // namespace cons

// Consumer roles, per chunk c (stage b = c & 1). Loader: once the producer has published chunk c
// and chunk c - 2's MMAs have completed (o[b]), copy its image into stage b (full[b]); publish
// consumption of chunk c - 2 at that point. MMA thread: wait for the image and for S_b^T(c) in TMEM,
// issue the chain (commit s); once the output warps have read accumulator b (chunk c - 2), issue
// the transposed output O^T = S_b^T P^T + U~^T A^T from the same TMEM copy (commit o[b]). State
// warps 0..7 (lane = value channel, two column halves): after s, the new state's bf16 copy into
// TMEM ("tmem ready": the critical path). Output warps 8..15 (32 tokens each): after o[b], the
// outputs ("o free"). No CTA-wide barrier inside
// the loop. S_b^T(c) in TMEM copy c & 1 is rewritten only after the chain of chunk c + 1 has
// completed, and so has O(c), issued before it by the same thread.
__device__ void consumer(const SplitParams &p, uint8_t *sm, int hd) {
    using namespace cons;
    constexpr uint32_t I_C = idesc_bf16_f32(128, 128, false, 0, 0);   // S_b^T M^T (A in TMEM)
    constexpr uint32_t I_K = idesc_bf16_f32(128, 128, false, 1, 1);   // U~^T K^
    constexpr uint32_t I_OP = idesc_bf16_f32(128, 64, false, 0, 0);   // S_b^T P^T (A in TMEM)
    constexpr uint32_t I_OA = idesc_bf16_f32(128, 64, false, 1, 0);   // U~^T A^T
    // full0, full1, s, (3: unused), o0, o1, tmem ready, (7: unused), o free 0, o free 1, teardown
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC);
    uint32_t *s_flags = reinterpret_cast<uint32_t *>(sm + MISC + 96); // abort, tmem
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const int H = p.H, v = hd / H, h = hd % H;
    const int64_t bos = p.cu_seqlens[v], eos = p.cu_seqlens[v + 1];
    const int nchunks = (int)((eos - bos + C - 1) / C);
    // v is a sequence, or with context parallelism the first segment of sequence vinfo[v].x: it
    // starts from the sequence's initial state; its end state goes to the scan if more segments follow
    const int4 vi = p.vinfo ? p.vinfo[v] : make_int4(v, 0, 1, 0);
    const float *s0b = init_state_block(p.s0, vi.x, H, h, (size_t)D * D, p.ss);
    float *sTb = vi.z > 1 ? p.seg_state + (size_t)hd * D * D
                          : final_state_block(p.sT, vi.x, H, h, (size_t)D * D, p.ss);
    if (s0b && !KDA_ACCESS_OK(p.status, p.dbg.init, s0b, D * D * 4, 1)) s0b = nullptr;
    if (sTb && !KDA_ACCESS_OK(p.status, vi.z > 1 ? p.dbg.ws : p.dbg.fin, sTb, D * D * 4, 2)) sTb = nullptr;

    if (tid == 0) {
        s_flags[0] = 0;
        for (int k = 0; k < 11; ++k) mbar_init(&bars[k], (k >= 6 && k <= 9) ? NTC / 2 : 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&s_flags[1], TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_flags[1];
    auto fail = [&]() {
        s_flags[0] = 1;
        atomicOr(p.status, 1);
    };

    if (tid == LDR) {
        // ------------------------------------------------ loader thread
        // Chunk c goes to stage c & 1 once the producer has published it (acquired ahead, so
        // the acquire's latency overlaps the wait) and chunk c - 2's MMAs have completed (o[b]);
        // that completion also means chunk c - 2's image had landed: its slot may be refilled.
        int requested = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (ld_volatile(&s_flags[0])) break;
            if (!wait_flag_ge(p.filled + hd * RING + (c % RING), c + 1, p.timeout_ns)) { fail(); break; }
            fence_proxy_async_global();
            if (c >= 2) {
                // chunk c - 2 is use (c - 2) / 2 of o[b]: phase parity ((c - 2) >> 1) & 1
                if (!mbar_wait_bounded(&bars[4 + b], (uint32_t)((c - 2) >> 1) & 1u, p.timeout_ns)) { fail(); break; }
                st_release(p.consumed + hd, c - 1);
            }
            const uint8_t *src = p.ring + ((size_t)hd * RING + (size_t)(c % RING)) * SLOT;
            mbar_arrive_expect_tx(&bars[b], SLOT);
            bulk_load(sm + (b ? STAGE1 : STAGE0), src, SLOT, &bars[b]);
            requested = c + 1;
        }
        // the last images land before the CTA exits (the MMA thread may have stopped early)
        for (int c = requested - 2 < 0 ? 0 : requested - 2; c < requested; ++c)
            if (!mbar_wait_bounded(&bars[c & 1], (uint32_t)(c >> 1) & 1u, p.timeout_ns)) fail();
        if (requested == nchunks) st_release(p.consumed + hd, nchunks);
    } else if (tid == CTL) {
        // ------------------------------------------------ MMA thread
        uint32_t ph_t = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (ld_volatile(&s_flags[0])) break;
            if (!mbar_wait_bounded(&bars[b], (uint32_t)(c >> 1) & 1u, p.timeout_ns)) { fail(); break; }
            if (!mbar_wait_bounded(&bars[6], ph_t, p.timeout_ns)) { fail(); break; }
            ph_t ^= 1u;
            tc_fence_after();
            const uint32_t st = sb + (b ? STAGE1 : STAGE0);
            const uint32_t tm_sb = tmem + (b ? TM_SB1 : TM_SB0);
            const uint32_t tm_o = tmem + (b ? TM_O1 : TM_O0);
            const uint64_t dM = desc_k(st + SL_M, 16384, 0), dK = desc_mn(st + SL_KH, 8192, 0);
            const uint64_t dU = desc_mn(st + SL_U, 8192, 0);
            const uint64_t dP = desc_k(st + SL_P, 8192, 0), dA = desc_k(st + SL_A, 8192, 0);
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk)  // S^T += S_b^T M^T ...
                mma_bf16_ts(tmem + TM_S, tm_sb + 8 * kk, desc_k_at(dM, 16384, kk), I_C, 1);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // ... + U~^T K^
                mma_bf16_ss(tmem + TM_S, desc_mn_at(dU, kk), desc_mn_at(dK, kk), I_K, 1);
            mma_commit(&bars[2]);
            if (c >= 2) {  // the output warps have read this accumulator's previous chunk
                if (!mbar_wait_bounded(&bars[8 + b], (uint32_t)((c - 2) >> 1) & 1u, p.timeout_ns)) { fail(); break; }
            }
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk)  // O^T = S_b^T P^T ...
                mma_bf16_ts(tm_o, tm_sb + 8 * kk, desc_k_at(dP, 8192, kk), I_OP, kk > 0);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // ... + U~^T A^T
                mma_bf16_ss(tm_o, desc_mn_at(dU, kk), desc_k_at(dA, 8192, kk), I_OA, 1);
            mma_commit(&bars[4 + b]);            // O and the stage are done
        }
        // teardown: every issued MMA completes before TMEM is freed
        mma_commit(&bars[10]);
        mbar_wait_bounded(&bars[10], 0, p.timeout_ns);
    } else if (warp < 8) {
        // ------------------------------------------------ state warps (lane = value channel d)
        // per chunk: the new state -> its bf16 copy in TMEM (the next chain's and the output's A
        // operand). Warps w and w + 4 share lanes 32 (w % 4) .. + 31: columns [64 hh, 64 hh + 64).
        const int d_me = 32 * quad + lane;
        const int hh = warp >> 2;
        auto wait_bar = [&](uint64_t *bar, uint32_t &ph) -> bool {
            const bool ok = mbar_wait_bounded(bar, ph, p.timeout_ns);
            ph ^= 1u;
            if (!ok) fail();
            return ok;
        };
        // 32 fp32 columns (state columns 64 hh + 32 part ..) -> 16 bf16 pairs of the copy at tm_sb
        auto pack_store = [&](const float (&v)[32], int part, uint32_t tm_sb) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = pack2(v[2 * e], v[2 * e + 1]);
            tmem_st16(tmem + lane_base + tm_sb + 32 * hh + 16 * part, w);
        };
        // initial state S[c][d] -> S^T in TMEM and its bf16 copy; empty sequences copy it out
        {
            const float *src = s0b ? s0b + (size_t)(64 * hh) * D + d_me : nullptr;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = src ? src[(size_t)(32 * part + e) * D] : 0.f;
                if (nchunks == 0) {
                    if (sTb) {
                        float *dst = sTb + (size_t)(64 * hh + 32 * part) * D + d_me;
#pragma unroll
                        for (int e = 0; e < 32; ++e) dst[(size_t)e * D] = v[e];
                    }
                } else {
                    tmem_st32(tmem + lane_base + TM_S + 64 * hh + 32 * part, v);
                    pack_store(v, part, TM_SB0);
                }
            }
        }
        if (nchunks > 0) {
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[6]);
        }
        uint32_t ph_s = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const bool last = c + 1 == nchunks;
            if (ld_volatile(&s_flags[0])) break;
            if (!wait_bar(&bars[2], ph_s)) break;
            tc_fence_after();
            float v[2][32];
            tmem_ld32(tmem + lane_base + TM_S + 64 * hh, v[0]);
            tmem_ld32(tmem + lane_base + TM_S + 64 * hh + 32, v[1]);
            tmem_wait_ld();
            if (!last) {
                pack_store(v[0], 0, b ? TM_SB0 : TM_SB1);  // the next chunk's copy
                pack_store(v[1], 1, b ? TM_SB0 : TM_SB1);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[6]);
            } else if (sTb) {
                float *dst = sTb + (size_t)(64 * hh) * D + d_me;
#pragma unroll
                for (int e = 0; e < 64; ++e) dst[(size_t)e * D] = v[e >> 5][e & 31];
            }
        }
        tc_fence_before();
    } else if (tid < NTC) {
        // ------------------------------------------------ output warps
        // O^T of chunk c (lane = value channel d, column = token) -> bf16 outputs; warps w and
        // w + 4 (w = 8..11) take tokens [32 th, 32 th + 32); for each token a warp stores 32
        // consecutive channels (64 bytes)
        const int d_me = 32 * quad + lane;
        const int th = (warp >> 2) & 1;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (ld_volatile(&s_flags[0])) break;
            const bool ok = mbar_wait_bounded(&bars[4 + b], (uint32_t)(c >> 1) & 1u, p.timeout_ns);
            if (!ok) { fail(); break; }
            tc_fence_after();
            const int64_t tc = bos + (int64_t)c * C + 32 * th;
            const int vc = (int)(eos - tc < 32 ? eos - tc : 32);
            const uint32_t tm_o = b ? TM_O1 : TM_O0;
            float vv[32];  // tokens 32 th .. 32 th + 31 of channel d_me
            tmem_ld32(tmem + lane_base + tm_o + 32 * th, vv);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars[8 + b]);  // read: this accumulator may take chunk c + 2
            __nv_bfloat16 *dst = p.out + ((size_t)tc * H + h) * D + d_me;
#pragma unroll
            for (int t = 0; t < 32; ++t)
                if (t < vc && KDA_ACCESS_OK(p.status, p.dbg.out, dst + (size_t)t * H * D, 2, 3))
                    st_stream_bf16(dst + (size_t)t * H * D, vv[t]);
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ---------------------------------------------------------------- consumer of a later segment
// Context parallelism: a segment g >= 1 of a long sequence runs its chain before the state it starts
// from is known. Its chunks see the true state S_j = S0_j + R_j S_start, where S0 is the chain from
// a zero state and R_j = F_{j-1} ... F_0 (F = I + M) the product of the segment's chunk transitions,
// so the output is O_j = O0_j + P_j R_j S_start. This consumer runs both chains on the same images,
//   S0^T += S0_b^T M^T + U~^T K^,   R^T += R_b^T M^T   (R^T starts at I),
// writes O0 = P S0_b + A U~ to `out`, and E_j = P_j R_j (computed transposed, E^T = R_b^T P^T) as a
// bf16 tile for the fix-up, and at its end S0 and R as fp32 for the scan. Every TMEM region is
// single-buffered (the two chains need 256 columns more than the plain consumer): the bf16 copies
// for chunk c + 1 are written once chunk c's outputs are complete.
namespace segc {
constexpr uint32_t TM_S = 0, TM_SB = 128, TM_R = 192, TM_RB = 320, TM_O = 384, TM_E = 448, TM_COLS = 512;
}  // namespace segc

__device__ void consumer_seg(const SplitParams &p, uint8_t *sm, int hd, int4 vi) {
    using namespace cons;
    using segc::TM_S; using segc::TM_SB; using segc::TM_R; using segc::TM_RB;
    using segc::TM_O; using segc::TM_E; using segc::TM_COLS;
    constexpr uint32_t I_C = idesc_bf16_f32(128, 128, false, 0, 0);   // X_b^T M^T (A in TMEM)
    constexpr uint32_t I_K = idesc_bf16_f32(128, 128, false, 1, 1);   // U~^T K^
    constexpr uint32_t I_OP = idesc_bf16_f32(128, 64, false, 0, 0);   // X_b^T P^T (A in TMEM)
    constexpr uint32_t I_OA = idesc_bf16_f32(128, 64, false, 1, 0);   // U~^T A^T
    // full0, full1, o0, o1, ready (bf16 copies written), free (O and E read), teardown
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC);
    // abort, tmem, first chunk whose R chain and E are not computed (R has decayed away)
    uint32_t *s_flags = reinterpret_cast<uint32_t *>(sm + MISC + 96);
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const int H = p.H, v = hd / H, h = hd % H;
    const int64_t bos = p.cu_seqlens[v], eos = p.cu_seqlens[v + 1];
    const int nchunks = (int)((eos - bos + C - 1) / C);
    auto r_live = [&](int c) { return c < (int)ld_volatile(&s_flags[2]); };
    float *s_end = p.seg_state + (size_t)hd * D * D;
    float *r_end = p.seg_trans + (size_t)hd * D * D;
    const bool ends_ok = KDA_ACCESS_OK(p.status, p.dbg.ws, s_end, D * D * 4, 4) &&
                         KDA_ACCESS_OK(p.status, p.dbg.ws, r_end, D * D * 4, 5);

    if (tid == 0) {
        s_flags[0] = 0;
        s_flags[2] = 0x7fffffffu;
        for (int k = 0; k < 7; ++k) mbar_init(&bars[k], (k == 4 || k == 5) ? NTC / 2 : 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&s_flags[1], TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_flags[1];
    auto fail = [&]() {
        s_flags[0] = 1;
        atomicOr(p.status, 1);
    };

    if (tid == LDR) {
        // ------------------------------------------------ loader thread (as in the plain consumer)
        int requested = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (ld_volatile(&s_flags[0])) break;
            if (!wait_flag_ge(p.filled + hd * RING + (c % RING), c + 1, p.timeout_ns)) { fail(); break; }
            fence_proxy_async_global();
            if (c >= 2) {
                if (!mbar_wait_bounded(&bars[2 + b], (uint32_t)((c - 2) >> 1) & 1u, p.timeout_ns)) { fail(); break; }
                st_release(p.consumed + hd, c - 1);
            }
            const uint8_t *src = p.ring + ((size_t)hd * RING + (size_t)(c % RING)) * SLOT;
            mbar_arrive_expect_tx(&bars[b], SLOT);
            bulk_load(sm + (b ? STAGE1 : STAGE0), src, SLOT, &bars[b]);
            requested = c + 1;
        }
        for (int c = requested - 2 < 0 ? 0 : requested - 2; c < requested; ++c)
            if (!mbar_wait_bounded(&bars[c & 1], (uint32_t)(c >> 1) & 1u, p.timeout_ns)) fail();
        if (requested == nchunks) st_release(p.consumed + hd, nchunks);
    } else if (tid == CTL) {
        // ------------------------------------------------ MMA thread
        uint32_t ph_ready = 0, ph_free = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (ld_volatile(&s_flags[0])) break;
            if (!mbar_wait_bounded(&bars[b], (uint32_t)(c >> 1) & 1u, p.timeout_ns)) { fail(); break; }
            if (!mbar_wait_bounded(&bars[4], ph_ready, p.timeout_ns)) { fail(); break; }
            ph_ready ^= 1u;
            tc_fence_after();
            const uint32_t st = sb + (b ? STAGE1 : STAGE0);
            const uint64_t dM = desc_k(st + SL_M, 16384, 0), dK = desc_mn(st + SL_KH, 8192, 0);
            const uint64_t dU = desc_mn(st + SL_U, 8192, 0);
            const uint64_t dP = desc_k(st + SL_P, 8192, 0), dA = desc_k(st + SL_A, 8192, 0);
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk)  // S0^T += S0_b^T M^T ...
                mma_bf16_ts(tmem + TM_S, tmem + TM_SB + 8 * kk, desc_k_at(dM, 16384, kk), I_C, 1);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // ... + U~^T K^
                mma_bf16_ss(tmem + TM_S, desc_mn_at(dU, kk), desc_mn_at(dK, kk), I_K, 1);
            const bool live = r_live(c);  // read after `ready`: the state warps set it before arriving
            if (live) {
#pragma unroll
                for (uint32_t kk = 0; kk < 8; ++kk)  // R^T += R_b^T M^T
                    mma_bf16_ts(tmem + TM_R, tmem + TM_RB + 8 * kk, desc_k_at(dM, 16384, kk), I_C, 1);
            }
            if (c >= 1) {  // the output warps have read O and E of chunk c - 1
                if (!mbar_wait_bounded(&bars[5], ph_free, p.timeout_ns)) { fail(); break; }
                ph_free ^= 1u;
            }
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk)  // O0^T = S0_b^T P^T ...
                mma_bf16_ts(tmem + TM_O, tmem + TM_SB + 8 * kk, desc_k_at(dP, 8192, kk), I_OP, kk > 0);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // ... + U~^T A^T
                mma_bf16_ss(tmem + TM_O, desc_mn_at(dU, kk), desc_k_at(dA, 8192, kk), I_OA, 1);
            if (live) {
#pragma unroll
                for (uint32_t kk = 0; kk < 8; ++kk)  // E^T = R_b^T P^T
                    mma_bf16_ts(tmem + TM_E, tmem + TM_RB + 8 * kk, desc_k_at(dP, 8192, kk), I_OP, kk > 0);
            }
            mma_commit(&bars[2 + b]);  // both chains, O, E and the stage are done
        }
        mma_commit(&bars[6]);
        mbar_wait_bounded(&bars[6], 0, p.timeout_ns);
    } else if (warp < 8) {
        // ------------------------------------------------ state warps (lane = value channel d for
        // S0^T, = column a of R for R^T; warps w and w + 4 take columns [64 hh, 64 hh + 64)); after
        // chunk c's outputs: the bf16 copies for chunk c + 1
        const int d_me = 32 * quad + lane;
        const int hh = warp >> 2;
        auto pack_store = [&](const float (&x)[32], uint32_t tm_b, int part) {
            uint32_t w[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) w[e] = pack2(x[2 * e], x[2 * e + 1]);
            tmem_st16(tmem + lane_base + tm_b + 32 * hh + 16 * part, w);
        };
        // S0^T = 0, R^T = I and their bf16 copies
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
            const uint32_t tm_x = which ? TM_R : TM_S, tm_b = which ? TM_RB : TM_SB;
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
                float x[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) x[e] = (which && 64 * hh + 32 * part + e == d_me) ? 1.f : 0.f;
                tmem_st32(tmem + lane_base + tm_x + 64 * hh + 32 * part, x);
                pack_store(x, tm_b, part);
            }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[4]);
        int dead_from = 0x7fffffff;  // the state warps' copy of s_flags[2]
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const bool last = c + 1 == nchunks;
            if (ld_volatile(&s_flags[0])) break;
            const bool ok = mbar_wait_bounded(&bars[2 + b], (uint32_t)(c >> 1) & 1u, p.timeout_ns);
            if (!ok) { fail(); break; }
            tc_fence_after();
            uint32_t rmax = 0;  // max |R| over this thread's columns (as float bits)
#pragma unroll 1
            for (int which = 0; which < 2; ++which) {
                if (which && !last && c + 1 > dead_from) continue;  // R decayed away: no copy needed
                const uint32_t tm_x = which ? TM_R : TM_S, tm_b = which ? TM_RB : TM_SB;
                float *dst_end = which ? r_end : s_end;
#pragma unroll 1
                for (int part = 0; part < 2; ++part) {
                    float x[32];
                    tmem_ld32(tmem + lane_base + tm_x + 64 * hh + 32 * part, x);
                    tmem_wait_ld();
                    if (which) {
#pragma unroll
                        for (int e = 0; e < 32; ++e) rmax = max(rmax, __float_as_uint(fabsf(x[e])));
                    }
                    if (!last) {
                        pack_store(x, tm_b, part);
                    } else if (ends_ok) {
                        // row d_me of S0^T (or column d_me of R) -> element [c][d_me]
                        float *dst = dst_end + (size_t)(64 * hh + 32 * part) * D + d_me;
#pragma unroll
                        for (int e = 0; e < 32; ++e) dst[(size_t)e * D] = x[e];
                    }
                }
            }
            if (!last && dead_from == 0x7fffffff) {
                // has R decayed away? (all 256 state threads: named barrier 3 with an OR)
                uint32_t any_alive;
                asm volatile(
                    "{\n\t.reg .pred p, q;\n\t"
                    "setp.ge.f32 q, %1, %2;\n\t"
                    "bar.red.or.pred p, 3, 256, q;\n\t"
                    "selp.u32 %0, 1, 0, p;\n\t}"
                    : "=r"(any_alive)
                    : "f"(__uint_as_float(rmax)), "f"(kSegDeadR)
                    : "memory");
                if (!any_alive) {
                    dead_from = c + 1;
                    if (tid == 0) s_flags[2] = (uint32_t)dead_from;  // seen by the MMA thread after `ready`
                }
            }
            if (!last) {
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[4]);
            }
        }
        if (tid == 0 && !ld_volatile(&s_flags[0]))
            p.e_live[hd] = dead_from < nchunks ? dead_from : nchunks;
        tc_fence_before();
    } else if (tid < NTC) {
        // ------------------------------------------------ output warps: O0 -> out, E^T -> its tile;
        // warps w and w + 4 (w = 8..11) take tokens [32 th, 32 th + 32)
        const int d_me = 32 * quad + lane;  // value channel of O0^T, row a of E^T
        const int th = (warp >> 2) & 1;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (ld_volatile(&s_flags[0])) break;
            const bool ok = mbar_wait_bounded(&bars[2 + b], (uint32_t)(c >> 1) & 1u, p.timeout_ns);
            if (!ok) { fail(); break; }
            tc_fence_after();
            const int64_t tc = bos + (int64_t)c * C + 32 * th;
            const int vc = (int)(eos - tc < 32 ? eos - tc : 32);
            // E^T row a = d_me, tokens 32 th .. + 31: four 16-byte chunks of a 128-byte swizzled
            // row of the [128][64] bf16 tile
            uint8_t *et = p.e_tiles + ((size_t)(vi.w + c) * H + h) * 16384 + (uint32_t)(d_me >> 3) * 1024 +
                          (uint32_t)(d_me & 7) * 128;
            const bool et_ok = KDA_ACCESS_OK(p.status, p.dbg.ws, et, 128, 6);
            float x[32];
            // E of a chunk after R decayed away was not computed (a late view of the flag only
            // writes a tile the fix-up never reads: it stops at the segment's live count)
            if (r_live(c)) {
                tmem_ld32(tmem + lane_base + TM_E + 32 * th, x);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint32_t q8 = 4 * th + q4;
                    if (et_ok) st_chunk(et + ((q8 ^ (uint32_t)(d_me & 7)) << 4), x + 8 * q4);
                }
            }
            tmem_ld32(tmem + lane_base + TM_O + 32 * th, x);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars[5]);  // read: O and E may take chunk c + 1
            __nv_bfloat16 *dst = p.out + ((size_t)tc * H + h) * D + d_me;
#pragma unroll
            for (int t = 0; t < 32; ++t)
                if (t < vc && KDA_ACCESS_OK(p.status, p.dbg.out, dst + (size_t)t * H * D, 2, 7))
                    st_stream_bf16(dst + (size_t)t * H * D, x[t]);
        }
        tc_fence_before();
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ---------------------------------------------------------------- producer (key-side half)
namespace prod {
constexpr uint32_t QK0 = 0, QK1 = 32768;  // raw q/k -> Q~/K~ -> P over Q~ (128-row tiles, 16 KB blocks)
constexpr uint32_t LA = 65536;            // raw log_alpha fp32 [t][c]
constexpr uint32_t VB = LA + 32768;       // V [j][d] -> U~
constexpr uint32_t KI = VB + 16384;       // K- [j][c]; with WN after it: M [c][c'] (2 x 16 KB)
constexpr uint32_t WN = KI + 16384;       // -W [j][c]
constexpr uint32_t KH = WN + 16384;       // K^ [j][c]
constexpr uint32_t TT = KH + 16384;       // T' [i][j]   \  [T'; 0] and [0; A]: 128-row
constexpr uint32_t ZB = TT + 8192;        // zero block   |  K-major operands
constexpr uint32_t AQK = ZB + 8192;       // A [i][j]    /
constexpr uint32_t LT = AQK + 8192;       // L -> T fp32 [64][LT_LD]
constexpr uint32_t PB = LT + 64 * LT_LD * 4;   // 32 x PB_LD fp32
constexpr uint32_t MISC = PB + 32 * PB_LD * 4; // beta, gamma, psum, flags, barriers
constexpr uint32_t PSUM_FLOATS = (NTC / 32 + 1) * 128;  // group totals per compute warp, chunk totals
constexpr uint32_t BYTES = MISC + 64 * 4 + 2 * 128 * 4 + PSUM_FLOATS * 4 + 64 + 10 * 8 + 4 * 32;
// TMEM: D1 = [Q~; K~] K-^T (M=128, 64 columns), W (M=64), D3 = [U~; -A W], D4 = -K^^T W
constexpr uint32_t TM_D1 = 0, TM_W = 128, TM_D3 = 256, TM_D4 = 384, TM_COLS = 512;
// Tiles of the tensor-core inverse (build option KDA_TC_INVERSE; 64x64 bf16, 8 KB each), over
// regions dead during it. The
// identity sits 8 KB after L_off, so [L_off | I] is one MN-major B operand of two 64-column
// blocks; N overwrites the identity once the first MMA has read it.
constexpr uint32_t IV_DINV = KI, IV_LOFF = KI + 8192, IV_EYE = IV_LOFF + 8192, IV_N = IV_EYE;
constexpr uint32_t IV_N2 = LT, IV_W1 = LT + 8192;
static_assert(IV_EYE == WN && IV_N2 % 1024 == 0 && IV_W1 + 8192 <= MISC, "inverse tiles");
}  // namespace prod

// Producer roles: the compute threads run the gating, the TMEM epilogues and the inverse; the
// control thread claims the items, issues the MMAs, the log_alpha loads and the first item's
// q/k; the store thread waits for a free ring slot, copies each image out in two parts with bulk
// stores, issues the next items' V and q/k loads into the buffers it has just read, and
// publishes the image. The phases are separated by barriers of the compute threads and the
// control warp.
template <bool PRO>
__device__ void producer(const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                         const CUtensorMap *tm_la, const SplitParams &p, uint8_t *sm, int pid, int nprod) {
    using namespace prod;
    constexpr uint32_t I_D1 = idesc_bf16_f32(128, 64);
    constexpr uint32_t I_W = idesc_bf16_f32(64, 128, false, 0, 1);
    constexpr uint32_t I_3 = idesc_bf16_f32(128, 128, false, 0, 1);
    constexpr uint32_t I_4 = idesc_bf16_f32(128, 128, false, 1, 1);
#ifdef KDA_TC_INVERSE
    constexpr uint32_t I_IV = idesc_bf16_f32(64, 64, false, 0, 1);   // inverse steps
    constexpr uint32_t I_IVN = idesc_bf16_f32(64, 64, true, 0, 1);   // the same, A negated
    constexpr uint32_t I_IV2 = idesc_bf16_f32(64, 128, false, 0, 1); // D^-1 [L_off | I]
#endif
    float *s_beta = reinterpret_cast<float *>(sm + MISC);
    float *s_gamma = s_beta + 64;
    float *s_psum = s_gamma + 2 * 128;  // s_gamma: one row of 128 per item in flight
    uint32_t *s_flags = reinterpret_cast<uint32_t *>(s_psum + PSUM_FLOATS);  // abort, tmem, gate
    // qk0, qk1, la, v (TMA loads), mma (W, D3/D4), srcM, img2, img1, src1 (hand-off of an image's two
    // parts), d1 (D1)
    uint64_t *bars = reinterpret_cast<uint64_t *>(s_flags + 16);
    float *LTp = reinterpret_cast<float *>(sm + LT);
#ifndef KDA_TC_INVERSE
    float *PBp = reinterpret_cast<float *>(sm + PB);
#endif
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // TMEM epilogues: warp w reads lanes 32 (w % 4) .. + 31, column part w / 4 of four
    const int quad = warp & 3, part = warp >> 2;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const bool compute = tid < NTC, ctl = tid == CTL;
    const int H = p.H;
    // Dynamic assignment: items k = chunk * heads + head are claimed from one counter in that
    // (chunk-major) order, so every head advances at the producers' common rate. A producer's
    // item only waits on consumption of earlier chunks of its head, whose items were claimed
    // earlier and are finished by producers that never wait on anything later: no cycle.
    (void)pid;
    (void)nprod;
    struct Item {
        int hd, c, h;
        int64_t bos, eos;
    };
    auto decode = [&](int k) -> Item {
        Item it;
        it.hd = k % p.heads;
        it.c = k / p.heads;
        it.h = it.hd % H;
        it.bos = p.cu_seqlens[it.hd / H];
        it.eos = p.cu_seqlens[it.hd / H + 1];
        return it;
    };
    // control thread: the next item with a chunk to make, or -1 when none is left
    auto claim = [&]() -> int {
        while (true) {
            const int k = atomicAdd(p.next_item, 1);
            const int c = k / p.heads, hdk = k % p.heads;
            if (c >= p.max_chunks) return -1;
            const int64_t len = p.cu_seqlens[hdk / H + 1] - p.cu_seqlens[hdk / H];
            if ((int64_t)c * C < len) return k;
        }
    };
    // Item n's record, rec[n % 4]: {head, chunk, head within the sequence, first token, valid
    // tokens} (head < 0: no item n). The control thread decodes each item it claims once; nothing
    // else reads cu_seqlens, so no thread stalls on a global load for it. Record n + 2 is written
    // during item n's gating and read from iteration n + 1 on (behind the barrier that ends it).
    struct ItemRec {
        int hd, c, h, t0, valid, pad[3];
    };
    ItemRec *s_rec = reinterpret_cast<ItemRec *>(bars + 10);
    auto put_rec = [&](int n, int k) {  // control thread
        ItemRec r;
        r.hd = -1;
        if (k >= 0) {
            const Item it = decode(k);
            r.hd = it.hd;
            r.c = it.c;
            r.h = it.h;
            const int64_t t0 = it.bos + (int64_t)it.c * C;
            r.t0 = (int)t0;
            r.valid = (int)(it.eos - t0 < C ? it.eos - t0 : C);
        }
        s_rec[n & 3] = r;
    };

    if (tid == 0) {
        s_flags[0] = 0;
        s_flags[7] = 0xffffffffu;  // *s_nimg = -1: items still running
        for (int k = 0; k < 10; ++k) mbar_init(&bars[k], 1);
        fence_mbarrier_init();
        prefetch_tmap(tm_q);
        prefetch_tmap(tm_k);
        prefetch_tmap(tm_v);
        prefetch_tmap(tm_la);
    }
    if (warp == 0) {
        tmem_alloc(&s_flags[1], TM_COLS);
        tmem_relinquish();
    }
    for (int e = tid; e < 16384 / 16; e += NTS)  // T' (its strictly upper 16x16 blocks) and ZB stay zero
        reinterpret_cast<uint4 *>(sm + TT)[e] = make_uint4(0u, 0u, 0u, 0u);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_flags[1];
    auto fail = [&]() {
        s_flags[0] = 1;
        atomicOr(p.status, 1);
    };

    // control thread; each buffer's previous contents were read by generic loads or bulk stores
    // that have completed (see the call sites). Inputs are read once: evict-first, so that the
    // stream of them does not push the ring's images out of L2.
    auto issue_qk = [&](const ItemRec &r, int b) {
        const int h = r.h, t0 = r.t0;
        uint8_t *qk = sm + (b ? QK1 : QK0);
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[b], 32768);
        tma_load_3d_pol(qk, tm_q, &bars[b], 0, h, (int32_t)t0, l2_evict_first());
        tma_load_3d_pol(qk + 8192, tm_k, &bars[b], 0, h, (int32_t)t0, l2_evict_first());
        tma_load_3d_pol(qk + 16384, tm_q, &bars[b], 64, h, (int32_t)t0, l2_evict_first());
        tma_load_3d_pol(qk + 24576, tm_k, &bars[b], 64, h, (int32_t)t0, l2_evict_first());
    };
    auto issue_la = [&](const ItemRec &r) {
        const int h = r.h, t0 = r.t0;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[2], 32768);
        tma_load_3d_pol(sm + LA, tm_la, &bars[2], 0, h, (int32_t)t0, l2_evict_first());
    };
    auto issue_v = [&](const ItemRec &r) {
        const int h = r.h, t0 = r.t0;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&bars[3], 16384);
        tma_load_3d_pol(sm + VB, tm_v, &bars[3], 0, h, (int32_t)t0, l2_evict_first());
        tma_load_3d_pol(sm + VB + 8192, tm_v, &bars[3], 64, h, (int32_t)t0, l2_evict_first());
    };
    auto load_beta = [&](const ItemRec &r) -> float {  // tid < C
        if (r.hd < 0 || tid >= r.valid) return 0.f;
        const float *bp = p.beta + (size_t)(r.t0 + tid) * H + r.h;
        if (!KDA_ACCESS_OK(p.status, p.dbg.beta, bp, 4, 8)) return 0.f;
        const float b = *bp;
        return (PRO && (p.pro.flags & KDA_PROLOGUE_BETA_SIGMOID)) ? beta_from_raw(b) : b;
    };
    // Hand-off of image n to the store thread, in two parts: the key-side part (K^ and A, final
    // once item n's A/L extraction is done) and the rest (M, U~, P, after item n's epilogue, one
    // iteration later). Entry n % 2 = {head, chunk, QK buffer} is written with the first part and
    // rewritten for image n + 2 only after the store thread has read image n + 1's first part
    // (src1), by which time it has finished image n. img1 / img2: one arrival per part; src1 /
    // srcM: the store thread has read the first part's sources / the rest's M, which may then be
    // rewritten. The rest's P and U~ buffers take the next items' loads, which the store thread
    // issues itself once it has read them (before M's copy, so the loads do not queue behind
    // it): V of item n + 1 over U~, q/k of item n + 2 over P. Neither
    // barrier gets two phases ahead of its waiters (each part of image n + 1 is handed over only
    // after a wait for the same part of image n). The end of the items is not an arrival but a
    // count, *s_nimg = images handed over in all.
    volatile int32_t *s_store = reinterpret_cast<volatile int32_t *>(s_flags + 8);
    volatile int32_t *s_nimg = reinterpret_cast<volatile int32_t *>(s_flags + 7);
    uint64_t *const b_mma = &bars[4], *const b_srcM = &bars[5], *const b_img2 = &bars[6];
    uint64_t *const b_img1 = &bars[7], *const b_src1 = &bars[8], *const b_d1 = &bars[9];

    if (ctl) {
        const int k0 = claim();
        put_rec(0, k0);
        put_rec(1, k0 >= 0 ? claim() : -1);
        if (k0 >= 0) {
            issue_qk(s_rec[0], 0);
            issue_la(s_rec[0]);
        }
    }
    __syncthreads();
    if (warp == STR / 32) {
        if (tid == STR) {
            // ------------------------------------------------ store thread
            // Per image, in item order: the first part once handed over (after a wait for its
            // ring slot's previous chunk to have been taken), then the rest; each part's sources
            // are released once the copies have read them, and the image is published once all
            // its copies are complete.
            auto wait_part = [&](uint64_t *bar, uint32_t ph) -> bool {
                const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
                while (true) {
                    if (mbar_try_wait(bar, ph)) return true;
                    if (ld_volatile(&s_flags[0]) != 0 || globaltimer_ns() > deadline) return false;
                    __nanosleep(64);
                }
            };
            // Loads it issues: V of item i on bars[3] (phase i), q/k of item i on bars[i % 2] (phase
            // i / 2); the last of each is waited for before the thread ends.
            int last_v = -1, last_qk0 = -1, last_qk1 = -1;
            auto load_v = [&](int i) {
                if (s_rec[i & 3].hd < 0) return;
                issue_v(s_rec[i & 3]);
                last_v = i;
            };
            auto load_qk = [&](int i) {
                if (s_rec[i & 3].hd < 0) return;
                issue_qk(s_rec[i & 3], i & 1);
                (i & 1 ? last_qk1 : last_qk0) = i;
            };
            load_v(0);   // into free buffers
            load_qk(1);
            uint32_t ph1 = 0, ph2 = 0;
            for (int n = 0;; ++n) {
                // image n's first part handed over, or the item loop ended with n images
                bool have = false, ended = false;
                const uint64_t deadline = globaltimer_ns() + p.timeout_ns;
                while (true) {
                    if (mbar_try_wait(b_img1, ph1)) { have = true; break; }
                    const int ni = *s_nimg;
                    if (ni >= 0 && ni <= n) { ended = true; break; }
                    if (ld_volatile(&s_flags[0]) != 0 || globaltimer_ns() > deadline) break;
                    __nanosleep(64);
                }
                if (!have) {
                    if (!ended) fail();
                    break;
                }
                ph1 ^= 1u;
                volatile int32_t *e = s_store + 4 * (n & 1);
                const int hd = e[0], c = e[1];
                const uint32_t b_img = (uint32_t)e[2];
                bool ok = c < RING || wait_flag_ge(p.consumed + hd, c - RING + 1, p.timeout_ns);
                uint8_t *slot = p.ring + ((size_t)hd * RING + (size_t)(c % RING)) * SLOT;
                if (ok) {
                    bulk_store(slot + SL_KH, sm + KH, 16384);
                    bulk_store(slot + SL_A, sm + AQK, 8192);
                    bulk_commit();
                    bulk_wait_read();
                }
                mbar_arrive(b_src1);  // (also on failure: the compute threads then see the stop)
                ok = ok && wait_part(b_img2, ph2);
                ph2 ^= 1u;
                if (ok) {  // P and U~ first: their buffers take the next items' loads
                    const uint8_t *qkb = sm + (b_img ? QK1 : QK0);
                    bulk_store(slot + SL_P, qkb, 8192);             // P, columns 0..63 (over Q~)
                    bulk_store(slot + SL_P + 8192, qkb + 16384, 8192);  // and 64..127
                    bulk_store(slot + SL_U, sm + VB, 16384);
                    bulk_commit();
                    bulk_wait_read();
                    load_v(n + 1);
                    load_qk(n + 2);
                    bulk_store(slot + SL_M, sm + KI, 32768);       // M: K- and W regions, contiguous
                    bulk_commit();
                    bulk_wait_read();
                }
                mbar_arrive(b_srcM);
                if (!ok) {
                    fail();
                    break;
                }
                bulk_wait_all();
                fence_proxy_async_global();
                __threadfence();
                st_release(p.filled + hd * RING + (c % RING), c + 1);
            }
            bulk_wait_all();
            if (last_v >= 0) mbar_wait_bounded(&bars[3], (uint32_t)(last_v & 1), p.timeout_ns);
            if (last_qk0 >= 0) mbar_wait_bounded(&bars[0], (uint32_t)((last_qk0 >> 1) & 1), p.timeout_ns);
            if (last_qk1 >= 0) mbar_wait_bounded(&bars[1], (uint32_t)((last_qk1 >> 1) & 1), p.timeout_ns);
        }
    } else {
    // Phase parities of the waited barriers and the control thread's loads in flight (q/k of item
    // 0, log_alpha), as bits of one word (the loop is at the register limit): parity of bars[k]
    // at bit k (k = 0..4: qk0, qk1, la, v, mma; bit 5: d1), load in flight at bit 8 + k. V and
    // the later q/k loads are the store thread's, which waits for its own.
    constexpr int B_MMA = 4, B_D1 = 5, PEND = 8;
    uint32_t phs = 0;
    auto wait_bar = [&](uint64_t *bar, int bit) {
        const bool ok = mbar_wait_bounded(bar, (phs >> bit) & 1u, p.timeout_ns);
        phs ^= 1u << bit;
        if (!ok) fail();
    };
    auto pend = [&](int k, bool on) { phs = on ? (phs | (1u << (PEND + k))) : (phs & ~(1u << (PEND + k))); };
    if (s_rec[0].hd >= 0) {
        pend(0, true);
        pend(2, true);
    }
    float beta_next = (tid < C) ? load_beta(s_rec[0]) : 0.f;
    int n_img = 0;
    // Iteration n runs the early phases of item n (E) and the late phases of item n - 1 (P), so
    // that each item's MMAs run while the compute threads work on the other item:
    //   a. P: W -> its tile; D3/D4(P) issued
    //   b. E: gating (D3/D4(P) run); D1(E) issued
    //   c. P: epilogue (D1(E) runs); the rest of image P to the store thread
    //   d. E: K^ to its tile, A and L; image E's first part to the store thread; log_alpha of E + 1
    //   e. E: inverse; W(E) issued
    // Item E's buffers: QK[n % 2], s_gamma[n % 2]; item P's: the others. Every phase ends with a
    // barrier of the compute threads and the control warp.
    for (int n = 0;; ++n) {
        const ItemRec &cur = s_rec[n & 3], &nx = s_rec[(n + 1) & 3];  // read where used
        const bool hasE = cur.hd >= 0, hasP = n > 0;
        if (!hasE && !hasP) break;
        uint8_t *const qkE = sm + ((n & 1) ? QK1 : QK0), *const qkP = sm + ((n & 1) ? QK0 : QK1);
        float *const gamE = s_gamma + 128 * (n & 1), *const gamP = s_gamma + 128 * ((n - 1) & 1);
        const uint32_t parP = (uint32_t)((n - 1) & 1), parPP = (uint32_t)(n & 1);  // phases of images n - 1, n - 2
        uint32_t ph_d34 = 0;

        // ---- a. item n - 1: W -> its tile (over M's second half of image n - 2), then D3/D4:
        // D3 = [T'; 0] V + [0; A] (-W) = [U~; -A W] and D4 = K^^T (-W)
        if (hasP) {
            wait_bar(b_mma, B_MMA);
            tc_fence_after();
            if (compute) {
                if (n >= 2 && !mbar_wait_bounded(b_srcM, parPP, p.timeout_ns)) fail();
                rows64_to_tile<32>(tmem + lane_base + TM_W + 32 * part, sm + WN, 8192, 32 * part, quad, lane, -1.f);
                fence_proxy_async_smem();
            }
            tc_fence_before();
            sync_work();
            if (ctl) {
                if (!mbar_wait_bounded(&bars[3], (phs >> 3) & 1u, p.timeout_ns)) fail();
                tc_fence_after();
#pragma unroll
                for (uint32_t kk = 0; kk < 4; ++kk)
                    mma_bf16_ss(tmem + TM_D3, desc_k(sb + TT, 16384, kk), desc_mn(sb + VB, 8192, kk), I_3, kk > 0);
#pragma unroll
                for (uint32_t kk = 0; kk < 4; ++kk)
                    mma_bf16_ss(tmem + TM_D3, desc_k(sb + ZB, 16384, kk), desc_mn(sb + WN, 8192, kk), I_3, 1);
#pragma unroll
                for (uint32_t kk = 0; kk < 4; ++kk)
                    mma_bf16_ss(tmem + TM_D4, desc_mn(sb + KH, 8192, kk), desc_mn(sb + WN, 8192, kk), I_4, kk > 0);
                mma_commit(b_mma);
            }
            phs ^= 1u << 3;
            ph_d34 = (phs >> B_MMA) & 1u;
        }

        // ---- b. item n: the gating. K- goes to the L/T scratch and K^ to the log_alpha buffer,
        // so the factored path writes nothing item n - 1 still needs; the exact path also writes A
        // over item n - 1's, so it first waits for D3 (which reads it) and for the store thread.
        if (hasE) {
            if (tid < C) s_beta[tid] = beta_next;
            wait_bar(&bars[n & 1], n & 1);
            wait_bar(&bars[2], 2);
            pend(n & 1, false);
            pend(2, false);
            if (tid < C) beta_next = load_beta(nx);
            if (compute) {
                const int g = gate_chunk<PRO, NTC, true>(qkE, reinterpret_cast<uint8_t *>(LTp), sm + AQK,
                                                         reinterpret_cast<float *>(sm + LA), LTp, s_beta, gamE,
                                                         s_psum, s_flags, cur.valid, tid, sm + LA,
                                                         hasP ? b_mma : nullptr, ph_d34, p.timeout_ns, p.pro,
                                                         hasP ? b_src1 : nullptr, parP);
                if (g < 0) atomicOr(p.status, 1);
                if (tid == 0) s_flags[2] = (uint32_t)(g + 1);
                fence_proxy_async_smem();
            }
            // the item after the next one, claimed while the compute threads run the gating; read
            // by all after the following barriers. Its record slot last served item n - 2.
            if (ctl) put_rec(n + 2, nx.hd >= 0 ? claim() : -1);
        }
        if (sync_work_or(ld_volatile(&s_flags[0]) != 0)) break;
        const int gate = hasE ? (int)s_flags[2] - 1 : 0;
        if (gate < 0) break;
        const bool exactE = gate == 1;
        if (ctl && hasE) {
            tc_fence_after();
            if (!exactE) {
#pragma unroll
                for (uint32_t kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tmem + TM_D1, desc_k(smem_u32(qkE), 16384, kk), desc_k(sb + LT, 8192, kk), I_D1,
                                kk > 0);
            }
            mma_commit(b_d1);
        }

        // ---- c. item n - 1: the epilogue. D3 rows 0..63: U~ [j][d] over V; rows 64..127: P =
        // Q~ - A W over Q~; D4 -> M = diag(gamma - 1) - K^^T W [c][c'] over K- and W.
        if (hasP) {
            wait_bar(b_mma, B_MMA);
            tc_fence_after();
            if (compute) {
                const int r = 32 * quad + lane;  // TMEM lane
                const int col = 32 * part;       // this thread's 32 columns of D3 and D4
                float v[32], m[32];  // both loads in flight before one wait
                tmem_ld32(tmem + lane_base + TM_D3 + col, v);
                tmem_ld32(tmem + lane_base + TM_D4 + col, m);
                tmem_wait_ld();
                if (r < 64) {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8)
                        st_chunk(sm + VB + tchunk(8192, r, col + 8 * q8), v + 8 * q8);
                } else {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        uint8_t *qp = qkP + tchunk(16384, r - 64, col + 8 * q8);
                        const uint4 raw = *reinterpret_cast<const uint4 *>(qp);
                        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
                            v[8 * q8 + 2 * e] += f.x;
                            v[8 * q8 + 2 * e + 1] += f.y;
                        }
                        st_chunk(qp, v + 8 * q8);
                    }
                }
                const float gm1 = gamP[r] - 1.f;
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (col + e == r) m[e] += gm1;
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    st_chunk(sm + KI + tchunk(16384, r, col + 8 * q8), m + 8 * q8);
                fence_proxy_async_smem();  // written by generic stores; the copy-out is async
            }
            tc_fence_before();
            if (sync_work_or(ld_volatile(&s_flags[0]) != 0)) break;
            if (ctl) mbar_arrive(b_img2);
        }
        if (!hasE) break;  // the last item's late phases were the last work

        // ---- d. item n: K^ to its tile and A, L from D1 (over item n - 1's K^ and A, once the
        // store thread has taken them; D4 and D3, which read them too, are complete)
        wait_bar(b_d1, B_D1);
        tc_fence_after();
        if (compute) {
            if (hasP && !mbar_wait_bounded(b_src1, parP, p.timeout_ns)) fail();
            for (int e = tid; e < 16384 / 16; e += NTC)  // K^: log_alpha buffer -> its image slot
                reinterpret_cast<uint4 *>(sm + KH)[e] = reinterpret_cast<const uint4 *>(sm + LA)[e];
            if (!exactE)
                extract_al<16>(tmem + lane_base + TM_D1 + 16 * part, sm + AQK, LTp, s_beta, 32 * quad + lane,
                               16 * part);
            fence_proxy_async_smem();
        }
        tc_fence_before();
        if (sync_work_or(ld_volatile(&s_flags[0]) != 0)) break;
        if (ctl) {
            if (nx.hd >= 0) issue_la(nx);  // K^ has left the log_alpha buffer
            volatile int32_t *e = s_store + 4 * (n & 1);
            e[0] = cur.hd;
            e[1] = cur.c;
            e[2] = n & 1;
            mbar_arrive(b_img1);
        }
        if (nx.hd >= 0) pend(2, true);
        ++n_img;

        // ---- e. item n: T' = (I + L)^-1 diag(beta), then W = T' K~
#ifdef KDA_TC_INVERSE
        // (build option) on the tensor cores, three rounds of MMAs (inv_tc_setup):
        //   1: [N | D^-1] = D^-1 [L_off | I]            (one N = 128 MMA: D^-1 lands in TMEM)
        //   2: W1 = D^-1 - N D^-1 (onto D^-1), N2 = N N
        //   3: T = W1 + N2 W1 (onto W1) = (I + N2)(I - N) D^-1
        // Tiles: D^-1 and L_off over K-, I and then N over W (both regions hold image n - 1's M
        // until the store thread has read it), N2 and W1 over the L/T scratch (L is read in step
        // 0). Accumulators: the W and D3 columns, free until those MMAs.
        if (compute) {
            if (hasP && !mbar_wait_bounded(b_srcM, parP, p.timeout_ns)) fail();
            inv_tc_setup<NTC>(LTp, sm + IV_DINV, sm + IV_LOFF, tid, warp, sm + IV_EYE);
            fence_proxy_async_smem();
        }
        tc_fence_before();
        sync_work();
        if (ctl) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + TM_W, desc_k(sb + IV_DINV, 8192, kk), desc_mn(sb + IV_LOFF, 8192, kk), I_IV2, kk > 0);
            mma_commit(b_mma);
        }
        wait_bar(b_mma, B_MMA);
        tc_fence_after();
        if (compute) {
            acc64_cols16_to_tile(tmem + lane_base + TM_W, sm + IV_N, 16 * part, quad, lane,
                                 [](int, int, float x) { return x; });
            fence_proxy_async_smem();
        }
        tc_fence_before();
        sync_work();
        if (ctl) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // W1 = D^-1 - N D^-1
                mma_bf16_ss(tmem + TM_W + 64, desc_k(sb + IV_N, 8192, kk), desc_mn(sb + IV_DINV, 8192, kk), I_IVN, 1);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // N2 = N N
                mma_bf16_ss(tmem + TM_D3, desc_k(sb + IV_N, 8192, kk), desc_mn(sb + IV_N, 8192, kk), I_IV, kk > 0);
            mma_commit(b_mma);
        }
        wait_bar(b_mma, B_MMA);
        tc_fence_after();
        if (compute) {
            acc64_cols16_to_tile(tmem + lane_base + TM_W + 64, sm + IV_W1, 16 * part, quad, lane,
                                 [](int, int, float x) { return x; });
            acc64_cols16_to_tile(tmem + lane_base + TM_D3, sm + IV_N2, 16 * part, quad, lane,
                                 [](int, int, float x) { return x; });
            fence_proxy_async_smem();
        }
        tc_fence_before();
        sync_work();
        if (ctl) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // T = W1 + N2 W1
                mma_bf16_ss(tmem + TM_W + 64, desc_k(sb + IV_N2, 8192, kk), desc_mn(sb + IV_W1, 8192, kk), I_IV, 1);
            mma_commit(b_mma);
        }
        wait_bar(b_mma, B_MMA);
        tc_fence_after();
        if (compute) {
            acc64_cols16_to_tile(tmem + lane_base + TM_W + 64, sm + TT, 16 * part, quad, lane,
                                 [s_beta](int, int c, float x) { return x * s_beta[c]; });
            fence_proxy_async_smem();
        }
        tc_fence_before();
#else
        if (compute) {
            // warps 0..3, one per SM sub-partition
            invert_unit_lower<NTC>(LTp, PBp, sm + TT, s_beta, tid, warp);
            fence_proxy_async_smem();
        }
#endif
        if (sync_work_or(ld_volatile(&s_flags[0]) != 0)) break;
        if (ctl) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // W = T' K~
                mma_bf16_ss(tmem + TM_W, desc_k(sb + TT, 8192, kk), desc_mn(smem_u32(qkE) + 8192, 16384, kk), I_W,
                            kk > 0);
            mma_commit(b_mma);
        }
    }

    if (ctl) {
        *s_nimg = n_img;  // no more images: the store thread ends after image n_img - 1
        for (int k = 0; k < 3; k += 2)  // q/k of item 0, log_alpha
            if ((phs >> (PEND + k)) & 1u) mbar_wait_bounded(&bars[k], (phs >> k) & 1u, p.timeout_ns);
        mma_commit(b_mma);
        mbar_wait_bounded(b_mma, (phs >> B_MMA) & 1u, p.timeout_ns);
    }
    }  // the work warps
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

constexpr uint32_t SPLIT_SMEM = (cons::BYTES > prod::BYTES ? cons::BYTES : prod::BYTES) + 1024;

template <bool PRO>
__global__ void __launch_bounds__(NTS, 1)
split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_la,
             const SplitParams p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned (128-byte swizzled tiles); offsetting the shared array itself keeps the
    // accesses in the shared state space (an integer round trip would make them generic)
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    // The consumers are the last `heads` blocks. Measured on two B200s (plain 1M-token, 16-head
    // prefill): consumers as the first blocks 24.5 and 31.9 ms, as the last blocks 20.7 and 20.8 ms,
    // spread evenly over the grid 29.3 ms (first GPU). The first blocks of a launch are
    // spread over the whole chip, so consumers among them probably share their part of the chip
    // (and its path to L2) with busy producers; the last blocks fill the SMs left over.
    const int first_cons = (int)gridDim.x - p.heads;
    if ((int)blockIdx.x >= first_cons) {
        const int hd = (int)blockIdx.x - first_cons;
        const int4 vi = p.vinfo ? p.vinfo[hd / p.H] : make_int4(0, 0, 1, 0);
        if (vi.y > 0)
            consumer_seg(p, sm, hd, vi);
        else
            consumer(p, sm, hd);
    } else
        producer<PRO>(&tm_q, &tm_k, &tm_v, &tm_la, p, sm, blockIdx.x, first_cons);
}

// Zeroes the status word and the ring flags.
__global__ void split_init_kernel(int32_t *status, int32_t *flags, int nflags) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nflags; i += gridDim.x * blockDim.x)
        flags[i] = 0;
}

int sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms;
}

size_t flags_bytes(int64_t heads) { return ((size_t)heads * (RING + 2) * 4 + 1023) / 1024 * 1024; }

}  // namespace

bool split_eligible(int64_t heads, kda_dtype_t dtype, int32_t dk, int32_t dv) {
    return dtype == KDA_BF16 && dk == D && dv == D && heads > 0 && heads * 4 <= sm_count();
}

bool split_eligible_seqs(int32_t num_seqs) { return num_seqs >= 1; }

size_t split_workspace_bytes(int64_t heads) {
    return 1024 + flags_bytes(heads) + (size_t)heads * RING * SLOT;
}

cudaError_t launch_prefill_split(const Problem &p, int32_t max_chunks, void *workspace,
                                 cudaStream_t stream, uint64_t timeout_ns, bool *not_coresident) {
    *not_coresident = false;
    // with context parallelism every segment is a chain of its own
    const int64_t heads = (int64_t)(p.seg ? p.seg->num_vseqs : p.num_seqs) * p.H;
    const int sms = sm_count();
    int per_sm = 0;
    static PerDeviceOnce<> once_plain, once_pro;
    const void *kern = p.pro.flags ? (const void *)split_kernel<true> : (const void *)split_kernel<false>;
    cudaError_t e = set_smem_limit_once(p.pro.flags ? once_pro : once_plain, kern, (int)SPLIT_SMEM);
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, NTS, SPLIT_SMEM);
    if (e != cudaSuccess) return e;
    const int grid = per_sm * sms;
    // Fewer resident blocks than the launch needs (fewer SMs visible, e.g. a partitioned
    // context): nothing is enqueued and the caller runs the single-role kernel instead.
    if (!split_coresident(per_sm, sms, heads)) {
        *not_coresident = true;
        return cudaSuccess;
    }

    CUtensorMap mq, mk, mv, mla;
    const uint64_t T = (uint64_t)p.total_tokens, H = (uint64_t)p.H;
    if (!make_token_map(&mq, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_token_map(&mk, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_token_map(&mv, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_token_map(&mla, p.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, H, T, D, false))
        return cudaErrorInvalidValue;

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *ring = ws + 1024 + flags_bytes(heads);  // 1024-byte aligned: slots are too (SLOT % 1024 == 0)
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    int32_t *flags = reinterpret_cast<int32_t *>(ws + 1024);
    const int nflags = (int)(heads * (RING + 2));
    split_init_kernel<<<(nflags + 255) / 256, 256, 0, stream>>>(status, flags, nflags);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    SplitParams sp;
    sp.cu_seqlens = p.seg ? p.seg->vcu : p.cu_seqlens;
    sp.vinfo = p.seg ? p.seg->vinfo : nullptr;
    sp.seg_state = p.seg ? p.seg->seg_state : nullptr;
    sp.seg_trans = p.seg ? p.seg->seg_trans : nullptr;
    sp.e_tiles = p.seg ? p.seg->e_tiles : nullptr;
    sp.e_live = p.seg ? p.seg->e_live : nullptr;
    sp.dbg = p.dbg;
    sp.beta = p.beta;
    sp.pro = p.pro;
    sp.s0 = p.initial_state;
    sp.sT = p.final_state;
    sp.ss = p.slots;
    sp.ss.status = status;
    sp.out = static_cast<__nv_bfloat16 *>(p.out);
    sp.status = status;
    sp.filled = flags;
    sp.consumed = flags + heads * RING;
    sp.next_item = flags + heads * (RING + 1);
    sp.ring = ring;
    sp.H = p.H;
    sp.heads = (int32_t)heads;
    sp.max_chunks = max_chunks;
    sp.timeout_ns = timeout_ns;
    void *args[] = {&mq, &mk, &mv, &mla, &sp};
    return cudaLaunchCooperativeKernel(kern, dim3(grid), dim3(NTS), args,
                                       SPLIT_SMEM, stream);
}

}  // namespace kda
