// Split-role chunked prefill for workloads with few (sequence, head) pairs.
//
// The chunk algebra is that of kda_chunk.cu. Its key-side half -- gating, the intra-chunk
// products A and L, T' = (I + L)^-1 diag(beta), W = T' K~ -- does not depend on the state and
// can run for any chunk at any time; only U = T'V - W S, O = Q~ S + A U and the state update
// form the sequential chain. With few heads a fused kernel leaves most SMs idle while each
// head's CTA serialises both halves. Here one persistent cooperative launch fills the GPU:
//
//   consumer CTAs (one per head, or two per head with 64 value channels each when the SMs
//     left over still give every head about three producers): the state chain. Per chunk:
//     [U; O] = [T'; 0] V + [-W; Q~] S (one MMA batch), U to bf16, S += K^^T U and
//     [U; O] += [0; A] U (a second batch), then the outputs and the state's bf16 copy. The fp32
//     state (pre-scaled by gamma while the first batch runs) stays in TMEM for the whole sequence.
//   producer CTAs (all other SMs): the key-side half for chunks ahead, chunk-major order,
//     written as ready-to-use shared-memory images (Q~, K- or K^, W, A, T' tiles, gamma,
//     path flag) into a ring of RING slots per head in the workspace (L2 resident).
//
// Hand-off: a producer fills slot (head, c % RING) with generic stores, then releases
// filled[slot] = c + 1; the consumer acquires it, copies the image into shared memory with a
// bulk copy, and releases consumed[consumer] = c + 1 once the copy has landed; the producer
// acquires both consumers' counters >= c - RING + 1 before reusing the slot. Producer items are
// ordered by chunk, and every producer works through its items in order, so the item a
// consumer waits for never waits on anything later: no cycle. Every spin and mbarrier wait is
// bounded; on timeout the status word is set and the CTA stops. The launch is cooperative,
// so all CTAs are resident together or the launch fails.
#include <cuda.h>

#include <mutex>

#include "kda_chunk_common.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace chunk;

constexpr int RING = 8;
// Chunk image (bytes), the same in a ring slot and in a consumer stage:
//   [0, 8K)      T' [i][j]                     \ with the zero block: [T'; 0] (K-major, 128 rows)
//   [8K, 16K)    zero block (consumer only)     |
//   [16K, 24K)   A [i][j]                      / with the zero block: [0; A] (K-major, 128 rows)
//   [24K, 56K)   [-W; Q~] (K-major, 128 rows, two 64-column blocks of 16 KB: rows 0..63 = -W,
//                rows 64..127 = Q~)
//   [56K, 72K)   K^ [j][c] (an MN-major A operand for K^^T U)
//   [72K, 72K + 512) gamma[128]
constexpr uint32_t SL_T = 0, SL_Z = 8192, SL_A = 16384, SL_WQ = 24576, SL_KH = 57344;
constexpr uint32_t SL_G = 73728, SLOT = 74752;
static_assert(SLOT % 1024 == 0, "slot layout");

struct SplitParams {
    const int32_t *cu_seqlens;
    const float *beta;
    const float *s0;
    float *sT;
    __nv_bfloat16 *out;
    int32_t *status;
    uint8_t *ring;       // [heads][RING][SLOT]
    int32_t *filled;     // [heads][RING]
    int32_t *consumed;   // [heads][2]: one counter per consumer (the second unused with one)
    int32_t H, heads, max_chunks, cph;
    uint64_t timeout_ns;
};

__device__ __forceinline__ int ld_acquire(const int32_t *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int32_t *p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Bounded spin until *p >= target; false on timeout.
__device__ __forceinline__ bool wait_flag_ge(const int32_t *p, int target, uint64_t timeout_ns) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t deadline = globaltimer_ns() + timeout_ns;
    while (true) {
        __nanosleep(100);
        if (ld_acquire(p) >= target) return true;
        if (globaltimer_ns() > deadline) return false;
    }
}
// Bulk (untiled) copy global -> shared, completing on `bar` (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Bulk (untiled) copy shared -> global, tracked by this thread's bulk async-group.
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_u32(src)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until the committed bulk stores have finished reading shared memory / are complete.
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------- consumer (state chain)
// CPH consumers per head, each owning DC = 128 / CPH value channels (columns of S are
// independent: the chain of one column block never reads another's).
template <int CPH>
struct Cons {
    static constexpr int DC = D / CPH;                            // value channels per consumer
    static constexpr int NP = DC / 64;                            // 32-column parts per thread
    static constexpr uint32_t STAGE0 = 0, STAGE1 = SLOT;
    static constexpr uint32_t V0 = 2 * SLOT, V1 = V0 + 128 * DC;  // V [j][d]; after batch 1, U
    static constexpr uint32_t S = V1 + 128 * DC;                  // S [c][d] bf16 128 x DC
    static constexpr uint32_t MISC = S + 256 * DC;                // barriers, flags
    static constexpr uint32_t BYTES = MISC + 256;
    // TMEM: the fp32 state (lane = key channel) and two accumulators D (rows 0..63 = U,
    // rows 64..127 = O; lane = row), used by alternate chunks.
    static constexpr uint32_t TM_S = 0, TM_D0 = DC, TM_D1 = 2 * DC, TM_COLS = CPH == 1 ? 512 : 256;
};

template <int CPH>
__device__ void consumer(const CUtensorMap *tm_v, const SplitParams &p, uint8_t *sm, int cid) {
    using L = Cons<CPH>;
    constexpr int DC = L::DC, NP = L::NP;
    constexpr uint32_t STAGE0 = L::STAGE0, STAGE1 = L::STAGE1, V0 = L::V0, V1 = L::V1, S = L::S;
    constexpr uint32_t MISC = L::MISC, TM_S = L::TM_S, TM_D0 = L::TM_D0, TM_D1 = L::TM_D1;
    constexpr uint32_t TM_COLS = L::TM_COLS;
    constexpr uint32_t I_D = idesc_bf16_f32(128, DC, false, 0, 1);  // [T';0]V + [-W;Q~]S, [0;A]U
    constexpr uint32_t I_S = idesc_bf16_f32(128, DC, false, 1, 1);  // K^^T U
    const int hd = cid / CPH, sub = cid % CPH, d0 = DC * sub;  // head, first value channel
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + MISC);         // in0, in1, u, s, o
    uint32_t *s_flags = reinterpret_cast<uint32_t *>(sm + MISC + 64); // abort, tmem
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const int H = p.H, n = hd / H, h = hd % H;
    const int c_me = 32 * quad + lane;  // TMEM lane of this thread
    const int64_t bos = p.cu_seqlens[n], eos = p.cu_seqlens[n + 1];
    const int nchunks = (int)((eos - bos + C - 1) / C);
    const size_t state_off = ((size_t)n * H + h) * (size_t)(D * D);

    if (tid == 0) {
        s_flags[0] = 0;
        for (int k = 0; k < 5; ++k) mbar_init(&bars[k], 1);
        fence_mbarrier_init();
        prefetch_tmap(tm_v);
    }
    if (warp == 0) {
        tmem_alloc(&s_flags[1], TM_COLS);
        tmem_relinquish();
    }
    for (int e = tid; e < 8192 / 16; e += NT) {  // the zero blocks of both stages
        reinterpret_cast<uint4 *>(sm + STAGE0 + SL_Z)[e] = make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4 *>(sm + STAGE1 + SL_Z)[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_flags[1];

    // Flag thread (lane 31 of warp 5: not the MMA-issuing warp, and it never stores outputs, so
    // its fences and release stores neither stall MMA issue nor wait behind output stores):
    // brings chunk c's image and V into stage c & 1 (block: wait for the producer) and
    // publishes what has been consumed.
    constexpr int FT = 5 * 32 + 31;
    int requested = 0;  // chunks requested so far (flag thread)
    auto request = [&](int c, bool block) -> bool {
        int32_t *fl = p.filled + hd * RING + (c % RING);
        if (block) {
            if (!wait_flag_ge(fl, c + 1, p.timeout_ns)) {
                s_flags[0] = 1;
                atomicOr(p.status, 1);
                return false;
            }
        } else if (ld_acquire(fl) < c + 1) {
            return false;
        }
        fence_proxy_async_global();
        fence_proxy_async_smem();
        const int b = c & 1;
        uint8_t *dst = sm + (b ? STAGE1 : STAGE0);
        const uint8_t *src = p.ring + ((size_t)hd * RING + (c % RING)) * SLOT;
        mbar_arrive_expect_tx(&bars[b], 8192 + (SL_G + 512 - SL_A) + 128 * DC);
        bulk_g2s(dst + SL_T, src + SL_T, 8192, &bars[b]);
        bulk_g2s(dst + SL_A, src + SL_A, SL_G + 512 - SL_A, &bars[b]);
        const int64_t t0 = bos + (int64_t)c * C;
#pragma unroll
        for (int part = 0; part < NP; ++part)
            tma_load_3d(sm + (b ? V1 : V0) + 8192 * part, tm_v, &bars[b], d0 + 64 * part, h, (int32_t)t0);
        requested = c + 1;
        return true;
    };
    // flag thread, non-blocking: request every chunk whose stage is free (the chunk two back has
    // finished all its MMAs: `done` chunks have) and whose image the producer has published
    int done = 0;
    auto poll_ahead = [&]() {
        while (requested < nchunks && requested < done + 2)
            if (!request(requested, false)) break;
    };

    // initial state -> TMEM (lane c, columns d) and its bf16 tile; empty sequences copy it out
    {
        const size_t row = state_off + (size_t)c_me * D + d0 + 32 * NP * half;
        const float *src = p.s0 ? p.s0 + row : nullptr;
        float *dst = p.sT ? p.sT + row : nullptr;
#pragma unroll
        for (int part = 0; part < NP; ++part) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                float4 f = src ? *reinterpret_cast<const float4 *>(src + 32 * part + e)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
                v[e] = f.x; v[e + 1] = f.y; v[e + 2] = f.z; v[e + 3] = f.w;
            }
            if (nchunks == 0) {
                if (dst) {
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4 *>(dst + 32 * part + e) =
                            make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                }
            } else {
                const int col = 32 * NP * half + 32 * part;
                tmem_st32(tmem + lane_base + TM_S + col, v);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    st_chunk(sm + S + tchunk(16384, c_me, col + 8 * q8), v + 8 * q8);
            }
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    uint32_t ph_in[2] = {0, 0}, ph_u = 0, ph_s = 0, ph_o = 0;
    auto wait_bar = [&](uint64_t *bar, uint32_t &ph) {
        const bool ok = mbar_wait_bounded(bar, ph, p.timeout_ns);
        ph ^= 1u;
        if (!ok) {
            s_flags[0] = 1;
            atomicOr(p.status, 1);
        }
    };
    // O of chunk cc: D rows 64..127 (lanes 64..127, quadrants 2 and 3) -> bf16 outputs
    auto store_o = [&](int cc, uint32_t tm_d) {
        const int64_t tc = bos + (int64_t)cc * C;
        const int vc = (int)(eos - tc < C ? eos - tc : C);
        const int i = c_me - 64;
        float v[32];
#pragma unroll
        for (int part = 0; part < NP; ++part) {
            const int col = 32 * NP * half + 32 * part;
            tmem_ld32(tmem + lane_base + tm_d + col, v);
            tmem_wait_ld();
            if (i < vc) {
                uint4 *dst = reinterpret_cast<uint4 *>(p.out + ((size_t)(tc + i) * H + h) * D + d0 + col);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    dst[q8] = make_uint4(pack2(v[8 * q8], v[8 * q8 + 1]), pack2(v[8 * q8 + 2], v[8 * q8 + 3]),
                                         pack2(v[8 * q8 + 4], v[8 * q8 + 5]), pack2(v[8 * q8 + 6], v[8 * q8 + 7]));
            }
        }
    };

    for (int c = 0; c < nchunks; ++c) {
        const int b = c & 1;
        const bool has_next = c + 1 < nchunks;
        const uint32_t tm_d = b ? TM_D1 : TM_D0;
        if (tid == FT && requested <= c) request(c, true);
        __syncthreads();
        if (s_flags[0]) break;
        wait_bar(&bars[b], ph_in[b]);
        uint8_t *stage = sm + (b ? STAGE1 : STAGE0);
        const uint32_t st_base = sb + (b ? STAGE1 : STAGE0);
        const uint32_t vb = sb + (b ? V1 : V0);
        if (tid == FT) {
            fence_proxy_async_global();
            st_release(p.consumed + 2 * hd + sub, c + 1);  // the image is in shared memory: slot reusable
            done = c;  // every MMA of chunk c - 1 was waited on at the end of its iteration
            poll_ahead();  // usually chunk c + 1 into the other stage: a whole chunk to land
        }
        const float *gam = reinterpret_cast<const float *>(stage + SL_G);

        if (tid == 0) {
            tc_fence_after();
            const uint64_t dTZ = desc_k(st_base + SL_T, 16384, 0), dWQ = desc_k(st_base + SL_WQ, 16384, 0);
            const uint64_t dV = desc_mn(vb, 8192, 0), dS = desc_mn(sb + S, 16384, 0);  // one N block
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // [U; O] = [T'; 0] V ...
                mma_bf16_ss(tmem + tm_d, desc_k_at(dTZ, 16384, kk), desc_mn_at(dV, kk), I_D, kk > 0);
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk)  // ... + [-W; Q~] S
                mma_bf16_ss(tmem + tm_d, desc_k_at(dWQ, 16384, kk), desc_mn_at(dS, kk), I_D, 1);
            mma_commit(&bars[2]);
        }
        // While the batch runs (it reads only shared memory and writes D): S <- diag(gamma) S in
        // TMEM ahead of S += K^^T U (warp 4 takes warp 0's columns: warp 0 issues the MMAs), and
        // (rows 64..127) the previous chunk's outputs.
        if (warp == 4)
            scale_tmem_row<DC>(tmem + lane_base + TM_S, gam[c_me]);
        else if (warp != 0)
            scale_tmem_row<DC / 2>(tmem + lane_base + TM_S + (DC / 2) * half, gam[c_me]);
        if (c > 0 && quad >= 2) store_o(c - 1, b ? TM_D0 : TM_D1);
        wait_bar(&bars[2], ph_u);
        tc_fence_after();

        // U (D rows 0..63) -> bf16 [j][d] into this stage's V buffer (V is consumed)
        if (quad < 2) {
#pragma unroll
            for (int part = 0; part < NP; ++part) {
                const int col = 32 * NP * half + 32 * part;
                float v[32];
                tmem_ld32(tmem + lane_base + tm_d + col, v);
                tmem_wait_ld();
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    st_chunk(sm + (b ? V1 : V0) + tchunk(8192, c_me, col + 8 * q8), v + 8 * q8);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;

        if (tid == 0) {
            tc_fence_after();
            const uint64_t dK = desc_mn(st_base + SL_KH, 8192, 0), dU = desc_mn(vb, 8192, 0);
            const uint64_t dAZ = desc_k(st_base + SL_Z, 16384, 0);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // S += K^^T U   (S already scaled by gamma)
                mma_bf16_ss(tmem + TM_S, desc_mn_at(dK, kk), desc_mn_at(dU, kk), I_S, 1);
            mma_commit(&bars[3]);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // [U; O] += [0; A] U
                mma_bf16_ss(tmem + tm_d, desc_k_at(dAZ, 16384, kk), desc_mn_at(dU, kk), I_D, 1);
            mma_commit(&bars[4]);
        }
        wait_bar(&bars[3], ph_s);
        tc_fence_after();

        // the next state's bf16 tile (and the final state after the last chunk)
#pragma unroll
        for (int part = 0; part < NP; ++part) {
            const int col = 32 * NP * half + 32 * part;
            float v[32];
            tmem_ld32(tmem + lane_base + TM_S + col, v);
            tmem_wait_ld();
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
                st_chunk(sm + S + tchunk(16384, c_me, col + 8 * q8), v + 8 * q8);
            if (!has_next && p.sT) {
                float *dst = p.sT + state_off + (size_t)c_me * D + d0 + col;
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(dst + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
            }
        }
        // this chunk's last MMA ([0; A] U): after it, its stage may take chunk c + 2
        wait_bar(&bars[4], ph_o);
        tc_fence_after();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }
    if (nchunks > 0 && !s_flags[0] && quad >= 2)  // outputs of the last chunk
        store_o(nchunks - 1, ((nchunks - 1) & 1) ? TM_D1 : TM_D0);

    // teardown: let requested copies and issued MMAs land before freeing TMEM
    if (s_flags[0] && tid == FT) {
        for (int c = 0; c < 2; ++c)
            if (requested > c) mbar_wait_bounded(&bars[c], ph_in[c], p.timeout_ns);
    }
    if (s_flags[0] && tid == 0) {
        mma_commit(&bars[2]);
        mbar_wait_bounded(&bars[2], ph_u, p.timeout_ns);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

// ---------------------------------------------------------------- producer (key-side half)
namespace prod {
constexpr uint32_t QK0 = 0, QK1 = 32768;       // raw q/k -> Q~/K~ (128-row tiles, 16 KB blocks)
constexpr uint32_t LA0 = 65536, LA1 = 98304;   // raw log_alpha fp32
constexpr uint32_t KI = 131072;                // K- / K^ [j][c] 64 x 128
constexpr uint32_t W = KI + 16384;             // W [i][c] 64 x 128
constexpr uint32_t AQK = W + 16384;            // A [i][j]
constexpr uint32_t TT = AQK + 8192;            // T' [i][j]
constexpr uint32_t LT = TT + 8192;             // L -> T fp32 [64][LT_LD]
constexpr uint32_t PB = LT + 64 * LT_LD * 4;   // 32 x PB_LD fp32
constexpr uint32_t MISC = PB + 32 * PB_LD * 4; // beta, gamma, psum, flags, barriers
constexpr uint32_t KH = (MISC + 64 * 4 + 128 * 4 + 4 * 128 * 4 + 64 + 64 + 1023) / 1024 * 1024;  // K^ [j][c]
constexpr uint32_t BYTES = KH + 16384;
constexpr uint32_t TM_D1 = 0, TM_W = 128, TM_COLS = 256;
}  // namespace prod

__device__ void producer(const CUtensorMap *tm_q, const CUtensorMap *tm_k, const CUtensorMap *tm_la,
                         const SplitParams &p, uint8_t *sm, int pid, int nprod) {
    using namespace prod;
    constexpr uint32_t I_D1 = idesc_bf16_f32(128, 64);
    constexpr uint32_t I_W = idesc_bf16_f32(64, 128, false, 0, 1);
    float *s_beta = reinterpret_cast<float *>(sm + MISC);
    float *s_gamma = s_beta + 64;
    float *s_psum = s_gamma + 128;
    uint32_t *s_flags = reinterpret_cast<uint32_t *>(s_psum + 512);  // abort, tmem
    uint64_t *bars = reinterpret_cast<uint64_t *>(s_flags + 16);     // in0, in1, mma
    float *LTp = reinterpret_cast<float *>(sm + LT);
    float *PBp = reinterpret_cast<float *>(sm + PB);
    const uint32_t sb = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const int H = p.H;
    // Static assignment: producer pid serves head hd = pid % heads, making chunks j, j + cnt, ...
    // (j = pid / heads, cnt = number of producers of that head), so it only ever waits on its
    // own head's consumer.
    const int hd = pid % p.heads, pj = pid / p.heads;
    const int pcnt = (nprod - 1 - hd) / p.heads + 1;
    const int h = hd % H;
    const int64_t bos = p.cu_seqlens[hd / H], eos = p.cu_seqlens[hd / H + 1];
    const int nch = (int)((eos - bos + C - 1) / C);

    if (tid == 0) {
        s_flags[0] = 0;
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init(&bars[2], 1);
        fence_mbarrier_init();
        prefetch_tmap(tm_q);
        prefetch_tmap(tm_k);
        prefetch_tmap(tm_la);
    }
    if (warp == 0) {
        tmem_alloc(&s_flags[1], TM_COLS);
        tmem_relinquish();
    }
    for (int e = tid; e < 8192 / 16; e += NT)  // strictly upper 16x16 blocks of T' stay zero
        reinterpret_cast<uint4 *>(sm + TT)[e] = make_uint4(0u, 0u, 0u, 0u);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_flags[1];

    auto issue_inputs = [&](int c, int b) {  // thread 0
        const int64_t t0 = bos + (int64_t)c * C;
        uint8_t *qk = sm + (b ? QK1 : QK0);
        fence_proxy_async_smem();  // the stage's previous contents were read by generic loads
        mbar_arrive_expect_tx(&bars[b], 32768 + 32768);
        tma_load_3d(qk, tm_q, &bars[b], 0, h, (int32_t)t0);
        tma_load_3d(qk + 8192, tm_k, &bars[b], 0, h, (int32_t)t0);
        tma_load_3d(qk + 16384, tm_q, &bars[b], 64, h, (int32_t)t0);
        tma_load_3d(qk + 24576, tm_k, &bars[b], 64, h, (int32_t)t0);
        tma_load_3d(sm + (b ? LA1 : LA0), tm_la, &bars[b], 0, h, (int32_t)t0);
    };
    auto load_beta = [&](int c) -> float {  // tid < C
        const int64_t t0 = bos + (int64_t)c * C;
        if (c >= nch || t0 + tid >= eos) return 0.f;
        return p.beta[(size_t)(t0 + tid) * H + h];
    };
    // Bulk-store thread (lane 31 of warp 7: not the MMA-issuing thread; warp 7 idles during the
    // first stage of the inverse, where the publish goes): issues an image's bulk stores, waits
    // for them to have read shared memory before the next item rewrites it (just before its
    // gating), and publishes the slot once they are complete (during the next item's inverse).
    constexpr int BT = NT - 1;
    int32_t *rel_flag = nullptr;
    int rel_val = 0;
    auto release = [&]() {
        if (rel_flag) {
            bulk_wait_all();
            fence_proxy_async_global();
            __threadfence();
            st_release(rel_flag, rel_val);
            rel_flag = nullptr;
        }
    };

    uint32_t ph_in[2] = {0, 0}, ph_mma = 0;
    bool pending[2] = {false, false};
    auto wait_bar = [&](uint64_t *bar, uint32_t &ph) {
        const bool ok = mbar_wait_bounded(bar, ph, p.timeout_ns);
        ph ^= 1u;
        if (!ok) {
            s_flags[0] = 1;
            atomicOr(p.status, 1);
        }
    };

    int item = pj;  // chunk index
    if (item < nch) {
        if (tid == 0) issue_inputs(item, 0);
        pending[0] = true;
    }
    float beta_next = (tid < C) ? load_beta(item) : 0.f;
    int b = 0;
    while (item < nch) {
        const int c = item;
        const int64_t t0 = bos + (int64_t)c * C;
        const int valid = (int)(eos - t0 < C ? eos - t0 : C);
        const int nxt = item + pcnt;
        if (tid < C) s_beta[tid] = beta_next;
        wait_bar(&bars[b], ph_in[b]);
        pending[b] = false;

        if (tid < C) beta_next = load_beta(nxt);
        uint8_t *qk = sm + (b ? QK1 : QK0);
        float *la = reinterpret_cast<float *>(sm + (b ? LA1 : LA0));

        if (tid == BT) bulk_wait_read();  // the previous image's sources are rewritten below
        const int gate = gate_chunk(qk, sm + KI, sm + AQK, la, LTp, s_beta, s_gamma, s_psum,
                                    s_flags, valid, tid, sm + KH);
        // The next item's inputs go to the other stage, whose Q~ the previous image's bulk
        // stores read: gate_chunk's barriers come after the bulk-store thread's read wait.
        if (nxt < nch && gate >= 0) {
            if (tid == 0) issue_inputs(nxt, b ^ 1);
            pending[b ^ 1] = true;
        }
        if (gate < 0) break;
        const bool safe = gate == 1;
        fence_proxy_async_smem();
        __syncthreads();

        if (tid == 0) {
            tc_fence_after();
            if (!safe) {
#pragma unroll
                for (uint32_t kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tmem + TM_D1, desc_k(smem_u32(qk), 16384, kk),
                                desc_k(sb + KI, 8192, kk), I_D1, kk > 0);
            }
            mma_commit(&bars[2]);
        }
        wait_bar(&bars[2], ph_mma);
        tc_fence_after();
        if (!safe) extract_al(tmem + lane_base + TM_D1 + 32 * half, sm + AQK, LTp, s_beta, 32 * quad + lane, half);
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;

        if (tid == BT) release();  // the previous item's image (warp 7 idles in the inverse's stage 1)
        invert_unit_lower(LTp, PBp, sm + TT, s_beta, tid);
        fence_proxy_async_smem();
        __syncthreads();

        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // W = T' K~
                mma_bf16_ss(tmem + TM_W, desc_k(sb + TT, 8192, kk),
                            desc_mn(smem_u32(qk) + 8192, 16384, kk), I_W, kk > 0);
            mma_commit(&bars[2]);
        }
        wait_bar(&bars[2], ph_mma);
        tc_fence_after();
        rows64_to_tile<64>(tmem + lane_base + TM_W + 64 * half, sm + W, 8192, 64 * half, quad, lane, -1.f);
        if (tid == BT && c >= RING) {  // the slot's previous chunk must have been taken
            if (!wait_flag_ge(p.consumed + 2 * hd, c - RING + 1, p.timeout_ns) ||
                (p.cph == 2 && !wait_flag_ge(p.consumed + 2 * hd + 1, c - RING + 1, p.timeout_ns))) {
                s_flags[0] = 1;
                atomicOr(p.status, 1);
            }
        }
        fence_proxy_async_smem();  // A, K^, W were written by generic stores; the copy-out is async
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;

        // copy the image out with bulk stores (layout at the top of this file); published at the
        // next item (see release)
        if (tid == BT) {
            uint8_t *slot = p.ring + ((size_t)hd * RING + (c % RING)) * SLOT;
            fence_proxy_async_smem();
            bulk_s2g(slot + SL_T, sm + TT, 8192);
            bulk_s2g(slot + SL_A, sm + AQK, 8192);
            bulk_s2g(slot + SL_WQ, sm + W, 8192);                  // -W, columns 0..63
            bulk_s2g(slot + SL_WQ + 8192, qk, 8192);               // Q~, columns 0..63
            bulk_s2g(slot + SL_WQ + 16384, sm + W + 8192, 8192);   // -W, columns 64..127
            bulk_s2g(slot + SL_WQ + 24576, qk + 16384, 8192);      // Q~, columns 64..127
            bulk_s2g(slot + SL_KH, sm + KH, 16384);
            bulk_s2g(slot + SL_G, s_gamma, 512);
            bulk_commit();
            rel_flag = p.filled + hd * RING + (c % RING);
            rel_val = c + 1;
        }
        __syncthreads();
        item = nxt;
        b ^= 1;
    }

    if (tid == BT && !s_flags[0]) release();
    if (s_flags[0] && tid == BT) bulk_wait_all();
    if (s_flags[0] && tid == 0) {
        for (int k = 0; k < 2; ++k)
            if (pending[k]) mbar_wait_bounded(&bars[k], ph_in[k], p.timeout_ns);
        mma_commit(&bars[2]);
        mbar_wait_bounded(&bars[2], ph_mma, p.timeout_ns);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
    }
}

constexpr uint32_t max3(uint32_t a, uint32_t b, uint32_t c) {
    return a > b ? (a > c ? a : c) : (b > c ? b : c);
}
constexpr uint32_t SPLIT_SMEM = max3(Cons<1>::BYTES, Cons<2>::BYTES, prod::BYTES) + 1024;

template <int CPH>
__global__ void __launch_bounds__(NT, 1)
split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_la,
             const SplitParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    if ((int)blockIdx.x < CPH * p.heads)
        consumer<CPH>(&tm_v, p, sm, blockIdx.x);
    else
        producer(&tm_q, &tm_k, &tm_la, p, sm, blockIdx.x - CPH * p.heads, gridDim.x - CPH * p.heads);
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
                                 cudaStream_t stream, uint64_t timeout_ns) {
    const int64_t heads = (int64_t)p.num_seqs * p.H;
    const int sms = sm_count();
    // Two consumers per head halve the chain's per-chunk work, but take SMs from the producers;
    // worth it only while every head still gets about three producers (a producer's item costs
    // about two and a half consumer chunks).
    const int cph = heads * 5 <= sms ? 2 : 1;
    const void *fn = cph == 2 ? (const void *)split_kernel<2> : (const void *)split_kernel<1>;
    int per_sm = 0;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(split_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)SPLIT_SMEM);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(split_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)SPLIT_SMEM);
    });
    if (attr_err != cudaSuccess) return attr_err;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, NT, SPLIT_SMEM);
    if (e != cudaSuccess) return e;
    const int grid = per_sm * sms;
    if (per_sm < 1 || grid < (cph + 1) * heads) return cudaErrorInvalidConfiguration;

    CUtensorMap mq, mk, mv, mla;
    const uint64_t T = (uint64_t)p.total_tokens, H = (uint64_t)p.H;
    if (!make_token_map(&mq, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_token_map(&mk, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_token_map(&mv, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_token_map(&mla, p.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, H, T, D, false))
        return cudaErrorInvalidValue;

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int32_t *status = reinterpret_cast<int32_t *>(ws);
    int32_t *flags = reinterpret_cast<int32_t *>(ws + 1024);
    const int nflags = (int)(heads * (RING + 2));
    split_init_kernel<<<(nflags + 255) / 256, 256, 0, stream>>>(status, flags, nflags);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    SplitParams sp;
    sp.cu_seqlens = p.cu_seqlens;
    sp.beta = p.beta;
    sp.s0 = p.initial_state;
    sp.sT = p.final_state;
    sp.out = static_cast<__nv_bfloat16 *>(p.out);
    sp.status = status;
    sp.filled = flags;
    sp.consumed = flags + heads * RING;
    sp.ring = ws + 1024 + flags_bytes(heads);
    sp.H = p.H;
    sp.heads = (int32_t)heads;
    sp.max_chunks = max_chunks;
    sp.cph = cph;
    sp.timeout_ns = timeout_ns;
    void *args[] = {&mq, &mk, &mv, &mla, &sp};
    return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(NT), args, SPLIT_SMEM, stream);
}

}  // namespace kda
