// Device building blocks shared by the chunked-prefill kernels (kda_chunk.cu, kda_chunk_split.cu):
// 128-byte-swizzled tile addressing, tcgen05 operand descriptors, bf16 packing, the 64x64 unit
// lower-triangular inverse, the gating of one chunk, and TMEM epilogues. See kda_chunk.cu for the
// chunk algebra these implement.
#pragma once

#include <cuda.h>

#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace chunk {

using namespace sm100;

constexpr int C = 64;    // chunk length
constexpr int D = 128;   // d_k = d_v
constexpr int NT = 256;  // compute threads per CTA
constexpr float kFastLimit = 60.f;  // max in-chunk decay exponent for the factored path

// Barrier over the NTC compute threads (warps 0 .. NTC/32 - 1) only: hardware barrier 1, so a
// CTA may run further warps (a control warp) that never join it.
template <int NTC = NT>
__device__ __forceinline__ void sync_compute() { asm volatile("bar.sync 1, %0;" ::"n"(NTC) : "memory"); }
// The same barrier, returning whether any compute thread passed a non-zero `pred`.
template <int NTC = NT>
__device__ __forceinline__ int sync_compute_or(int pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "n"(NTC)
        : "memory");
    return (int)r;
}

// ---------------------------------------------------------------- global flags between CTAs
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
// Bounded spin until *p >= target (acquire); false once timeout_ns have passed on %globaltimer.
__device__ __forceinline__ bool wait_flag_ge(const int32_t *p, int target, uint64_t timeout_ns) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t deadline = globaltimer_ns() + timeout_ns;
    while (true) {
        __nanosleep(100);
        if (ld_acquire(p) >= target) return true;
        if (globaltimer_ns() > deadline) return false;
    }
}

// ---------------------------------------------------------------- tile addressing
// bf16 tiles use the 128-byte swizzle: 128-byte rows of 64 elements, 8-row groups
// 1024 bytes apart, 16-byte chunk index XOR (row % 8); 64-column blocks `bs` bytes apart.
__device__ __forceinline__ uint32_t tchunk(uint32_t bs, uint32_t row, uint32_t col) {
    return (col >> 6) * bs + (row >> 3) * 1024 + (row & 7) * 128 +
           ((((col & 63) >> 3) ^ (row & 7)) << 4);
}
__device__ __forceinline__ uint32_t telem(uint32_t bs, uint32_t row, uint32_t col) {
    return tchunk(bs, row, col) + ((col & 7) << 1);
}

// Operand descriptors for K step kk (16 elements along K).
// K-major tile (rows = M/N, columns = K): K advances 32 bytes inside a row, K blocks at bs.
__device__ __forceinline__ uint64_t desc_k(uint32_t base, uint32_t bs, uint32_t kk) {
    return smem_desc_sw128(base + (kk >> 2) * bs + (kk & 3) * 32, 16, 1024);
}
// MN-major tile (rows = K, columns = M/N): K advances two 8-row groups, MN blocks at bs.
__device__ __forceinline__ uint64_t desc_mn(uint32_t base, uint32_t bs, uint32_t kk) {
    return smem_desc_sw128(base + kk * 2048, bs, 1024);
}

// The same descriptors from a precomputed step-0 descriptor: only the start-address field
// (address / 16, low 14 bits; shared addresses stay below 256 KB, so no carry) moves.
__device__ __forceinline__ uint64_t desc_k_at(uint64_t d0, uint32_t bs, uint32_t kk) {
    return d0 + (((kk >> 2) * bs + (kk & 3) * 32) >> 4);
}
__device__ __forceinline__ uint64_t desc_mn_at(uint64_t d0, uint32_t kk) { return d0 + kk * 128; }

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ void st_chunk(uint8_t *p, const float *v) {
    *reinterpret_cast<uint4 *>(p) = make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]),
                                               pack2(v[4], v[5]), pack2(v[6], v[7]));
}
__device__ __forceinline__ float2 ld_bf2(const uint8_t *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
__device__ __forceinline__ void st_bf2(uint8_t *p, float a, float b) {
    *reinterpret_cast<uint32_t *>(p) = pack2(a, b);
}
__device__ __forceinline__ float ld_bf(const uint8_t *p) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
}
__device__ __forceinline__ void st_bf(uint8_t *p, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(p) = __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------- 64x64 unit lower-triangular inverse
constexpr int LT_LD = 68;  // fp32 pitch of the L / T scratch
constexpr int PB_LD = 36;  // fp32 pitch of the 32x32 block-product scratch

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// acc (a 16x16 tile as two m16n8 fragments) += A[16][K] * B[K][16], fp32 in shared memory,
// multiplied with tf32 operands by the warp-level mma.sync m16n8k8.
__device__ __forceinline__ void warp_mm16(float (&acc)[2][4], const float *A, int pa,
                                          const float *B, int pb, int K) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    for (int k = 0; k < K; k += 8) {
        const uint32_t a0 = to_tf32(A[gid * pa + k + tig]);
        const uint32_t a1 = to_tf32(A[(gid + 8) * pa + k + tig]);
        const uint32_t a2 = to_tf32(A[gid * pa + k + tig + 4]);
        const uint32_t a3 = to_tf32(A[(gid + 8) * pa + k + tig + 4]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = to_tf32(B[(k + tig) * pb + 8 * nt + gid]);
            const uint32_t b1 = to_tf32(B[(k + tig + 4) * pb + 8 * nt + gid]);
            asm volatile(
                "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, "
                "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                : "+f"(acc[nt][0]), "+f"(acc[nt][1]), "+f"(acc[nt][2]), "+f"(acc[nt][3])
                : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        }
    }
}
__device__ __forceinline__ void warp_store16(float *X, int px, const float (&acc)[2][4], float s) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        X[gid * px + 8 * nt + 2 * tig] = s * acc[nt][0];
        X[gid * px + 8 * nt + 2 * tig + 1] = s * acc[nt][1];
        X[(gid + 8) * px + 8 * nt + 2 * tig] = s * acc[nt][2];
        X[(gid + 8) * px + 8 * nt + 2 * tig + 1] = s * acc[nt][3];
    }
}

// Column `col` of (I + L)^-1 for one 16x16 diagonal block (L strictly lower, fp32 rows LT_LD
// apart from Lb, which is 16-byte aligned) by forward substitution in row order:
// x_i = [i == col] - sum_{j<i} L_ij x_j. Each row's values come in as 16-byte broadcast loads
// (36 for the block), and every row sum runs as two interleaved partial sums.
__device__ __forceinline__ void unit_lower16_column(const float *Lb, int col, float (&x)[16]) {
    x[0] = (col == 0) ? 1.f : 0.f;
#pragma unroll
    for (int i = 1; i < 16; ++i) {
        float s0 = (col == i) ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
        for (int j4 = 0; 4 * j4 < i; ++j4) {
            const float4 l = *reinterpret_cast<const float4 *>(Lb + i * LT_LD + 4 * j4);
            const int j = 4 * j4;
            s0 = fmaf(-l.x, x[j], s0);
            if (j + 1 < i) s1 = fmaf(-l.y, x[j + 1], s1);
            if (j + 2 < i) s0 = fmaf(-l.z, x[j + 2], s0);
            if (j + 3 < i) s1 = fmaf(-l.w, x[j + 3], s1);
        }
        x[i] = s0 + s1;
    }
}

// Writes rows of a 16x16 fragment tile as bf16 T' = T diag(beta) into the TT tile at (r0, c0).
__device__ __forceinline__ void frag_to_tt(uint8_t *TT, int r0, int c0, const float (&acc)[2][4],
                                           float s, const float *beta) {
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int c = c0 + 8 * nt + 2 * tig;
        const float b0 = s * beta[c], b1 = s * beta[c + 1];
        st_bf2(TT + telem(8192, r0 + gid, c), acc[nt][0] * b0, acc[nt][1] * b1);
        st_bf2(TT + telem(8192, r0 + gid + 8, c), acc[nt][2] * b0, acc[nt][3] * b1);
    }
}

// T = (I + L)^-1 for strictly lower-triangular L (fp32 in LT, pitch LT_LD, zeros on and
// above the diagonal), written as bf16 T' = T diag(beta) into the lower blocks of TT (its
// strictly upper 16x16 blocks must already be zero). Blocks of 16: the diagonal blocks by
// forward substitution, then the block inverse [[A,0],[B,C]]^-1 = [[A^-1,0],[-C^-1 B A^-1,
// C^-1]] at 16 and then at 32, on the tensor cores (tf32 mma.sync). LT keeps the fp32 blocks
// later stages need. Called by the NT compute threads (synchronised among themselves with
// sync_compute); ends with the TT stores issued (no barrier).
// `warp` is the caller's logical warp index for the inverse: 0..3 do its work, any other value
// (e.g. -1 for a warp that does other work meanwhile) only joins its barriers.
template <int NTC = NT>
static __device__ __forceinline__ void invert_unit_lower(float *LT, float *PB, uint8_t *TT, const float *beta,
                                                         int tid, int warp) {
    const int lane = tid & 31;
    if (warp >= 0 && warp < 4 && lane < 16) {
        const int b0 = 16 * warp;
        float x[16];
        unit_lower16_column(LT + b0 * LT_LD + b0, lane, x);
        __syncwarp(0x0000ffffu);
        float *Tb = LT + b0 * LT_LD + b0;
        const float bl = beta[b0 + lane];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            Tb[i * LT_LD + lane] = x[i];
            st_bf(TT + telem(8192, b0 + i, b0 + lane), x[i] * bl);
        }
    }
    sync_compute<NTC>();
    if (warp >= 0 && warp < 2) {
        // warp 0: T10 = -T11 (L10 T00); warp 1: T32 = -T33 (L32 T22)
        const int r0 = warp ? 48 : 16, c0 = warp ? 32 : 0;
        float *P = PB + warp * 16 * PB_LD;
        float acc[2][4] = {};
        warp_mm16(acc, LT + r0 * LT_LD + c0, LT_LD, LT + c0 * LT_LD + c0, LT_LD, 16);
        warp_store16(P, PB_LD, acc, 1.f);
        __syncwarp();
        float acc2[2][4] = {};
        warp_mm16(acc2, LT + r0 * LT_LD + r0, LT_LD, P, PB_LD, 16);
        warp_store16(LT + r0 * LT_LD + c0, LT_LD, acc2, -1.f);
        frag_to_tt(TT, r0, c0, acc2, -1.f, beta);
    }
    sync_compute<NTC>();
    // rows 32..63 x cols 0..31: P = L[32:64, 0:32] T[0:32, 0:32];  T[32:64, 0:32] = -T[32:64, 32:64] P
    const int rt = (warp >> 1) & 1, ct = warp & 1;
    if (warp >= 0 && warp < 4) {
        float acc[2][4] = {};
        warp_mm16(acc, LT + (32 + 16 * rt) * LT_LD, LT_LD, LT + 16 * ct, LT_LD, 32);
        warp_store16(PB + (16 * rt) * PB_LD + 16 * ct, PB_LD, acc, 1.f);
    }
    sync_compute<NTC>();
    if (warp >= 0 && warp < 4) {
        float acc[2][4] = {};
        warp_mm16(acc, LT + (32 + 16 * rt) * LT_LD + 32, LT_LD, PB + 16 * ct, PB_LD, 32);
        frag_to_tt(TT, 32 + 16 * rt, 16 * ct, acc, -1.f, beta);
    }
}


// ---------------------------------------------------------------- the same inverse on tcgen05
// With D = I + (the 16x16 diagonal blocks of L) and L_off = L outside those blocks,
// I + L = D (I + N) with N = D^-1 L_off. N's blocks lie strictly below the block diagonal, so
// N^4 = 0 and (I + N)^-1 = (I + N^2)(I - N):
//   T = (I + L)^-1 = (I + N^2)(I - N) D^-1,
// three rounds of dependent bf16 MMAs with fp32 accumulation, which the caller issues:
//   [N | D^-1] = D^-1 [L_off | I];   W1 = D^-1 - N D^-1 (onto D^-1, A negated), N2 = N N;
//   T = W1 + N2 W1 (onto W1).
// Every operand is a 64x64 bf16 tile in the natural row layout (tchunk, one 64-column block),
// which is both a K-major A operand and an MN-major B operand. Rounding: D^-1, L_off, N, N2 and
// W1 are rounded to bf16 once each as operands (the accumulators stay fp32); T' = T diag(beta)
// is rounded to bf16 anyway for the MMAs that use it, and that rounding dominates (checked
// against the mma.sync tf32 merges above).

// Step 0, before the first MMA: D^-1 into t_dinv (the four diagonal blocks by forward
// substitution, lanes 0..15 of logical warps 0..3; the other blocks zero), L_off into t_loff and
// the identity into t_eye. Called by the NTC compute threads; ends with the tile stores issued
// (no barrier).
template <int NTC = NT>
static __device__ __forceinline__ void inv_tc_setup(const float *LT, uint8_t *t_dinv, uint8_t *t_loff,
                                                    int tid, int warp, uint8_t *t_eye) {
    static_assert(NTC > 128, "the tile writers are the warps after the first four");
    const int lane = tid & 31;
    if (warp >= 0 && warp < 4) {
        if (lane < 16) {
            const int b0 = 16 * warp;
            float x[16];  // column `lane` of the block's inverse
            unit_lower16_column(LT + b0 * LT_LD + b0, lane, x);
#pragma unroll
            for (int i = 0; i < 16; ++i) st_bf(t_dinv + telem(8192, b0 + i, b0 + lane), x[i]);
        }
        return;
    }
    // 16-byte chunks (8 columns, inside one 16-column block): L_off everywhere, zeros of D^-1
    // outside the diagonal blocks (the forward substitution writes those chunks)
    const float zero[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int q = tid - 128; q < 512; q += NTC - 128) {
        const int r = q >> 3, c0 = (q & 7) * 8;
        if ((r >> 4) == (c0 >> 4)) {
            st_chunk(t_loff + tchunk(8192, r, c0), zero);
        } else {
            const float4 a = *reinterpret_cast<const float4 *>(LT + r * LT_LD + c0);
            const float4 b = *reinterpret_cast<const float4 *>(LT + r * LT_LD + c0 + 4);
            const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            st_chunk(t_loff + tchunk(8192, r, c0), v);
            st_chunk(t_dinv + tchunk(8192, r, c0), zero);
        }
        float e[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) e[x] = (c0 + x == r) ? 1.f : 0.f;
        st_chunk(t_eye + tchunk(8192, r, c0), e);
    }
}

// 16 columns col0.. of an M=64 accumulator (row 16 quad + lane in lanes 0..15 of each quadrant;
// taddr includes the warp's lane base) -> the same rows and columns of a 64x64 bf16 tile, as
// op(row, col, value).
template <typename Op>
__device__ __forceinline__ void acc64_cols16_to_tile(uint32_t taddr, uint8_t *tile, int col0, int quad,
                                                     int lane, Op op) {
    float v[16];
    tmem_ld16(taddr + (uint32_t)col0, v);
    tmem_wait_ld();
    if (lane < 16) {
        const int row = 16 * quad + lane;
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = op(row, col0 + e, v[e]);
        st_chunk(tile + tchunk(8192, row, col0), v);
        st_chunk(tile + tchunk(8192, row, col0 + 8), v + 8);
    }
}

// ---------------------------------------------------------------- gating of one chunk
// The NTC compute threads (synchronised among themselves with sync_compute<NTC>). In: QK holds
// raw q (rows 0..63) and k (rows 64..127) as a K-major tile with 16 KB blocks, LA the chunk's raw
// log_alpha [t][c] fp32, s_beta the chunk's beta (0 past `valid`).
// Out: QK holds Q~ and K~ in place, KI holds K- (factored path) or K^ (exact path), s_gamma =
// e^(g_{C-1}); the exact path also writes A into AQK and beta-scaled L into LT (zeros elsewhere).
// Thread mapping: channels 4 lane .. 4 lane + 3 of the TPG = C / (NTC / 32) tokens of group
// `warp` (tokens TPG warp .. TPG warp + TPG - 1); s_psum holds [NTC / 32 + 1][D] floats (the
// groups' totals, turned in place into exclusive prefixes by a scan, plus the chunk totals).
// If KH is not null it also receives K^ = k e^(g_{C-1} - g) on both paths. If src_free is not
// null, the writes to KI, KH and AQK first wait (bounded by timeout_ns) for that mbarrier's
// phase with parity src_parity, and then for src_free2's phase with parity src_parity2 if that
// is not null: other threads or the tensor core may still be reading those tiles.
// Returns 1 for the exact path, 0 for the factored path, -1 if the wait timed out (which sets
// *s_abort). Every compute thread passes every barrier inside (the path is decided by a barrier
// reduction, and a failed wait only sets a flag), so no thread is left waiting at one.
// PRO: the prologue (raw q, k rows and raw gates, per pro.flags) is compiled in; without it the
// function is the plain gating.
// SCRATCH: only the exact path waits for src_free (it writes AQK and LT); the factored path
// writes nothing but QK, KI (K-) and KH (K^), so KI and KH may be scratch regions outside the
// previous image (KH may be LA itself: it is written after the last read of LA). On the exact
// path KI is not written at all (its D1 is never issued).
template <bool PRO = false, int NTC = NT, bool SCRATCH = false>
__device__ __forceinline__ int gate_chunk(uint8_t *QK, uint8_t *KI, uint8_t *AQK, float *LA,
                                          float *LT, const float *s_beta, float *s_gamma,
                                          float *s_psum, uint32_t *s_abort, int valid,
                                          int tid, uint8_t *KH = nullptr,
                                          uint64_t *src_free = nullptr, uint32_t src_parity = 0,
                                          uint64_t timeout_ns = 0, const Prologue pro = Prologue(),
                                          uint64_t *src_free2 = nullptr, uint32_t src_parity2 = 0) {
    constexpr int G = NTC / 32, TPG = C / G;  // token groups (one per warp), tokens per group
    static_assert(G * TPG == C && TPG >= 1 && TPG <= 8, "gating thread mapping");
    const int warp = tid >> 5, lane = tid & 31;
    const int to = warp, c4 = 4 * lane;  // group `to`: tokens TPG to .. + TPG - 1; channels c4 .. c4 + 3
    const uint32_t cx = (uint32_t)(c4 & 63) >> 3;
    // Byte offset of token row t, channels c4 .. c4 + 3, in a 128-byte-swizzled tile (64-column
    // blocks `bs` bytes apart): telem(bs, t, c4) with the block term left to the caller.
    auto row_off = [&](int t) {
        return (uint32_t)(t >> 3) * 1024 + (uint32_t)(t & 7) * 128 + ((cx ^ (uint32_t)(t & 7)) << 4) +
               (uint32_t)(c4 & 7) * 2;
    };
    if (PRO && (pro.flags & KDA_PROLOGUE_QK_L2NORM)) {
        // Raw q and k rows -> x / sqrt(x.x + eps), in place. A warp holds its tokens' whole rows
        // (lane: 4 channels), addressed as in the operand loop below.
        uint8_t *const q0 = QK + (uint32_t)(c4 >> 6) * 16384;
        auto widen = [](uint32_t u) { return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u)); };
#pragma unroll
        for (int i = 0; i < TPG; ++i) {
            const int t = TPG * to + i;
            if (t >= valid) break;  // the same for the whole warp
            uint2 *qp = reinterpret_cast<uint2 *>(q0 + row_off(t));
            uint2 *kp = reinterpret_cast<uint2 *>(q0 + 8192 + row_off(t));
            const uint2 qu = *qp, ku = *kp;
            const float2 qa = widen(qu.x), qb = widen(qu.y), ka = widen(ku.x), kb = widen(ku.y);
            float sq = qa.x * qa.x + qa.y * qa.y + qb.x * qb.x + qb.y * qb.y;
            float sk = ka.x * ka.x + ka.y * ka.y + kb.x * kb.x + kb.y * kb.y;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
            }
            const float rq = rsqrtf(sq + kL2NormEps), rk = rsqrtf(sk + kL2NormEps);
            *qp = make_uint2(pack2(qa.x * rq, qa.y * rq), pack2(qb.x * rq, qb.y * rq));
            *kp = make_uint2(pack2(ka.x * rk, ka.y * rk), pack2(kb.x * rk, kb.y * rk));
        }
    }
    // ---- gates: log_alpha of TPG tokens x 4 channels into registers, group totals
    float4 la[TPG];
    float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < TPG; ++i) {
        const int t = TPG * to + i;
        la[i] = (t < valid) ? *reinterpret_cast<const float4 *>(LA + t * D + c4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        if (PRO && (pro.flags & KDA_PROLOGUE_GATE_SOFTPLUS) && t < valid) {
            const float sc = pro.gate_scale;
            la[i] = make_float4(gate_from_raw(la[i].x, sc), gate_from_raw(la[i].y, sc),
                                gate_from_raw(la[i].z, sc), gate_from_raw(la[i].w, sc));
        }
        tot.x += la[i].x;
        tot.y += la[i].y;
        tot.z += la[i].z;
        tot.w += la[i].w;
    }
    *reinterpret_cast<float4 *>(s_psum + to * D + c4) = tot;
    // A group decaying by more than e^(kFastLimit/G) in some channel sends the chunk down the
    // exact path; otherwise the whole chunk decays by at most e^kFastLimit.
    // (NaN gates also take the exact path: the comparisons are false for NaN.)
    const float lim = kFastLimit / (float)G;
    const int unsafe = !(-tot.x <= lim) || !(-tot.y <= lim) || !(-tot.z <= lim) || !(-tot.w <= lim);
    const bool safe = sync_compute_or<NTC>(unsafe) != 0;
    bool failed = false;
    // Per channel, the groups' totals -> exclusive prefixes (in place) and the chunk total (row
    // G), by one thread per channel: each thread then reads two values instead of all G rows.
    if (tid < D) {
        float run = 0.f;
#pragma unroll
        for (int o = 0; o < G; ++o) {
            const float a = s_psum[o * D + tid];
            s_psum[o * D + tid] = run;
            run += a;
        }
        s_psum[G * D + tid] = run;
        s_gamma[tid] = __expf(run);
    }
    if (src_free && (!SCRATCH || safe) &&
        (!mbar_wait_bounded(src_free, src_parity, timeout_ns) ||
         (src_free2 && !mbar_wait_bounded(src_free2, src_parity2, timeout_ns)))) {
        *s_abort = 1;
        failed = true;  // the writes below go on (shared memory only); the caller stops
    }
    sync_compute<NTC>();
    const float4 goff = *reinterpret_cast<const float4 *>(s_psum + to * D + c4);
    const float4 gC = *reinterpret_cast<const float4 *>(s_psum + G * D + c4);

    if (safe) {
        // Exact path: A and L pairwise from raw q, k and the full g (no factored exponentials).
        {
            float4 g = goff;
#pragma unroll
            for (int i = 0; i < TPG; ++i) {
                g.x += la[i].x;
                g.y += la[i].y;
                g.z += la[i].z;
                g.w += la[i].w;
                *reinterpret_cast<float4 *>(LA + (TPG * to + i) * D + c4) = g;
            }
        }
        for (int e = tid; e < 64 * 64; e += NTC) {
            const int i = e >> 6, j = e & 63;
            st_bf(AQK + telem(8192, i, j), 0.f);
            LT[i * LT_LD + j] = 0.f;
        }
        sync_compute<NTC>();
        for (int e = warp; e < 64 * 64; e += NTC / 32) {
            const int i = e >> 6, j = e & 63;
            if (j > i || i >= valid) continue;
            float a = 0.f, l = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int cc = lane + 32 * m;
                const float ex = __expf(LA[i * D + cc] - LA[j * D + cc]);
                const float kj = ld_bf(QK + telem(16384, 64 + j, cc)) * ex;
                a = fmaf(ld_bf(QK + telem(16384, i, cc)), kj, a);
                l = fmaf(ld_bf(QK + telem(16384, 64 + i, cc)), kj, l);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                a += __shfl_xor_sync(0xffffffffu, a, off);
                l += __shfl_xor_sync(0xffffffffu, l, off);
            }
            if (lane == 0) {
                st_bf(AQK + telem(8192, i, j), a);
                if (j < i) LT[i * LT_LD + j] = s_beta[i] * l;
            }
        }
        sync_compute<NTC>();  // raw q, k are read above and overwritten below
    }

    // ---- gated operands. With alpha = e^log_alpha, prefix products P_i and suffix
    // products R_i (within the group): e^g_i = e^goff P_i; e^-g_i = e^(-goff-tot) R_i;
    // e^(g_C - g_i) = e^(g_C-goff-tot) R_i. Q~, K~ overwrite q, k in place; the KI tile
    // gets K- (fast path) or K^ (exact path).
    {
        float4 al[TPG];
#pragma unroll
        for (int i = 0; i < TPG; ++i)
            al[i] = make_float4(__expf(la[i].x), __expf(la[i].y), __expf(la[i].z), __expf(la[i].w));
        const float4 eA = make_float4(__expf(goff.x), __expf(goff.y), __expf(goff.z), __expf(goff.w));
        // e^(g_C - goff - tot) and e^(-goff - tot): on the factored path the first is the second
        // times gamma (the scan's e^(g_C)); the exact path needs only the first, which cannot
        // overflow, and uses it for both.
        float4 eH, eB;
        if (safe) {
            eH = make_float4(__expf(gC.x - goff.x - tot.x), __expf(gC.y - goff.y - tot.y),
                             __expf(gC.z - goff.z - tot.z), __expf(gC.w - goff.w - tot.w));
            eB = eH;
        } else {
            eB = make_float4(__expf(-goff.x - tot.x), __expf(-goff.y - tot.y), __expf(-goff.z - tot.z),
                             __expf(-goff.w - tot.w));
            const float4 gm = *reinterpret_cast<const float4 *>(s_gamma + c4);
            eH = make_float4(eB.x * gm.x, eB.y * gm.y, eB.z * gm.z, eB.w * gm.w);
        }
        float4 R[TPG];
        float4 run = make_float4(1.f, 1.f, 1.f, 1.f);
#pragma unroll
        for (int i = TPG - 1; i >= 0; --i) {
            R[i] = run;
            run.x *= al[i].x;
            run.y *= al[i].y;
            run.z *= al[i].z;
            run.w *= al[i].w;
        }
        // K~ rows (64 + t) sit 8 row groups (8 KB) after the Q~ rows. Four channels = one 8-byte
        // access.
        uint8_t *const q0 = QK + (uint32_t)(c4 >> 6) * 16384;
        uint8_t *const i0 = KI + (uint32_t)(c4 >> 6) * 8192;
        uint8_t *const h0 = KH ? KH + (uint32_t)(c4 >> 6) * 8192 : nullptr;
        auto unpack4 = [](uint2 u) {
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
            const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
            return make_float4(a.x, a.y, b.x, b.y);
        };
        auto pack4 = [](float a, float b, float c, float d) { return make_uint2(pack2(a, b), pack2(c, d)); };
        // all of this thread's q and k first: each element is rewritten in place by the thread
        // that reads it, so no load has to wait behind a store
        uint2 qraw[TPG], kraw[TPG];
#pragma unroll
        for (int i = 0; i < TPG; ++i) {
            const uint32_t off = row_off(TPG * to + i);
            qraw[i] = *reinterpret_cast<const uint2 *>(q0 + off);
            kraw[i] = *reinterpret_cast<const uint2 *>(q0 + 8192 + off);
        }
        float4 P = eA;
#pragma unroll
        for (int i = 0; i < TPG; ++i) {
            const int t = TPG * to + i;
            P.x *= al[i].x;
            P.y *= al[i].y;
            P.z *= al[i].z;
            P.w *= al[i].w;
            const uint32_t off = row_off(t);
            uint2 *qp = reinterpret_cast<uint2 *>(q0 + off);
            uint2 *kp = reinterpret_cast<uint2 *>(q0 + 8192 + off);
            float4 qv = unpack4(qraw[i]), kv = unpack4(kraw[i]);
            if (t >= valid) qv = kv = make_float4(0.f, 0.f, 0.f, 0.f);
            *qp = pack4(qv.x * P.x, qv.y * P.y, qv.z * P.z, qv.w * P.w);
            *kp = pack4(kv.x * P.x, kv.y * P.y, kv.z * P.z, kv.w * P.w);
            const float4 kr = make_float4(kv.x * R[i].x, kv.y * R[i].y, kv.z * R[i].z, kv.w * R[i].w);
            if (!SCRATCH || !safe)
                *reinterpret_cast<uint2 *>(i0 + off) = pack4(kr.x * eB.x, kr.y * eB.y, kr.z * eB.z, kr.w * eB.w);
            if (KH)
                *reinterpret_cast<uint2 *>(h0 + off) = pack4(kr.x * eH.x, kr.y * eH.y, kr.z * eH.z, kr.w * eH.w);
        }
    }
    return failed ? -1 : (safe ? 1 : 0);
}

// ---------------------------------------------------------------- TMEM epilogues
// D1 (M=128: rows 0..63 = Q~ K-^T, rows 64..127 = K~ K-^T) -> A (bf16, j <= i) into AQK and
// L (fp32, times beta_i, j < i) into LT. Thread: TMEM lane r, NC columns from col0 (taddr points
// at column col0 of D1).
template <int NC = 32>
__device__ __forceinline__ void extract_al(uint32_t taddr, uint8_t *AQK, float *LT,
                                           const float *s_beta, int r, int col0) {
    static_assert(NC == 16 || NC == 32, "extract_al columns");
    float v[NC];
    if constexpr (NC == 32) {
        tmem_ld32(taddr, v);
    } else {
        tmem_ld16(taddr, v);
    }
    tmem_wait_ld();
    if (r < 64) {
#pragma unroll
        for (int e = 0; e < NC; ++e) v[e] = (col0 + e <= r) ? v[e] : 0.f;
#pragma unroll
        for (int q8 = 0; q8 < NC / 8; ++q8)
            st_chunk(AQK + tchunk(8192, r, col0 + 8 * q8), v + 8 * q8);
    } else {
        const int i = r - 64;
        const float b = s_beta[i];
        float4 *dst = reinterpret_cast<float4 *>(LT + i * LT_LD + col0);
#pragma unroll
        for (int e4 = 0; e4 < NC / 4; ++e4) {
            const int j = col0 + 4 * e4;
            dst[e4] = make_float4(j + 0 < i ? b * v[4 * e4 + 0] : 0.f,
                                  j + 1 < i ? b * v[4 * e4 + 1] : 0.f,
                                  j + 2 < i ? b * v[4 * e4 + 2] : 0.f,
                                  j + 3 < i ? b * v[4 * e4 + 3] : 0.f);
        }
    }
}

// An M=64 accumulator (row 16*quad + lane in lanes 0..15 of each quadrant) -> bf16 tile rows,
// NCOLS columns starting at column col0 of both the TMEM region (taddr) and the tile.
template <int NCOLS>
__device__ __forceinline__ void rows64_to_tile(uint32_t taddr, uint8_t *tile, uint32_t bs,
                                               int col0, int quad, int lane, float scale = 1.f) {
    float vv[NCOLS / 32][32];  // every 32-column load in flight before one wait
#pragma unroll
    for (int part = 0; part < NCOLS / 32; ++part) tmem_ld32(taddr + 32 * part, vv[part]);
    tmem_wait_ld();
#pragma unroll
    for (int part = 0; part < NCOLS / 32; ++part) {
        float *v = vv[part];
        if (scale != 1.f) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= scale;
        }
        if (lane < 16) {
            const int row = 16 * quad + lane;
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
                st_chunk(tile + tchunk(bs, row, col0 + 32 * part + 8 * q8), v + 8 * q8);
        }
    }
}

// S <- diag(gamma) S in TMEM for this thread's lane (gamma) and NCOLS columns at taddr.
template <int NCOLS>
__device__ __forceinline__ void scale_tmem_row(uint32_t taddr, float gm) {
#pragma unroll
    for (int part = 0; part < NCOLS / 32; ++part) {
        float v[32];
        tmem_ld32(taddr + 32 * part, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= gm;
        tmem_st32(taddr + 32 * part, v);
    }
    tmem_wait_st();
}

}  // namespace chunk

// 3-D TMA map over [T][H][inner] with a box of (box_inner, 1, 64 tokens); false on failure.
bool make_token_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint32_t esize,
                    uint64_t inner, uint64_t H, uint64_t T, uint32_t box_inner, bool swizzle);

}  // namespace kda
