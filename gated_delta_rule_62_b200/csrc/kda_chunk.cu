// Chunked KDA prefill on tcgen05 tensor cores (bf16 operands, fp32 accumulators in TMEM).
//
// The KDA update is computed over blocks of tokens so that it runs on the GPU's matrix
// units (shivam2003.com Kimi K3 article, section "Kimi Delta Attention: the
// load-bearing choice"). The blockwise form is derived from the per-token
// recurrence (channel-wise decay, delta-rule write of the error, read after
// the write). For a chunk of C = 64 tokens entered with state S (d_k x d_v),
// g_i = sum_{s<=i} log_alpha_s (inclusive, per key channel), gamma = e^(g_{C-1}):
//
//   Q~ = q*e^g,  K~ = k*e^g,  K- = k*e^-g                       (rows = tokens)
//   A  = tril(Q~ K-^T)          (j <= i)
//   L  = diag(beta) strictly_tril(K~ K-^T),   T' = (I + L)^-1 diag(beta)
//   W  = T' K~,   U~ = T' V,    U = U~ - W S           (the errors the delta rule writes)
//   O  = Q~ S + A U
//   S_next = diag(gamma) (S + K-^T U)
//
// the WY/UT form of the product of the per-token transitions (I - beta k k^T) Diag(alpha).
// Tokens are the M dimension of the token-row products (M = 64); the state update
// has M = 128 key channels. K~, V, U and S enter the MMAs as MN-major operands
// straight from the tiles TMA or the epilogues write, so no tile is transposed.
// The fp32 master state S stays in TMEM for the whole sequence (lane = key channel).
//
// Factoring e^(g_i - g_j) = e^(g_i) e^(-g_j) overflows when a chunk decays by more
// than ~e^88 in some channel. A chunk whose decay exceeds e^60 in any channel takes
// an exact path: A and L are formed pairwise on CUDA cores, the K- tile holds
// K^ = k e^(g_{C-1} - g), and S is scaled by gamma before S += K^^T U.
//
// One CTA of 256 threads per (sequence, head, d_v slice); DS = 128 / NSPLIT value
// channels per CTA (NSPLIT = 2 doubles the CTAs for workloads with few heads, at the
// price of repeating the key-side work). Every on-device wait is bounded; on timeout
// the kernel records KDA_ERR_TIMEOUT in the workspace status word and returns.
// (Sixteen warps, a quarter of each phase per warp as in the split kernel's producers, were
// measured slower here: 8.64 against 8.07-8.38 ms on the varlen workload, same box.)
#include <cuda.h>

#include <mutex>

#include "kda_chunk_common.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace chunk;

// ---------------------------------------------------------------- shared memory map
template <int DS>
struct Smem {
    static constexpr uint32_t QK = 0;                       // [q~ ; k~] 128 rows x 128, blocks 16 KB
    static constexpr uint32_t KI = QK + 32768;              // K- (or K^) [j][c] 64 x 128, blocks 8 KB
    static constexpr uint32_t W = KI + 16384;               // W [i][c] 64 x 128, blocks 8 KB
    static constexpr uint32_t S = W + 16384;                // S [c][d] bf16 128 x DS, blocks 16 KB
    static constexpr uint32_t V = S + 256 * DS;             // V [j][d] 64 x DS, blocks 8 KB
    static constexpr uint32_t U = V + 128 * DS;             // U [j][d] 64 x DS, blocks 8 KB
    static constexpr uint32_t AQK = U + 128 * DS;           // A [i][j] 64 x 64
    static constexpr uint32_t TT = AQK + 8192;              // T' [i][j] 64 x 64
    static constexpr uint32_t LA = TT + 8192;               // log_alpha [t][c] fp32, then g
    static constexpr uint32_t LT = LA + 32768;              // L -> T fp32 [64][LT_LD]
    static constexpr uint32_t PB = LT + 64 * LT_LD * 4;     // 32 x PB_LD fp32
    static constexpr uint32_t MISC = PB + 32 * PB_LD * 4;   // beta, gamma, psum, flags, barriers
    static constexpr uint32_t MISC_BYTES = 64 * 4 + 128 * 4 + 9 * 128 * 4 + 64 + 64;
    static constexpr uint32_t BYTES = MISC + MISC_BYTES + 1024;  // + alignment slack
};

// TMEM columns (fp32, 128 lanes). DS <= 64: O has its own columns; DS = 128: O takes D1's
// columns and the 64 after them, free once A and L are out of D1, so O = Q~ S runs during the
// inverse.
template <int DS>
struct Tmem {
    static constexpr uint32_t S = 0;
    static constexpr uint32_t U = DS <= 64 ? 192 : 128;
    static constexpr uint32_t W = U + DS;
    static constexpr uint32_t D1 = DS <= 64 ? 128 : W + 128;
    static constexpr uint32_t O = DS <= 64 ? W + 128 : D1;
    static constexpr uint32_t COLS = 512;
    static_assert(O + DS <= COLS && W + 128 <= COLS, "TMEM overflow");
};

struct ChunkParams {
    const int32_t *cu_seqlens;
    const int32_t *order;  // sequences, longest first
    const float *beta;
    Prologue pro;
    const float *s0;  // initial states, or the state pool
    float *sT;        // final states, or the state pool
    __nv_bfloat16 *out;
    int32_t *status;
    int32_t H;
    uint64_t timeout_ns;
    StateSlots ss;
    DebugRanges dbg;  // buffer ranges (checked by debug builds only)
};

template <int DS, bool PRO>
__global__ void __launch_bounds__(NT, 1)
chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_la,
             const ChunkParams p) {
    using SM = Smem<DS>;
    using TM = Tmem<DS>;
    constexpr int NSPLIT = D / DS;
    constexpr uint32_t I_D1 = idesc_bf16_f32(128, 64);               // [Q~;K~] x K-
    constexpr uint32_t I_W = idesc_bf16_f32(64, 128, false, 0, 1);    // T' x K~ (B MN-major)
    constexpr uint32_t I_UT = idesc_bf16_f32(64, DS, false, 0, 1);    // T' x V, Q~ x S, A x U
    constexpr uint32_t I_UWS = idesc_bf16_f32(64, DS, true, 0, 1);    // -W x S
    constexpr uint32_t I_S = idesc_bf16_f32(128, DS, false, 1, 1);    // K-^T x U (A MN-major)
    constexpr int SCOLS = DS / 2;  // TMEM columns of S / U / O per thread (two threads per lane)

    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned (128-byte swizzled tiles); offsetting the shared array itself keeps the
    // accesses in the shared state space (an integer round trip would make them generic)
    uint8_t *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float *s_beta = reinterpret_cast<float *>(sm + SM::MISC);  // [64]
    float *s_gamma = s_beta + 64;                               // [128]
    float *s_psum = s_gamma + 128;                              // [8 + 1][128]
    uint32_t *s_flags = reinterpret_cast<uint32_t *>(s_psum + 9 * 128);  // abort, exact path, tmem
    uint64_t *bars = reinterpret_cast<uint64_t *>(s_flags + 16);     // qk, la, v, mma
    uint64_t *bar_qk = bars, *bar_la = bars + 1, *bar_v = bars + 2, *bar_mma = bars + 3;
    float *LA = reinterpret_cast<float *>(sm + SM::LA);
    float *LT = reinterpret_cast<float *>(sm + SM::LT);
    float *PB = reinterpret_cast<float *>(sm + SM::PB);
    const uint32_t sb = smem_u32(sm);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, half = warp >> 2;
    const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
    const int H = p.H;
    const int split = blockIdx.x % NSPLIT;
    const int hs = blockIdx.x / NSPLIT;
    const int slot = hs / H, h = hs % H;
    const int n = p.order ? p.order[slot] : slot;
    const int d0 = split * DS;  // first value channel of this CTA
    const int64_t bos = p.cu_seqlens[n], eos = p.cu_seqlens[n + 1];
    const int nchunks = (int)((eos - bos + C - 1) / C);
    const float *s0b = init_state_block(p.s0, n, H, h, (size_t)D * D, p.ss);
    float *sTb = final_state_block(p.sT, n, H, h, (size_t)D * D, p.ss);
    if (s0b && !KDA_ACCESS_OK(p.status, p.dbg.init, s0b, D * D * 4, 11)) s0b = nullptr;
    if (sTb && !KDA_ACCESS_OK(p.status, p.dbg.fin, sTb, D * D * 4, 12)) sTb = nullptr;
    const int c_me = 32 * quad + lane;  // key channel = TMEM lane of this thread

    if (tid == 0) {
        s_flags[0] = 0;
        mbar_init(bar_qk, 1);
        mbar_init(bar_la, 1);
        mbar_init(bar_v, 1);
        mbar_init(bar_mma, 1);
        fence_mbarrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_la);
    }
    if (warp == 0) {
        tmem_alloc(&s_flags[2], TM::COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_flags[2];

    auto issue_qk = [&](int64_t t0) {
        mbar_arrive_expect_tx(bar_qk, 32768);
        tma_load_3d(sm + SM::QK, &tm_q, bar_qk, 0, h, (int32_t)t0);
        tma_load_3d(sm + SM::QK + 8192, &tm_k, bar_qk, 0, h, (int32_t)t0);
        tma_load_3d(sm + SM::QK + 16384, &tm_q, bar_qk, 64, h, (int32_t)t0);
        tma_load_3d(sm + SM::QK + 24576, &tm_k, bar_qk, 64, h, (int32_t)t0);
    };
    auto issue_la = [&](int64_t t0) {
        fence_proxy_async_smem();  // the previous contents were read by generic loads
        mbar_arrive_expect_tx(bar_la, 32768);
        tma_load_3d(sm + SM::LA, &tm_la, bar_la, 0, h, (int32_t)t0);
    };
    auto issue_v = [&](int64_t t0) {
        mbar_arrive_expect_tx(bar_v, 128 * DS);
#pragma unroll
        for (int b = 0; b < DS / 64; ++b)
            tma_load_3d(sm + SM::V + 8192 * b, &tm_v, bar_v, d0 + 64 * b, h, (int32_t)t0);
    };
    bool qk_pending = false, la_pending = false, v_pending = false;
    if (nchunks > 0) {
        if (tid == 0) {
            issue_qk(bos);
            issue_la(bos);
            issue_v(bos);
        }
        qk_pending = la_pending = v_pending = true;
    }

    // The strictly upper 16x16 blocks of T' are zero for every chunk.
    for (int e = tid; e < 8192 / 16; e += NT)
        reinterpret_cast<uint4 *>(sm + SM::TT)[e] = make_uint4(0u, 0u, 0u, 0u);

    // Initial state -> S (TMEM fp32, lane c, columns d) and its bf16 tile [c][d].
    {
        const size_t row = (size_t)c_me * D + d0 + half * SCOLS;
        const float *src = s0b ? s0b + row : nullptr;
        float *dst = sTb ? sTb + row : nullptr;
#pragma unroll
        for (int part = 0; part < SCOLS / 32; ++part) {
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
                const int col = half * SCOLS + 32 * part;
                tmem_st32(tmem + lane_base + TM::S + col, v);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    st_chunk(sm + SM::S + tchunk(16384, c_me, col + 8 * q8), v + 8 * q8);
            }
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    uint32_t ph_qk = 0, ph_la = 0, ph_v = 0, ph_mma = 0;
    auto wait_bar = [&](uint64_t *bar, uint32_t &ph) {
        const bool ok = mbar_wait_bounded(bar, ph, p.timeout_ns);
        ph ^= 1u;
        if (!ok) {
            s_flags[0] = 1;
            atomicOr(p.status, 1);
        }
    };

    // beta of the next chunk is loaded one chunk ahead (one value per thread < C)
    const bool raw_beta = PRO && (p.pro.flags & KDA_PROLOGUE_BETA_SIGMOID) != 0;
    auto load_beta = [&](int64_t t) {
        const float *bp = p.beta + (size_t)t * H + h;
        if (!KDA_ACCESS_OK(p.status, p.dbg.beta, bp, 4, 14)) return 0.f;
        const float b = *bp;
        return raw_beta ? beta_from_raw(b) : b;
    };
    float beta_next = 0.f;
    if (nchunks > 0 && tid < C && bos + tid < eos) beta_next = load_beta(bos + tid);

    for (int ci = 0; ci < nchunks; ++ci) {
        const int64_t t0 = bos + (int64_t)ci * C;
        const int valid = (int)(eos - t0 < C ? eos - t0 : C);
        const bool has_next = ci + 1 < nchunks;
        if (tid < C) {
            s_beta[tid] = beta_next;
            beta_next = (has_next && t0 + C + tid < eos) ? load_beta(t0 + C + tid) : 0.f;
        }
        wait_bar(bar_la, ph_la);
        wait_bar(bar_qk, ph_qk);
        la_pending = qk_pending = false;

        // ---- gates and gated operands (exact path: also A and L, and S <- diag(gamma) S)
        const int gate = gate_chunk<PRO>(sm + SM::QK, sm + SM::KI, sm + SM::AQK, LA, LT, s_beta, s_gamma,
                                    s_psum, s_flags, valid, tid, nullptr, nullptr, 0, 0, p.pro);
        if (gate < 0) break;
        const bool safe = gate == 1;
        if (safe) {
            scale_tmem_row<SCOLS>(tmem + lane_base + TM::S + half * SCOLS, s_gamma[c_me]);
            tc_fence_before();
        }
        fence_proxy_async_smem();
        __syncthreads();

        if (tid == 0) {
            tc_fence_after();
            if (!safe) {
#pragma unroll
                for (uint32_t kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tmem + TM::D1, desc_k(sb + SM::QK, 16384, kk),
                                desc_k(sb + SM::KI, 8192, kk), I_D1, kk > 0);
            }
            if (DS <= 64) {  // O = Q~ S now (own TMEM columns)
#pragma unroll
                for (uint32_t kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tmem + TM::O, desc_k(sb + SM::QK, 16384, kk),
                                desc_mn(sb + SM::S, 16384, kk), I_UT, kk > 0);
            }
            mma_commit(bar_mma);
            if (has_next) issue_la(t0 + C);  // the gating is done with log_alpha
        }
        la_pending = has_next;
        wait_bar(bar_mma, ph_mma);
        tc_fence_after();

        // ---- A (D1 rows 0..63) to bf16, L (rows 64..127, times beta_i, j < i) to fp32
        if (!safe) extract_al(tmem + lane_base + TM::D1 + 32 * half, sm + SM::AQK, LT, s_beta, c_me, 32 * half);
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;
        if (DS > 64 && tid == 0) {  // O = Q~ S over D1's columns, while the inverse runs
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk)
                mma_bf16_ss(tmem + TM::O, desc_k(sb + SM::QK, 16384, kk),
                            desc_mn(sb + SM::S, 16384, kk), I_UT, kk > 0);
        }

        // ---- T' = (I + L)^-1 diag(beta), bf16, into the TT tile
        invert_unit_lower(LT, PB, sm + SM::TT, s_beta, tid, tid >> 5);
        fence_proxy_async_smem();
        __syncthreads();

        wait_bar(bar_v, ph_v);  // V of this chunk
        v_pending = false;
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // W = T' K~
                mma_bf16_ss(tmem + TM::W, desc_k(sb + SM::TT, 8192, kk),
                            desc_mn(sb + SM::QK + 8192, 16384, kk), I_W, kk > 0);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // U~ = T' V
                mma_bf16_ss(tmem + TM::U, desc_k(sb + SM::TT, 8192, kk),
                            desc_mn(sb + SM::V, 8192, kk), I_UT, kk > 0);
            mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma);
        tc_fence_after();
        if (tid == 0 && has_next) {
            issue_v(t0 + C);
            issue_qk(t0 + C);  // Q~ and K~ are consumed (O = Q~ S was issued before W)
        }
        v_pending = has_next;
        qk_pending = has_next;

        // ---- W (TMEM, M=64: row 16*quad + lane for lane < 16) -> bf16 tile [i][c]
        rows64_to_tile<64>(tmem + lane_base + TM::W + 64 * half, sm + SM::W, 8192, 64 * half, quad, lane);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;

        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk)  // U = U~ - W S
                mma_bf16_ss(tmem + TM::U, desc_k(sb + SM::W, 8192, kk),
                            desc_mn(sb + SM::S, 16384, kk), I_UWS, 1);
            mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma);
        tc_fence_after();

        // ---- U (TMEM, M=64) -> bf16 tile [j][d]
        rows64_to_tile<SCOLS>(tmem + lane_base + TM::U + half * SCOLS, sm + SM::U, 8192, half * SCOLS, quad, lane);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;

        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // O += A U
                mma_bf16_ss(tmem + TM::O, desc_k(sb + SM::AQK, 8192, kk),
                            desc_mn(sb + SM::U, 8192, kk), I_UT, 1);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)  // S += K-^T U   (K^^T U on the exact path)
                mma_bf16_ss(tmem + TM::S, desc_mn(sb + SM::KI, 8192, kk),
                            desc_mn(sb + SM::U, 8192, kk), I_S, 1);
            mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma);
        tc_fence_after();

        // ---- outputs (O: M=64 rows) and the next state (S *= gamma on the fast path)
        {
            constexpr int NPART = SCOLS / 32;
            float vv[NPART][32];  // every 32-column load in flight before one wait
#pragma unroll
            for (int part = 0; part < NPART; ++part)
                tmem_ld32(tmem + lane_base + TM::O + half * SCOLS + 32 * part, vv[part]);
            tmem_wait_ld();
#pragma unroll
            for (int part = 0; part < NPART; ++part) {
                const int col = half * SCOLS + 32 * part;
                const float *v = vv[part];
                const int i = 16 * quad + lane;
                if (lane < 16 && i < valid &&
                    KDA_ACCESS_OK(p.status, p.dbg.out, p.out + ((size_t)(t0 + i) * H + h) * D + d0 + col, 64, 13)) {
                    uint4 *dst = reinterpret_cast<uint4 *>(
                        p.out + ((size_t)(t0 + i) * H + h) * D + d0 + col);
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8)
                        dst[q8] = make_uint4(pack2(v[8 * q8], v[8 * q8 + 1]),
                                             pack2(v[8 * q8 + 2], v[8 * q8 + 3]),
                                             pack2(v[8 * q8 + 4], v[8 * q8 + 5]),
                                             pack2(v[8 * q8 + 6], v[8 * q8 + 7]));
                }
            }
            const float gm = safe ? 1.f : s_gamma[c_me];
#pragma unroll
            for (int part = 0; part < NPART; ++part)
                tmem_ld32(tmem + lane_base + TM::S + half * SCOLS + 32 * part, vv[part]);
            tmem_wait_ld();
#pragma unroll
            for (int part = 0; part < NPART; ++part) {
                const int col = half * SCOLS + 32 * part;
                const uint32_t ta = tmem + lane_base + TM::S + col;
                float *v = vv[part];
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] *= gm;
                if (!safe) tmem_st32(ta, vv[part]);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    st_chunk(sm + SM::S + tchunk(16384, c_me, col + 8 * q8), v + 8 * q8);
                if (!has_next && sTb) {
                    float *dst = sTb + (size_t)c_me * D + d0 + col;
#pragma unroll
                    for (int e = 0; e < 32; e += 4)
                        *reinterpret_cast<float4 *>(dst + e) =
                            make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                }
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;
    }

    // ---- teardown: on an abort, let in-flight copies and MMAs land before freeing TMEM
    if (s_flags[0] && tid == 0) {
        if (qk_pending) mbar_wait_bounded(bar_qk, ph_qk, p.timeout_ns);
        if (la_pending) mbar_wait_bounded(bar_la, ph_la, p.timeout_ns);
        if (v_pending) mbar_wait_bounded(bar_v, ph_v, p.timeout_ns);
        mma_commit(bar_mma);
        mbar_wait_bounded(bar_mma, ph_mma, p.timeout_ns);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM::COLS);
    }
}

// Longest-first order of the sequences (ties by index); the first CTAs take the
// longest sequences so the longest chain does not set the tail. Also clears the
// device status word.
__global__ void plan_kernel(const int32_t *__restrict__ cu, int32_t N, int32_t *__restrict__ order,
                            int32_t *__restrict__ status) {
    if (blockIdx.x == 0 && threadIdx.x == 0) *status = 0;
    for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < N; n += gridDim.x * blockDim.x) {
        const int32_t ln = cu[n + 1] - cu[n];
        int32_t rank = 0;
        for (int m = 0; m < N; ++m) {
            const int32_t lm = cu[m + 1] - cu[m];
            rank += (lm > ln) || (lm == ln && m < n);
        }
        order[rank] = n;
    }
}

// Waits on an mbarrier that nothing ever arrives at, with the same bounded wait the
// chunk kernel uses; records the timeout in the status word and returns.
__global__ void bounded_wait_probe(int32_t *status, uint64_t timeout_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbarrier_init();
    }
    __syncthreads();
    if (!mbar_wait_bounded(&bar, 0, timeout_ns) && threadIdx.x == 0)
        atomicOr(status, 1);
}

// Waits on a global word that nothing writes (cleared here, released at 1) with the split
// kernel's inter-CTA flag wait; records the timeout in the status word and returns.
__global__ void flag_wait_probe(int32_t *status, int32_t *flag, uint64_t timeout_ns) {
    if (threadIdx.x == 0) {
        if (!wait_flag_ge(flag, 1, timeout_ns)) atomicOr(status, 1);
    }
}

template <int DS, bool PRO>
cudaError_t launch_ds(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                      const CUtensorMap &mla, const ChunkParams &cp, unsigned grid,
                      cudaStream_t stream) {
    static PerDeviceOnce<> once;
    const cudaError_t attr_err =
        set_smem_limit_once(once, (const void *)chunk_kernel<DS, PRO>, (int)Smem<DS>::BYTES);
    if (attr_err != cudaSuccess) return attr_err;
    chunk_kernel<DS, PRO><<<grid, NT, Smem<DS>::BYTES, stream>>>(mq, mk, mv, mla, cp);
    return cudaGetLastError();
}

}  // namespace

namespace {
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

}  // namespace

bool make_token_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint32_t esize,
              uint64_t inner, uint64_t H, uint64_t T, uint32_t box_inner, bool swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {inner, H, T};
    cuuint64_t strides[2] = {inner * esize, inner * H * esize};
    cuuint32_t box[3] = {box_inner, 1, (cuuint32_t)C};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_bounded_wait_probe(void *workspace, uint64_t timeout_ns, cudaStream_t stream) {
    bounded_wait_probe<<<1, 32, 0, stream>>>(static_cast<int32_t *>(workspace), timeout_ns);
    return cudaGetLastError();
}

cudaError_t launch_flag_wait_probe(void *workspace, uint64_t timeout_ns, cudaStream_t stream) {
    // status word at byte 0, the never-released flag at byte 128 (both zeroed by the caller)
    int32_t *ws = static_cast<int32_t *>(workspace);
    flag_wait_probe<<<1, 32, 0, stream>>>(ws, ws + 32, timeout_ns);
    return cudaGetLastError();
}

bool chunk_supported(const Problem &p) {
    return p.dtype == KDA_BF16 && p.dk == D && p.dv == D && p.total_tokens > 0;
}

size_t chunk_workspace_bytes(int32_t num_seqs) {
    return 256 + ((size_t)num_seqs * 4 + 255) / 256 * 256;
}

cudaError_t launch_prefill_chunk(const Problem &p, void *workspace, cudaStream_t stream,
                                 uint64_t timeout_ns) {
    // Few (sequence, head) pairs cannot fill the GPU: split d_v across two CTAs per head.
    int sms = 148;
    {
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const int64_t heads = (int64_t)p.num_seqs * p.H;
    const int nsplit = heads * 2 <= sms ? 2 : 1;
    CUtensorMap mq, mk, mv, mla;
    const uint64_t T = (uint64_t)p.total_tokens, H = (uint64_t)p.H;
    if (!make_token_map(&mq, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_token_map(&mk, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_token_map(&mv, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_token_map(&mla, p.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, H, T, D, false))
        return cudaErrorInvalidValue;
    int32_t *status = reinterpret_cast<int32_t *>(workspace);
    int32_t *order = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) + 256);
    const int plan_threads = 256;
    const int plan_blocks = (p.num_seqs + plan_threads - 1) / plan_threads;
    plan_kernel<<<plan_blocks, plan_threads, 0, stream>>>(p.cu_seqlens, p.num_seqs, order, status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    ChunkParams cp;
    cp.cu_seqlens = p.cu_seqlens;
    cp.order = order;
    cp.beta = p.beta;
    cp.pro = p.pro;
    cp.s0 = p.initial_state;
    cp.sT = p.final_state;
    cp.dbg = p.dbg;
    cp.out = static_cast<__nv_bfloat16 *>(p.out);
    cp.status = status;
    cp.ss = p.slots;
    cp.ss.status = status;
    cp.H = p.H;
    cp.timeout_ns = timeout_ns;
    const unsigned grid = (unsigned)(heads * nsplit);
    if (p.pro.flags)
        return nsplit == 2 ? launch_ds<64, true>(mq, mk, mv, mla, cp, grid, stream)
                           : launch_ds<128, true>(mq, mk, mv, mla, cp, grid, stream);
    return nsplit == 2 ? launch_ds<64, false>(mq, mk, mv, mla, cp, grid, stream)
                       : launch_ds<128, false>(mq, mk, mv, mla, cp, grid, stream);
}

}  // namespace kda
