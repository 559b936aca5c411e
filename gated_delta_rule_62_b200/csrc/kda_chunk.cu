// Chunked KDA prefill on tcgen05 tensor cores (bf16 operands, fp32 accumulators in TMEM).
//
// "KDA's update is organized blockwise ... so it maps onto GPU matrix units"
// (shivam2003.com Kimi K3 article, section "Kimi Delta Attention: the
// load-bearing choice"). The blockwise form used here is derived from the
// per-token recurrence (decay, delta-rule write, read after the write):
//
// For a chunk of C = 64 tokens starting from state S (d_k x d_v), with
// g_i = sum_{s<=i} log_alpha_s (inclusive, per key channel), gamma = exp(g_{C-1}),
//   Q~ = q * e^g,  K~ = k * e^g,  K- = k * e^-g,  K^ = k * e^(g_{C-1} - g)      (rows = tokens)
//   A  = tril(Q~ K-^T)        (j <= i),    L = diag(beta) strictly_tril(K~ K-^T)
//   T  = (I + L)^-1,  W = T diag(beta) K~,  U~ = T diag(beta) V
//   U  = U~ - W S                          (the errors the delta rule writes)
//   O  = Q~ S + A U
//   S' = diag(gamma) S + K^^T U
// which is the WY/UT form of the product of the per-token transitions
// (I - beta k k^T) Diag(alpha) over the chunk. Every product is computed
// transposed so that M = 128 (d_v or d_k) fills the tensor core's 128 lanes:
//   U^T = (beta V)^T T^T - S^T W^T,  O^T = S^T Q~^T + U^T A^T,
//   S'^T = S^T diag(gamma) + U^T K^,  W^T = (beta K~)^T T^T,  [Q~; K~] K-^T.
// The fp32 master state S^T stays in TMEM for the whole sequence (lane = value
// channel, column = key channel); a bf16 copy in shared memory feeds the MMAs.
//
// Factoring e^(g_i - g_j) = e^(g_i) e^(-g_j) overflows when a chunk decays by more
// than ~e^88 in some channel. Chunks whose total decay exceeds e^60 take an
// exact path that forms A and L pairwise on CUDA cores instead.
//
// One CTA (256 threads, 1 per SM) per (sequence, head); TMA brings each chunk's
// q, k (128-byte swizzled, directly in the MMA operand layout), v and
// log_alpha tiles into shared memory, prefetching the next chunk while the
// current one computes. Every on-device wait is bounded; on timeout the
// kernel records KDA_ERR_TIMEOUT in the workspace status word and returns.
#include <cuda.h>

#include <mutex>

#include "kda_internal.cuh"
#include "sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = 64;    // chunk length
constexpr int D = 128;   // d_k = d_v
constexpr int NT = 256;  // threads per CTA
constexpr float kFastLimit = 60.f;  // max in-chunk decay exponent for the factored path

// Shared-memory map (byte offsets from a 1024-aligned base). bf16 operand tiles are
// K-major with the 128-byte swizzle; a tile with K = 128 is two 64-wide K atoms.
constexpr uint32_t OFF_QK = 0;                   // [Q~; K~] 128 rows x K=128 (raw q/k on arrival)
constexpr uint32_t OFF_KI = OFF_QK + 32768;      // K- [j][c] 64 x 128, later W [i][c]
constexpr uint32_t OFF_KBT = OFF_KI + 16384;     // (beta K~)^T [c][j] 128 x 64, later U^T [d][j]
constexpr uint32_t OFF_VBT = OFF_KBT + 16384;    // (beta V)^T [d][j] 128 x 64
constexpr uint32_t OFF_KHT = OFF_VBT + 16384;    // K^^T [c][j] 128 x 64
constexpr uint32_t OFF_AQK = OFF_KHT + 16384;    // A [i][j] 64 x 64
constexpr uint32_t OFF_TT = OFF_AQK + 8192;      // T [i][j] 64 x 64
constexpr uint32_t OFF_ST = OFF_TT + 8192;       // S^T bf16 [d][c] 128 x 128
constexpr uint32_t OFF_VR = OFF_ST + 32768;      // raw v [t][d] bf16 (TMA, unswizzled)
constexpr uint32_t OFF_LA = OFF_VR + 16384;      // raw log_alpha [t][c] fp32 (TMA), then g
constexpr uint32_t LT_LD = 68;                   // fp32 pitch of the L / T scratch
constexpr uint32_t OFF_LT = OFF_LA + 32768;      // L -> T fp32 [64][68]
constexpr uint32_t OFF_P = OFF_LT + 64 * LT_LD * 4;  // 3 x 16 x 16 fp32 block products
constexpr uint32_t OFF_MISC = OFF_P + 3 * 256 * 4;
constexpr uint32_t MISC_BYTES = 64 * 4 + 128 * 4 + 256 * 4 + 64 + 64;
constexpr uint32_t SMEM_BYTES = OFF_MISC + MISC_BYTES + 1024;  // + alignment slack

// TMEM columns (fp32, 128 lanes).
constexpr uint32_t TM_S = 0, TM_D1 = 128, TM_W = 192, TM_U = 256, TM_O = 320, TM_COLS = 512;

constexpr uint32_t IDESC_N64 = idesc_bf16_f32(128, 64);
constexpr uint32_t IDESC_N64_NEG = idesc_bf16_f32(128, 64, true);
constexpr uint32_t IDESC_N128 = idesc_bf16_f32(128, 128);

struct ChunkParams {
    const int32_t *cu_seqlens;
    const int32_t *order;  // sequences, longest first
    const float *beta;
    const float *s0;
    float *sT;
    __nv_bfloat16 *out;
    int32_t *status;
    int32_t H;
    uint64_t timeout_ns;
};

// Byte offset of element (row, k) in a K-major SW128 bf16 tile of `rows` rows.
__device__ __forceinline__ uint32_t sw_off(uint32_t rows, uint32_t row, uint32_t k) {
    const uint32_t kk = k & 63;
    return (k >> 6) * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128 +
           (((kk >> 3) ^ (row & 7)) << 4) + ((kk & 7) << 1);
}
// Byte offset of the 16-byte chunk holding elements (row, k .. k+7), k % 8 == 0.
__device__ __forceinline__ uint32_t sw_chunk(uint32_t rows, uint32_t row, uint32_t k) {
    const uint32_t kk = k & 63;
    return (k >> 6) * rows * 128 + (row >> 3) * 1024 + (row & 7) * 128 +
           (((kk >> 3) ^ (row & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}
__device__ __forceinline__ void st_chunk(uint8_t *p, const float *v) {
    uint4 u = make_uint4(pack2(v[0], v[1]), pack2(v[2], v[3]), pack2(v[4], v[5]),
                         pack2(v[6], v[7]));
    *reinterpret_cast<uint4 *>(p) = u;
}
__device__ __forceinline__ float ld_bf(const uint8_t *p) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p));
}
__device__ __forceinline__ void st_bf(uint8_t *p, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(p) = __float2bfloat16_rn(x);
}

// Descriptor of K-step kk (16 elements) of a K-major SW128 tile with `rows` rows.
__device__ __forceinline__ uint64_t kdesc(uint32_t base, uint32_t rows, uint32_t kk) {
    return smem_desc_sw128(base + (kk >> 2) * rows * 128 + (kk & 3) * 32);
}

// T = (I + L)^-1 for strictly lower-triangular L (fp32, pitch LT_LD), in place.
// Diagonal 16x16 blocks by forward substitution (one column per lane), then the
// off-diagonal blocks row by row: T_rc = -T_rr sum_{k=c}^{r-1} L_rk T_kc.
__device__ void invert_unit_lower(float *LT, float *P, int tid) {
    if (tid < 128 && (tid & 31) < 16) {
        const int w = tid >> 5, l = tid & 31;
        float *Lb = LT + (16 * w) * LT_LD + 16 * w;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float s = (i == l) ? 1.f : 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) s = fmaf(-Lb[i * LT_LD + j], x[j], s);
            x[i] = s;
        }
        __syncwarp(0x0000ffffu);
#pragma unroll
        for (int i = 0; i < 16; ++i) Lb[i * LT_LD + l] = x[i];
    }
    __syncthreads();
    for (int r = 1; r < 4; ++r) {
        for (int e = tid; e < r * 256; e += NT) {
            const int cb = e >> 8, i = (e >> 4) & 15, j = e & 15;
            const float *Lrow = LT + (16 * r + i) * LT_LD;
            float s = 0.f;
            for (int k = 16 * cb; k < 16 * r; ++k) s = fmaf(Lrow[k], LT[k * LT_LD + 16 * cb + j], s);
            P[e] = s;
        }
        __syncthreads();
        for (int e = tid; e < r * 256; e += NT) {
            const int cb = e >> 8, i = (e >> 4) & 15, j = e & 15;
            const float *Trow = LT + (16 * r + i) * LT_LD + 16 * r;
            float s = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m) s = fmaf(Trow[m], P[cb * 256 + m * 16 + j], s);
            LT[(16 * r + i) * LT_LD + 16 * cb + j] = -s;
        }
        __syncthreads();
    }
}

__global__ void __launch_bounds__(NT, 1)
chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_la,
             const ChunkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    float *s_beta = reinterpret_cast<float *>(sm + OFF_MISC);  // [64]
    float *s_gamma = s_beta + 64;                                // [128]
    float *s_psum = s_gamma + 128;                               // [2][128]
    uint32_t *s_flags = reinterpret_cast<uint32_t *>(s_psum + 256);  // abort, maxdecay, tmem
    uint64_t *bars = reinterpret_cast<uint64_t *>(s_flags + 16);     // qk, lv, mma
    uint64_t *bar_qk = bars, *bar_lv = bars + 1, *bar_mma = bars + 2;
    float *LA = reinterpret_cast<float *>(sm + OFF_LA);
    float *LT = reinterpret_cast<float *>(sm + OFF_LT);
    float *P = reinterpret_cast<float *>(sm + OFF_P);
    const uint32_t sbase = smem_u32(sm);

    const int tid = threadIdx.x;
    const int r = tid & 127, hf = tid >> 7, warp = tid >> 5;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int H = p.H;
    const int slot = blockIdx.x / H, h = blockIdx.x % H;
    const int n = p.order ? p.order[slot] : slot;
    const int64_t bos = p.cu_seqlens[n], eos = p.cu_seqlens[n + 1];
    const int nchunks = (int)((eos - bos + C - 1) / C);
    const size_t state_off = ((size_t)n * H + h) * (size_t)(D * D);

    if (tid == 0) {
        s_flags[0] = 0;
        mbar_init(bar_qk, 1);
        mbar_init(bar_lv, 1);
        mbar_init(bar_mma, 1);
        fence_mbarrier_init();
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_la);
    }
    if (warp == 0) {
        tmem_alloc(&s_flags[2], TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_flags[2];

    auto issue_qk = [&](int64_t t0) {
        mbar_arrive_expect_tx(bar_qk, 32768);
        tma_load_3d(sm + OFF_QK, &tm_q, bar_qk, 0, h, (int32_t)t0);
        tma_load_3d(sm + OFF_QK + 8192, &tm_k, bar_qk, 0, h, (int32_t)t0);
        tma_load_3d(sm + OFF_QK + 16384, &tm_q, bar_qk, 64, h, (int32_t)t0);
        tma_load_3d(sm + OFF_QK + 24576, &tm_k, bar_qk, 64, h, (int32_t)t0);
    };
    auto issue_lv = [&](int64_t t0) {
        mbar_arrive_expect_tx(bar_lv, 32768 + 16384);
        tma_load_3d(sm + OFF_LA, &tm_la, bar_lv, 0, h, (int32_t)t0);
        tma_load_3d(sm + OFF_VR, &tm_v, bar_lv, 0, h, (int32_t)t0);
    };
    bool qk_pending = false, lv_pending = false;
    if (nchunks > 0 && tid == 0) {
        issue_qk(bos);
        issue_lv(bos);
    }
    if (nchunks > 0) qk_pending = lv_pending = true;

    // Initial state -> S^T (TMEM fp32, lane d, column c) and its bf16 copy (rows d).
    {
        const int d = r;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            const int c0 = 64 * hf + 32 * part;
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e)
                v[e] = p.s0 ? p.s0[state_off + (size_t)(c0 + e) * D + d] : 0.f;
            if (nchunks == 0) {
                if (p.sT) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) p.sT[state_off + (size_t)(c0 + e) * D + d] = v[e];
                }
            } else {
                tmem_st32(tmem + lane_base + TM_S + c0, v);
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    st_chunk(sm + OFF_ST + sw_chunk(128, d, c0 + 8 * q8), v + 8 * q8);
            }
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    uint32_t ph_qk = 0, ph_lv = 0, ph_mma = 0;
    const uint64_t deadline_step = p.timeout_ns;
    auto wait_bar = [&](uint64_t *bar, uint32_t &ph) {
        const bool ok = mbar_wait_bounded(bar, ph, globaltimer_ns() + deadline_step);
        ph ^= 1u;
        if (!ok) {
            s_flags[0] = 1;
            atomicOr(p.status, 1);
        }
    };

    for (int ci = 0; ci < nchunks; ++ci) {
        const int64_t t0 = bos + (int64_t)ci * C;
        const int valid = (int)(eos - t0 < C ? eos - t0 : C);
        const bool has_next = ci + 1 < nchunks;
        if (tid < C) s_beta[tid] = (tid < valid) ? p.beta[(size_t)(t0 + tid) * H + h] : 0.f;
        if (tid == 0) s_flags[1] = 0;
        wait_bar(bar_lv, ph_lv);
        wait_bar(bar_qk, ph_qk);
        lv_pending = qk_pending = false;
        __syncthreads();
        if (s_flags[0]) break;

        // ---- gate cumsum: thread (c = r, half hf) scans tokens [32 hf, 32 hf + 32)
        const int c = r, i0 = 32 * hf;
        {
            float acc = 0.f;
#pragma unroll 8
            for (int i = 0; i < 32; ++i) {
                const int t = i0 + i;
                const float x = (t < valid) ? LA[t * D + c] : 0.f;
                acc += x;
                LA[t * D + c] = acc;
            }
            s_psum[hf * D + c] = acc;
        }
        __syncthreads();
        float goff = hf ? s_psum[c] : 0.f;
        const float gC = s_psum[c] + s_psum[D + c];
        if (hf == 0) {
            s_gamma[c] = __expf(gC);
            // Any channel decaying by more than e^kFastLimit sends the chunk down the exact path.
            // (Also taken for non-finite gates: the comparison below is false for NaN.)
            if (!(-gC <= kFastLimit)) s_flags[1] = 1u;
        }
        __syncthreads();
        const bool safe = s_flags[1] != 0u;

        if (safe) {
            // Exact path: A and L formed pairwise from raw q, k and g (no factored exponentials).
            if (hf) {
                for (int i = 0; i < 32; ++i) LA[(i0 + i) * D + c] += goff;
            }
            goff = 0.f;
            for (int e = tid; e < 64 * 64; e += NT) {
                const int i = e >> 6, j = e & 63;
                st_bf(sm + OFF_AQK + sw_off(64, i, j), 0.f);
                LT[i * LT_LD + j] = 0.f;
            }
            __syncthreads();
            const int lane = tid & 31;
            for (int e = warp; e < 64 * 64; e += NT / 32) {
                const int i = e >> 6, j = e & 63;
                if (j > i || i >= valid) continue;
                float a = 0.f, l = 0.f;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int cc = lane + 32 * m;
                    const float ex = __expf(LA[i * D + cc] - LA[j * D + cc]);
                    const float kj = ld_bf(sm + OFF_QK + sw_off(128, 64 + j, cc)) * ex;
                    a = fmaf(ld_bf(sm + OFF_QK + sw_off(128, i, cc)), kj, a);
                    l = fmaf(ld_bf(sm + OFF_QK + sw_off(128, 64 + i, cc)), kj, l);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    a += __shfl_xor_sync(0xffffffffu, a, off);
                    l += __shfl_xor_sync(0xffffffffu, l, off);
                }
                if (lane == 0) {
                    st_bf(sm + OFF_AQK + sw_off(64, i, j), a);
                    if (j < i) LT[i * LT_LD + j] = s_beta[i] * l;
                }
            }
            __syncthreads();
        }

        // ---- gated operands for tokens [i0, i0 + 32) of channel c (and value channel d = r)
        {
            const float gam = s_gamma[c];
            float khat[8], kbt[8], vbt[8];
#pragma unroll 1
            for (int i8 = 0; i8 < 32; i8 += 8) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int t = i0 + i8 + u;
                    const bool ok = t < valid;
                    const float g = goff + LA[t * D + c];
                    const float eg = __expf(g), emg = __expf(-g);
                    uint8_t *qp = sm + OFF_QK + sw_off(128, t, c);
                    uint8_t *kp = sm + OFF_QK + sw_off(128, 64 + t, c);
                    const float qv = ok ? ld_bf(qp) : 0.f;
                    const float kv = ok ? ld_bf(kp) : 0.f;
                    const float bt = s_beta[t];
                    st_bf(qp, qv * eg);
                    st_bf(kp, kv * eg);
                    if (!safe) st_bf(sm + OFF_KI + sw_off(64, t, c), kv * emg);
                    khat[u] = safe ? kv * __expf(gC - g) : kv * emg * gam;
                    kbt[u] = bt * kv * eg;
                    const __nv_bfloat16 vr =
                        reinterpret_cast<const __nv_bfloat16 *>(sm + OFF_VR)[t * D + r];
                    vbt[u] = ok ? bt * __bfloat162float(vr) : 0.f;
                }
                st_chunk(sm + OFF_KHT + sw_chunk(128, c, i0 + i8), khat);
                st_chunk(sm + OFF_KBT + sw_chunk(128, c, i0 + i8), kbt);
                st_chunk(sm + OFF_VBT + sw_chunk(128, r, i0 + i8), vbt);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();

        if (tid == 0) {
            if (has_next) {
                fence_proxy_async_smem();
                issue_lv(t0 + C);
            }
            tc_fence_after();
            if (!safe) {
#pragma unroll
                for (uint32_t kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tmem + TM_D1, kdesc(sbase + OFF_QK, 128, kk),
                                kdesc(sbase + OFF_KI, 64, kk), IDESC_N64, kk > 0);
            }
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk)
                mma_bf16_ss(tmem + TM_O, kdesc(sbase + OFF_ST, 128, kk),
                            kdesc(sbase + OFF_QK, 128, kk), IDESC_N64, kk > 0);
            mma_commit(bar_mma);
        }
        lv_pending = has_next;
        wait_bar(bar_mma, ph_mma);
        tc_fence_after();
        if (tid == 0 && has_next) {
            fence_proxy_async_smem();
            issue_qk(t0 + C);
        }
        qk_pending = has_next;

        // ---- A (rows 0..63 of D1) to bf16, L (rows 64..127) to fp32 scratch
        if (!safe) {
            float v[32];
            tmem_ld32(tmem + lane_base + TM_D1 + 32 * hf, v);
            tmem_wait_ld();
            if (r < 64) {
                const int i = r;
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = (32 * hf + e <= i) ? v[e] : 0.f;
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    st_chunk(sm + OFF_AQK + sw_chunk(64, i, 32 * hf + 8 * q8), v + 8 * q8);
            } else {
                const int i = r - 64;
                const float b = s_beta[i];
                float4 *dst = reinterpret_cast<float4 *>(LT + i * LT_LD + 32 * hf);
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                    float4 w;
                    w.x = (32 * hf + 4 * e4 + 0 < i) ? b * v[4 * e4 + 0] : 0.f;
                    w.y = (32 * hf + 4 * e4 + 1 < i) ? b * v[4 * e4 + 1] : 0.f;
                    w.z = (32 * hf + 4 * e4 + 2 < i) ? b * v[4 * e4 + 2] : 0.f;
                    w.w = (32 * hf + 4 * e4 + 3 < i) ? b * v[4 * e4 + 3] : 0.f;
                    dst[e4] = w;
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;

        // ---- T = (I + L)^-1, then bf16 into the MMA tile
        invert_unit_lower(LT, P, tid);
        {
            const int i = tid >> 2, j0 = (tid & 3) * 16;
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = LT[i * LT_LD + j0 + e];
            st_chunk(sm + OFF_TT + sw_chunk(64, i, j0), v);
            st_chunk(sm + OFF_TT + sw_chunk(64, i, j0 + 8), v + 8);
        }
        fence_proxy_async_smem();
        __syncthreads();

        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + TM_W, kdesc(sbase + OFF_KBT, 128, kk),
                            kdesc(sbase + OFF_TT, 64, kk), IDESC_N64, kk > 0);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + TM_U, kdesc(sbase + OFF_VBT, 128, kk),
                            kdesc(sbase + OFF_TT, 64, kk), IDESC_N64, kk > 0);
            mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma);
        tc_fence_after();

        // ---- W^T (lane c, column i) -> W [i][c] bf16 (reuses the K- tile)
        {
            float v[32];
            tmem_ld32(tmem + lane_base + TM_W + 32 * hf, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) st_bf(sm + OFF_KI + sw_off(64, 32 * hf + e, c), v[e]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;

        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 8; ++kk)
                mma_bf16_ss(tmem + TM_U, kdesc(sbase + OFF_ST, 128, kk),
                            kdesc(sbase + OFF_KI, 64, kk), IDESC_N64_NEG, 1);
            mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma);
        tc_fence_after();

        // ---- U^T (lane d, column j) -> bf16 tile (reuses the (beta K~)^T tile); S^T *= gamma
        {
            float v[32];
            tmem_ld32(tmem + lane_base + TM_U + 32 * hf, v);
            tmem_wait_ld();
#pragma unroll
            for (int q8 = 0; q8 < 4; ++q8)
                st_chunk(sm + OFF_KBT + sw_chunk(128, r, 32 * hf + 8 * q8), v + 8 * q8);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const int c0 = 64 * hf + 32 * part;
                tmem_ld32(tmem + lane_base + TM_S + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] *= s_gamma[c0 + e];
                tmem_st32(tmem + lane_base + TM_S + c0, v);
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;

        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + TM_O, kdesc(sbase + OFF_KBT, 128, kk),
                            kdesc(sbase + OFF_AQK, 64, kk), IDESC_N64, 1);
#pragma unroll
            for (uint32_t kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tmem + TM_S, kdesc(sbase + OFF_KBT, 128, kk),
                            kdesc(sbase + OFF_KHT, 128, kk), IDESC_N128, 1);
            mma_commit(bar_mma);
        }
        wait_bar(bar_mma, ph_mma);
        tc_fence_after();

        // ---- outputs (O^T: lane d, column i) and the new state's bf16 copy
        {
            const int d = r;
            float v[32];
            tmem_ld32(tmem + lane_base + TM_O + 32 * hf, v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int i = 32 * hf + e;
                if (i < valid) p.out[((size_t)(t0 + i) * H + h) * D + d] = __float2bfloat16_rn(v[e]);
            }
            const bool last = ci + 1 == nchunks;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const int c0 = 64 * hf + 32 * part;
                tmem_ld32(tmem + lane_base + TM_S + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int q8 = 0; q8 < 4; ++q8)
                    st_chunk(sm + OFF_ST + sw_chunk(128, d, c0 + 8 * q8), v + 8 * q8);
                if (last && p.sT) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) p.sT[state_off + (size_t)(c0 + e) * D + d] = v[e];
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (s_flags[0]) break;
    }

    // ---- teardown: on an abort, let in-flight copies and MMAs land before freeing TMEM
    if (s_flags[0] && tid == 0) {
        const uint64_t dl = globaltimer_ns() + deadline_step;
        if (qk_pending) mbar_wait_bounded(bar_qk, ph_qk, dl);
        if (lv_pending) mbar_wait_bounded(bar_lv, ph_lv, dl);
        mma_commit(bar_mma);
        mbar_wait_bounded(bar_mma, ph_mma, dl);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, TM_COLS);
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
    if (!mbar_wait_bounded(&bar, 0, globaltimer_ns() + timeout_ns) && threadIdx.x == 0)
        atomicOr(status, 1);
}

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

// 3-D map over [T][H][inner] with a box of (box_inner, 1, 64 tokens).
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint32_t esize,
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

}  // namespace

cudaError_t launch_bounded_wait_probe(void *workspace, uint64_t timeout_ns, cudaStream_t stream) {
    bounded_wait_probe<<<1, 32, 0, stream>>>(static_cast<int32_t *>(workspace), timeout_ns);
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
    CUtensorMap mq, mk, mv, mla;
    const uint64_t T = (uint64_t)p.total_tokens, H = (uint64_t)p.H;
    if (!make_map(&mq, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_map(&mk, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, 64, true) ||
        !make_map(&mv, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, H, T, D, false) ||
        !make_map(&mla, p.log_alpha, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, D, H, T, D, false))
        return cudaErrorInvalidValue;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)SMEM_BYTES);
    });
    if (attr_err != cudaSuccess) return attr_err;
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
    cp.s0 = p.initial_state;
    cp.sT = p.final_state;
    cp.out = static_cast<__nv_bfloat16 *>(p.out);
    cp.status = status;
    cp.H = p.H;
    cp.timeout_ns = timeout_ns;
    const unsigned grid = (unsigned)p.num_seqs * (unsigned)p.H;
    chunk_kernel<<<grid, NT, SMEM_BYTES, stream>>>(mq, mk, mv, mla, cp);
    return cudaGetLastError();
}

}  // namespace kda
