// Token-serial KDA prefill: the recurrence walked one token at a time in fp32.
//
// Used for fp32 inputs and for head sizes the tensor-core chunk kernel does not
// cover. Per token (channel-wise forgetting, then the delta-rule write of the
// error, then the read -- "How the delta rule actually works" and "Kimi Delta
// Attention: the load-bearing choice" in the shivam2003.com Kimi K3 article):
//   S <- Diag(alpha) S;  a = S^T k;  b = S^T q;  u = beta (v - a);
//   S <- S + k u^T;      o = S^T q = b + (k.q) u.
// The last identity lets one pass over S produce both reductions.
//
// Mapping: one 128-thread block per (sequence, head, 32-column slice of d_v).
// Warp w owns columns [8w, 8w+8) of the slice; lane l owns key rows l + 32m.
// The state slice lives in registers for the whole sequence.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kCols = 8;           // value columns per warp
constexpr int kSlice = 4 * kCols;  // value columns per block

template <typename Tin, int DK>
__global__ void __launch_bounds__(128)
recurrent_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                 const float *__restrict__ log_alpha, const float *__restrict__ beta,
                 const float *s0, const int32_t *__restrict__ cu_seqlens, int H,
                 int dv, Tin *__restrict__ out, float *sT, const StateSlots ss,
                 const Prologue pro, const DebugRanges dbg) {
    constexpr int R = DK / 32;  // key rows per lane
    const int n = blockIdx.x, h = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col0 = blockIdx.z * kSlice + warp * kCols;
    const int64_t bos = cu_seqlens[n], eos = cu_seqlens[n + 1];

    float S[R][kCols];
    const float *src = init_state_block(s0, n, H, h, (size_t)DK * dv, ss);
    if (src && !KDA_ACCESS_OK(ss.status, dbg.init, src, DK * dv * 4, 41)) src = nullptr;
#pragma unroll
    for (int m = 0; m < R; ++m)
#pragma unroll
        for (int j = 0; j < kCols; ++j)
            S[m][j] = src ? src[(size_t)(lane + 32 * m) * dv + col0 + j] : 0.f;

    // Software pipeline: the next token's operands are loaded while this one computes.
    float kc[R], qc[R], lc[R], vj[kCols], bt = 0.f;
    auto load = [&](int64_t t, float *kk, float *qq, float *ll, float *vv, float &bb) {
        const size_t rk = ((size_t)t * H + h) * DK, rv = ((size_t)t * H + h) * dv + col0;
#pragma unroll
        for (int m = 0; m < R; ++m) {
            kk[m] = to_f32(k[rk + lane + 32 * m]);
            qq[m] = to_f32(q[rk + lane + 32 * m]);
            ll[m] = log_alpha[rk + lane + 32 * m];
        }
#pragma unroll
        for (int j = 0; j < kCols; ++j) vv[j] = to_f32(v[rv + j]);
        bb = beta[(size_t)t * H + h];
    };
    if (bos < eos) load(bos, kc, qc, lc, vj, bt);

    for (int64_t t = bos; t < eos; ++t) {
        float nk[R], nq[R], nl[R], nv[kCols], nb = 0.f;
        if (t + 1 < eos) load(t + 1, nk, nq, nl, nv, nb);

        // the prologue on this token's inputs (the next token's loads stay in flight)
        if (pro.flags & KDA_PROLOGUE_GATE_SOFTPLUS) {
#pragma unroll
            for (int m = 0; m < R; ++m) lc[m] = gate_from_raw(lc[m], pro.gate_scale);
        }
        if (pro.flags & KDA_PROLOGUE_BETA_SIGMOID) bt = beta_from_raw(bt);
        if (pro.flags & KDA_PROLOGUE_QK_L2NORM) {  // raw rows: x / sqrt(x.x + eps), lanes hold all d_k
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int m = 0; m < R; ++m) { sk = fmaf(kc[m], kc[m], sk); sq = fmaf(qc[m], qc[m], sq); }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
            }
            const float rk = rsqrtf(sk + kL2NormEps), rq = rsqrtf(sq + kL2NormEps);
#pragma unroll
            for (int m = 0; m < R; ++m) { kc[m] *= rk; qc[m] *= rq; }
        }
        float pa[kCols], pb[kCols], kq = 0.f;
#pragma unroll
        for (int j = 0; j < kCols; ++j) pa[j] = pb[j] = 0.f;
#pragma unroll
        for (int m = 0; m < R; ++m) {
            const float a = __expf(lc[m]);
            kq = fmaf(kc[m], qc[m], kq);
#pragma unroll
            for (int j = 0; j < kCols; ++j) {
                S[m][j] *= a;
                pa[j] = fmaf(S[m][j], kc[m], pa[j]);
                pb[j] = fmaf(S[m][j], qc[m], pb[j]);
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            kq += __shfl_xor_sync(0xffffffffu, kq, off);
#pragma unroll
            for (int j = 0; j < kCols; ++j) {
                pa[j] += __shfl_xor_sync(0xffffffffu, pa[j], off);
                pb[j] += __shfl_xor_sync(0xffffffffu, pb[j], off);
            }
        }
        float o_mine = 0.f;
#pragma unroll
        for (int j = 0; j < kCols; ++j) {
            const float u = bt * (vj[j] - pa[j]);
#pragma unroll
            for (int m = 0; m < R; ++m) S[m][j] = fmaf(kc[m], u, S[m][j]);
            const float o = fmaf(kq, u, pb[j]);
            if (lane == j) o_mine = o;
        }
        if (lane < kCols &&
            KDA_ACCESS_OK(ss.status, dbg.out, out + ((size_t)t * H + h) * dv + col0 + lane, sizeof(Tin), 43))
            out[((size_t)t * H + h) * dv + col0 + lane] = from_f32<Tin>(o_mine);

#pragma unroll
        for (int m = 0; m < R; ++m) { kc[m] = nk[m]; qc[m] = nq[m]; lc[m] = nl[m]; }
#pragma unroll
        for (int j = 0; j < kCols; ++j) vj[j] = nv[j];
        bt = nb;
    }
    float *dst = final_state_block(sT, n, H, h, (size_t)DK * dv, ss);
    if (dst && KDA_ACCESS_OK(ss.status, dbg.fin, dst, DK * dv * 4, 42)) {
#pragma unroll
        for (int m = 0; m < R; ++m)
#pragma unroll
            for (int j = 0; j < kCols; ++j)
                dst[(size_t)(lane + 32 * m) * dv + col0 + j] = S[m][j];
    }
}

template <typename Tin>
cudaError_t launch_typed(const Problem &p, cudaStream_t stream) {
    dim3 grid(p.num_seqs, p.H, p.dv / kSlice);
    auto args = [&](auto kern) {
        kern<<<grid, 128, 0, stream>>>((const Tin *)p.q, (const Tin *)p.k, (const Tin *)p.v,
                                       p.log_alpha, p.beta, p.initial_state, p.cu_seqlens, p.H,
                                       p.dv, (Tin *)p.out, p.final_state, p.slots, p.pro, p.dbg);
    };
    switch (p.dk) {
        case 32: args(recurrent_kernel<Tin, 32>); break;
        case 64: args(recurrent_kernel<Tin, 64>); break;
        case 128: args(recurrent_kernel<Tin, 128>); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_recurrent(const Problem &p, cudaStream_t stream) {
    if (p.num_seqs == 0) return cudaSuccess;
    return p.dtype == KDA_BF16 ? launch_typed<__nv_bfloat16>(p, stream)
                               : launch_typed<float>(p, stream);
}

}  // namespace kda
