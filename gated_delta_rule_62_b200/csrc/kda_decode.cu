// Fused KDA decode step: one token per (sequence, head), state updated in place.
//
// The per-token cost is constant ("Decoding throughput stays roughly flat as
// context grows": shivam2003.com Kimi K3 article, section "Kimi Delta Attention:
// the load-bearing choice"); the step is bound by streaming the fp32 state
// through HBM once in and once out. With S' = Diag(alpha) S:
//   a = S'^T k,  b = S'^T q,  u = beta (v - a),  S_new = S' + k u^T,
//   o = S_new^T q = b + (k.q) u,
// so one read of S feeds both column reductions and one write stores S_new.
//
// Mapping: one block per (sequence, head). A row of the state (d_v floats) is
// covered by d_v/4 threads with 16-byte loads, so each warp reads 512 contiguous
// bytes per instruction for d_v = 128; the other threads take further rows.
// Column sums over the key rows go through shared memory.
#include "kda_internal.cuh"

namespace kda {
namespace {

template <int DK, int DV>
struct DecodeShape {
    static constexpr int CG = DV / 4;                            // float4 column groups per row
    static constexpr int NT = (CG * DK < 512) ? CG * DK : 512;   // threads per block
    static constexpr int R = NT / CG;                            // row groups
    static constexpr int RPT = DK / R;                           // rows per thread
    static_assert(NT % 32 == 0 && DK % R == 0, "bad decode shape");
};

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::NT)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ log_alpha, const float *__restrict__ beta,
              float *__restrict__ state, Tin *__restrict__ out, int H, const StateSlots ss) {
    using Sh = DecodeShape<DK, DV>;
    constexpr int CG = Sh::CG, NT = Sh::NT, R = Sh::R, RPT = Sh::RPT;
    __shared__ float s_k[DK], s_q[DK], s_a[DK];
    __shared__ __align__(16) float s_red[2][R][DV];
    __shared__ __align__(16) float s_u[DV];
    __shared__ float s_kq;

    const size_t head = blockIdx.x;  // n * H + h
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    // this head's state: entry `head`, or its sequence's slot of the pool (none: zeros, not stored)
    float *blk = final_state_block(state, (int)(head / H), H, (int)(head % H), (size_t)(DK * DV), ss);
    float4 *S4 = reinterpret_cast<float4 *>(blk);

    // Issue the state loads first: they are the only long-latency traffic.
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        s[i] = blk ? __ldcs(&S4[(size_t)(rg + i * R) * CG + cg]) : make_float4(0.f, 0.f, 0.f, 0.f);

    for (int c = tid; c < DK; c += NT) {
        s_k[c] = to_f32(k[head * DK + c]);
        s_q[c] = to_f32(q[head * DK + c]);
        s_a[c] = __expf(log_alpha[head * DK + c]);
    }
    __syncthreads();

    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = pa;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int c = rg + i * R;
        const float al = s_a[c], kc = s_k[c], qc = s_q[c];
        s[i].x *= al; s[i].y *= al; s[i].z *= al; s[i].w *= al;
        pa.x = fmaf(s[i].x, kc, pa.x); pa.y = fmaf(s[i].y, kc, pa.y);
        pa.z = fmaf(s[i].z, kc, pa.z); pa.w = fmaf(s[i].w, kc, pa.w);
        pb.x = fmaf(s[i].x, qc, pb.x); pb.y = fmaf(s[i].y, qc, pb.y);
        pb.z = fmaf(s[i].z, qc, pb.z); pb.w = fmaf(s[i].w, qc, pb.w);
    }
    reinterpret_cast<float4 *>(&s_red[0][rg][0])[cg] = pa;
    reinterpret_cast<float4 *>(&s_red[1][rg][0])[cg] = pb;
    if (tid < 32) {  // k.q by the first warp
        float kq = 0.f;
        for (int c = tid; c < DK; c += 32) kq = fmaf(s_k[c], s_q[c], kq);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
        if (tid == 0) s_kq = kq;
    }
    __syncthreads();

    if (tid < DV) {
        float a = 0.f, b = 0.f;
#pragma unroll 8
        for (int r = 0; r < R; ++r) { a += s_red[0][r][tid]; b += s_red[1][r][tid]; }
        const float u = beta[head] * (to_f32(v[head * DV + tid]) - a);
        s_u[tid] = u;
        out[head * DV + tid] = from_f32<Tin>(fmaf(s_kq, u, b));
    }
    __syncthreads();

    const float4 u4 = reinterpret_cast<const float4 *>(s_u)[cg];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float kc = s_k[rg + i * R];
        s[i].x = fmaf(kc, u4.x, s[i].x); s[i].y = fmaf(kc, u4.y, s[i].y);
        s[i].z = fmaf(kc, u4.z, s[i].z); s[i].w = fmaf(kc, u4.w, s[i].w);
        if (blk) __stcs(&S4[(size_t)(rg + i * R) * CG + cg], s[i]);
    }
}

template <typename Tin, int DK, int DV>
cudaError_t launch3(const DecodeProblem &p, cudaStream_t stream) {
    const unsigned blocks = (unsigned)p.num_seqs * (unsigned)p.H;
    decode_kernel<Tin, DK, DV><<<blocks, DecodeShape<DK, DV>::NT, 0, stream>>>(
        (const Tin *)p.q, (const Tin *)p.k, (const Tin *)p.v, p.log_alpha, p.beta, p.state,
        (Tin *)p.out, p.H, p.slots);
    return cudaGetLastError();
}

template <typename Tin, int DK>
cudaError_t launch2(const DecodeProblem &p, cudaStream_t stream) {
    switch (p.dv) {
        case 32: return launch3<Tin, DK, 32>(p, stream);
        case 64: return launch3<Tin, DK, 64>(p, stream);
        case 128: return launch3<Tin, DK, 128>(p, stream);
    }
    return cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t launch1(const DecodeProblem &p, cudaStream_t stream) {
    switch (p.dk) {
        case 32: return launch2<Tin, 32>(p, stream);
        case 64: return launch2<Tin, 64>(p, stream);
        case 128: return launch2<Tin, 128>(p, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const DecodeProblem &p, cudaStream_t stream) {
    if (p.num_seqs == 0) return cudaSuccess;
    return p.dtype == KDA_BF16 ? launch1<__nv_bfloat16>(p, stream) : launch1<float>(p, stream);
}

}  // namespace kda
