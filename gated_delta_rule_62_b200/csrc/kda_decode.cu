// Fused KDA decode step: one token per (sequence, head), state updated in place.
//
// The per-token decode cost does not depend on how long the context is (the
// shivam2003.com Kimi K3 article, section "Kimi Delta Attention: the load-bearing
// choice"); the step is bound by streaming the fp32 state through HBM once in and
// once out. With S' = Diag(alpha) S:
//   a = S'^T k,  b = S'^T q,  u = beta (v - a),  S_new = S' + k u^T,
//   o = S_new^T q = b + (k.q) u,
// so one read of S feeds both column reductions and one write stores S_new.
//
// Mapping: one block per (sequence, head). A row of the state (d_v floats) is
// covered by d_v/4 threads with 16-byte loads, so each warp reads 512 contiguous
// bytes per instruction for d_v = 128; the other threads take further rows.
// Column sums over the key rows go through shared memory.
#include <type_traits>

#include "kda_internal.cuh"

namespace kda {
namespace {

// Value columns evolve independently, so d_v = 128 splits into two blocks of 64 columns (256
// threads: four blocks per SM in flight instead of two of 512); the row groups R, and with them
// the order of every sum, stay those of one 512-thread block over all columns.
template <int DK, int DV>
struct DecodeShape {
    static constexpr int SW = DV == 128 ? 64 : DV;               // value columns per block
    static constexpr int NSLICE = DV / SW;                       // blocks per head
    static constexpr int CG = SW / 4;                            // float4 column groups per row
    static constexpr int NTMAX = DV == 128 ? 256 : 512;
    static constexpr int NT = (CG * DK < NTMAX) ? CG * DK : NTMAX;  // threads per block
    static constexpr int R = NT / CG;                            // row groups
    static constexpr int RPT = DK / R;                           // rows per thread
    static_assert(NT % 32 == 0 && DK % R == 0 && DV % SW == 0, "bad decode shape");
};

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::NT)
decode_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
              const float *__restrict__ log_alpha, const float *__restrict__ beta,
              float *__restrict__ state, Tin *__restrict__ out, int H, const StateSlots ss,
              const DebugRanges dbg) {
    using Sh = DecodeShape<DK, DV>;
    constexpr int SW = Sh::SW, CG = Sh::CG, NT = Sh::NT, R = Sh::R, RPT = Sh::RPT;
    __shared__ float s_k[DK], s_q[DK], s_a[DK];
    __shared__ __align__(16) float s_red[2][R][SW];
    __shared__ __align__(16) float s_u[SW];
    __shared__ float s_kq;

    const size_t head = blockIdx.x;  // n * H + h
    const int col0 = blockIdx.y * SW;  // this block's value columns
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    // Launched with programmatic stream serialization: the next decode step's blocks may become
    // resident while this grid drains, and this grid's while the previous one drains. Nothing is
    // read before the wait, which returns once the previous kernel in the stream has completed
    // and its writes are visible (without that launch attribute both are no-ops).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // this head's state: entry `head`, or its sequence's slot of the pool (none: zeros, not stored)
    float *blk = final_state_block(state, (int)(head / H), H, (int)(head % H), (size_t)(DK * DV), ss);
    if (blk && !KDA_ACCESS_OK(ss.status, dbg.fin, blk, DK * DV * 4, 31)) blk = nullptr;
    float4 *S4 = blk ? reinterpret_cast<float4 *>(blk + col0) : nullptr;

    // Issue the state loads first: they are the only long-latency traffic.
    float4 s[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i)
        s[i] = S4 ? __ldcs(&S4[(size_t)(rg + i * R) * (DV / 4) + cg]) : make_float4(0.f, 0.f, 0.f, 0.f);

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

    if (tid < SW) {
        float a = 0.f, b = 0.f;
#pragma unroll 8
        for (int r = 0; r < R; ++r) { a += s_red[0][r][tid]; b += s_red[1][r][tid]; }
        const size_t o = head * DV + col0 + tid;
        const float u = beta[head] * (to_f32(v[o]) - a);
        s_u[tid] = u;
        if (KDA_ACCESS_OK(ss.status, dbg.out, out + o, sizeof(Tin), 32)) out[o] = from_f32<Tin>(fmaf(s_kq, u, b));
    }
    __syncthreads();

    const float4 u4 = reinterpret_cast<const float4 *>(s_u)[cg];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float kc = s_k[rg + i * R];
        s[i].x = fmaf(kc, u4.x, s[i].x); s[i].y = fmaf(kc, u4.y, s[i].y);
        s[i].z = fmaf(kc, u4.z, s[i].z); s[i].w = fmaf(kc, u4.w, s[i].w);
        if (S4) __stcs(&S4[(size_t)(rg + i * R) * (DV / 4) + cg], s[i]);
    }
}

// ---- speculative (multi-token) decode ----------------------------------------------------
// The draft model proposes T tokens per sequence and the main model checks them in one pass
// ("Optimization for Inference: 4-Bit and Speculative Decoding" in the Kimi K3 article). The
// verify kernel reads each state once for all T tokens and leaves it unchanged; per token it
// keeps the correction u_t = beta_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t), with which
//   S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T,
// so the commit kernel advances a state by any accepted prefix without its v, q or beta.
// Both use the decode mapping and arithmetic above, token by token: the outputs and the
// committed states equal those of T (resp. the accepted number of) decode steps bit for bit.
// The verify kernel gives each block one slice of at most 32 value columns of a head (grid y),
// with the decode kernel's row groups: each column's sums run over the same rows in the same
// order, and small blocks (128 threads for d_v = 128) let several heads' token loops overlap
// on one SM while others wait for their states.
// WIDE (the commit-only launch, which has no sums over rows): the decode kernel's column blocks,
// whose rows a warp reads in longer pieces.
template <int DK, int DV, bool WIDE = false>
struct VerifyShape {
    static constexpr int SW = WIDE ? DecodeShape<DK, DV>::SW : (DV < 32 ? DV : 32);  // value columns per block
    static constexpr int NSLICE = DV / SW;
    static constexpr int CG = SW / 4;                  // float4 column groups per row
    static constexpr int R = DecodeShape<DK, DV>::R;   // row groups, as in the decode kernel
    static constexpr int NT = CG * R;
    static constexpr int RPT = DK / R;
    static_assert(NT % 32 == 0 && NT <= 1024, "bad verify shape");
};

// Shared memory of one block, in floats: the draft's k, q, alpha [T][DK] as duplicated pairs
// (x, x), v [T][SW] and beta [T, padded to 4] (verify); then the accepted tokens' k, alpha
// [T_prev][DK] as pairs and u [T_prev][SW] (commit). Every region starts on a 16-byte boundary.
// The pairs feed the paired fp32 instructions (two columns of the state per instruction), whose
// lanes round exactly as the scalar ones: results stay those of the decode kernel, bit for bit.
template <int DK, int DV, bool WIDE = false>
struct SpecSmem {
    static constexpr int SW = VerifyShape<DK, DV, WIDE>::SW;
    int k, q, a, v, b, ck, ca, cu, total;
    __host__ __device__ constexpr SpecSmem(int T, int TP)
        : k(0), q(2 * T * DK), a(4 * T * DK), v(6 * T * DK), b(6 * T * DK + T * SW),
          ck(b + ((T + 3) & ~3)), ca(ck + 2 * TP * DK), cu(ca + 2 * TP * DK), total(cu + TP * SW) {}
};
static_assert(SpecSmem<32, 32>(3, 5).cu % 4 == 0 && SpecSmem<128, 128>(1, 16).cu % 4 == 0 &&
              SpecSmem<64, 64>(7, 3).cu % 4 == 0, "u rows must be 16-byte aligned");

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {  // bf16 -> fp32 is exact: a shift
    const uint2 r = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u),
                       __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
}
// (x, y, z, w) -> pairs (x, x), (y, y), (z, z), (w, w) at dst[0..3]
__device__ __forceinline__ void st_dup4(float2 *dst, float4 x) {
    reinterpret_cast<float4 *>(dst)[0] = make_float4(x.x, x.x, x.y, x.y);
    reinterpret_cast<float4 *>(dst)[1] = make_float4(x.z, x.z, x.w, x.w);
}
__device__ __forceinline__ float4 exp4(float4 x) {
    return make_float4(__expf(x.x), __expf(x.y), __expf(x.z), __expf(x.w));
}

// COMMIT: advance the state by accepted[n] tokens of the previous draft (k, alpha, u) and store
// it; VERIFY: run the T draft tokens from the (advanced) state, writing out and u_cache.
template <typename Tin, int DK, int DV, bool COMMIT, bool VERIFY>
__global__ void __launch_bounds__(VerifyShape<DK, DV, COMMIT && !VERIFY>::NT) spec_kernel(const VerifyProblem p) {
    using Sh = VerifyShape<DK, DV, COMMIT && !VERIFY>;
    constexpr int SW = Sh::SW, CG = Sh::CG, NT = Sh::NT, R = Sh::R, RPT = Sh::RPT;
    extern __shared__ __align__(16) float s_in[];
    __shared__ __align__(16) float2 s_red[R][SW];  // (S'^T k, S'^T q) partials per row group
    __shared__ __align__(16) float s_u[SW];
    __shared__ float s_kq;
    const int T = VERIFY ? p.T : 0, TP = COMMIT ? p.T_prev : 0, H = p.H;
    const SpecSmem<DK, DV, COMMIT && !VERIFY> L(T, TP);
    float2 *s_k = reinterpret_cast<float2 *>(s_in + L.k), *s_q = reinterpret_cast<float2 *>(s_in + L.q),
           *s_a = reinterpret_cast<float2 *>(s_in + L.a);
    float *s_v = s_in + L.v, *s_b = s_in + L.b, *c_u = s_in + L.cu;
    float2 *c_k = reinterpret_cast<float2 *>(s_in + L.ck), *c_a = reinterpret_cast<float2 *>(s_in + L.ca);

    const int n = blockIdx.x / H, h = blockIdx.x % H, col0 = blockIdx.y * SW;
    const int tid = threadIdx.x;
    const int cg = tid % CG, rg = tid / CG;
    // the slot table (if any) names the state both read and written
    float *blk = final_state_block(p.state, n, H, h, (size_t)(DK * DV), p.slots);
    int acc = 0;
    if (COMMIT && blk) {
        acc = p.accepted[n];
        if (acc < 0 || acc > TP) {
            if (tid == 0 && h == 0 && blockIdx.y == 0 && p.slots.status)
                atomicOr(p.slots.status, kStatusBadAccept);
            acc = 0;
        }
    }
    if (!VERIFY && acc == 0) return;  // commit only, nothing accepted: the state stays as it is
    float4 *S4 = blk ? reinterpret_cast<float4 *>(blk + col0) : nullptr;

    // state columns 4cg..4cg+3 of rows rg + i*R, as pairs (4cg, 4cg+1), (4cg+2, 4cg+3)
    float2 s[2 * RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const float4 x = S4 ? __ldcs(&S4[(size_t)(rg + i * R) * (DV / 4) + cg]) : make_float4(0.f, 0.f, 0.f, 0.f);
        s[2 * i] = make_float2(x.x, x.y);
        s[2 * i + 1] = make_float2(x.z, x.w);
    }

    // Inputs staged once, four elements per thread and load: token t of sequence n is row
    // n*T + t (n*T_prev + t for the commit). Each thread issues a group's loads before any of
    // its stores, so their latencies overlap.
    const size_t row0 = (size_t)n * T, prow0 = (size_t)n * TP;
    constexpr int G = 1;
    if (VERIFY) {
        const Tin *q = (const Tin *)p.q, *k = (const Tin *)p.k, *v = (const Tin *)p.v;
        for (int i0 = 4 * tid; i0 < T * DK; i0 += 4 * G * NT) {
            float4 kk[G], qq[G], ll[G];
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const int i = i0 + 4 * j * NT;
                if (i < T * DK) {
                    const size_t g = ((row0 + i / DK) * H + h) * DK + i % DK;
                    kk[j] = ld4(k + g); qq[j] = ld4(q + g); ll[j] = ld4(p.log_alpha + g);
                }
            }
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const int i = i0 + 4 * j * NT;
                if (i < T * DK) { st_dup4(s_k + i, kk[j]); st_dup4(s_q + i, qq[j]); st_dup4(s_a + i, exp4(ll[j])); }
            }
        }
        for (int i = 4 * tid; i < T * SW; i += 4 * NT)
            *reinterpret_cast<float4 *>(s_v + i) = ld4(v + ((row0 + i / SW) * H + h) * DV + col0 + i % SW);
        for (int i = tid; i < T; i += NT) s_b[i] = p.beta[(row0 + i) * H + h];
    }
    if (COMMIT) {
        const Tin *pk = (const Tin *)p.prev_k;
        for (int i0 = 4 * tid; i0 < acc * DK; i0 += 4 * G * NT) {
            float4 kk[G], ll[G];
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const int i = i0 + 4 * j * NT;
                if (i < acc * DK) {
                    const size_t g = ((prow0 + i / DK) * H + h) * DK + i % DK;
                    kk[j] = ld4(pk + g); ll[j] = ld4(p.prev_log_alpha + g);
                }
            }
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const int i = i0 + 4 * j * NT;
                if (i < acc * DK) { st_dup4(c_k + i, kk[j]); st_dup4(c_a + i, exp4(ll[j])); }
            }
        }
        for (int i = 4 * tid; i < acc * SW; i += 4 * NT)
            *reinterpret_cast<float4 *>(c_u + i) = ld4(p.prev_u + ((prow0 + i / SW) * H + h) * DV + col0 + i % SW);
    }
    __syncthreads();

    if (COMMIT && acc > 0) {
        // S_t = Diag(alpha_t) S_{t-1} + k_t u_t^T, the decode step's own two roundings
        for (int t = 0; t < acc; ++t) {
            const float4 u4 = reinterpret_cast<const float4 *>(c_u + t * SW)[cg];
            const float2 u01 = make_float2(u4.x, u4.y), u23 = make_float2(u4.z, u4.w);
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const int c = rg + i * R;
                const float2 al = c_a[t * DK + c], kc = c_k[t * DK + c];
                s[2 * i] = __ffma2_rn(kc, u01, __fmul2_rn(s[2 * i], al));
                s[2 * i + 1] = __ffma2_rn(kc, u23, __fmul2_rn(s[2 * i + 1], al));
            }
        }
#pragma unroll
        for (int i = 0; i < RPT; ++i)
            __stcs(&S4[(size_t)(rg + i * R) * (DV / 4) + cg],
                   make_float4(s[2 * i].x, s[2 * i].y, s[2 * i + 1].x, s[2 * i + 1].y));
    }
    if (!VERIFY) return;

    Tin *out = (Tin *)p.out;
    for (int t = 0; t < T; ++t) {
        const float2 *tk = s_k + t * DK, *tq = s_q + t * DK, *ta = s_a + t * DK;
        float2 pa0 = make_float2(0.f, 0.f), pa1 = pa0, pb0 = pa0, pb1 = pa0;
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int c = rg + i * R;
            const float2 al = ta[c], kc = tk[c], qc = tq[c];
            s[2 * i] = __fmul2_rn(s[2 * i], al);
            s[2 * i + 1] = __fmul2_rn(s[2 * i + 1], al);
            pa0 = __ffma2_rn(s[2 * i], kc, pa0); pa1 = __ffma2_rn(s[2 * i + 1], kc, pa1);
            pb0 = __ffma2_rn(s[2 * i], qc, pb0); pb1 = __ffma2_rn(s[2 * i + 1], qc, pb1);
        }
        float4 *red = reinterpret_cast<float4 *>(&s_red[rg][4 * cg]);
        red[0] = make_float4(pa0.x, pb0.x, pa0.y, pb0.y);
        red[1] = make_float4(pa1.x, pb1.x, pa1.y, pb1.y);
        if (tid < 32) {
            float kq = 0.f;
            for (int c = tid; c < DK; c += 32) kq = fmaf(tk[c].x, tq[c].x, kq);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
            if (tid == 0) s_kq = kq;
        }
        __syncthreads();

        if (tid < SW) {
            float2 ab = make_float2(0.f, 0.f);  // (S'^T k, S'^T q) for this column
#pragma unroll 8
            for (int r = 0; r < R; ++r) ab = __fadd2_rn(ab, s_red[r][tid]);
            const float u = s_b[t] * (s_v[t * SW + tid] - ab.x);
            s_u[tid] = u;
            const size_t o = ((row0 + t) * H + h) * DV + col0 + tid;
            out[o] = from_f32<Tin>(fmaf(s_kq, u, ab.y));
            p.u_cache[o] = u;
        }
        __syncthreads();
        // s_red, s_u and s_kq are next written after the next token's first barrier (s_u) or
        // after this one (s_red, s_kq, whose readers all passed it): two barriers suffice.
        const float4 u4 = reinterpret_cast<const float4 *>(s_u)[cg];
        const float2 u01 = make_float2(u4.x, u4.y), u23 = make_float2(u4.z, u4.w);
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const float2 kc = tk[rg + i * R];
            s[2 * i] = __ffma2_rn(kc, u01, s[2 * i]);
            s[2 * i + 1] = __ffma2_rn(kc, u23, s[2 * i + 1]);
        }
    }
}

template <typename Tin, int DK, int DV, bool COMMIT, bool VERIFY>
cudaError_t launch_spec(const VerifyProblem &p, cudaStream_t stream) {
    using VS = VerifyShape<DK, DV, COMMIT && !VERIFY>;
    auto kern = spec_kernel<Tin, DK, DV, COMMIT, VERIFY>;
    const SpecSmem<DK, DV, COMMIT && !VERIFY> L(VERIFY ? p.T : 0, COMMIT ? p.T_prev : 0);
    if (L.cu % 4 != 0) return cudaErrorInvalidValue;  // float4 reads of the u rows
    const size_t smem = (size_t)L.total * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<dim3((unsigned)p.num_seqs * (unsigned)p.H, VS::NSLICE), VS::NT, smem, stream>>>(p);
    return cudaGetLastError();
}

template <typename Tin, int DK, int DV>
cudaError_t launch_verify3(const VerifyProblem &p, cudaStream_t stream) {
    const bool commit = p.accepted != nullptr, verify = p.q != nullptr;
    if (commit && verify) return launch_spec<Tin, DK, DV, true, true>(p, stream);
    if (commit) return launch_spec<Tin, DK, DV, true, false>(p, stream);
    return launch_spec<Tin, DK, DV, false, true>(p, stream);
}

template <typename Tin, int DK, int DV>
cudaError_t launch3(const DecodeProblem &p, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.num_seqs * (unsigned)p.H, DecodeShape<DK, DV>::NSLICE);
    cfg.blockDim = dim3(DecodeShape<DK, DV>::NT);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<Tin, DK, DV>, (const Tin *)p.q, (const Tin *)p.k,
                              (const Tin *)p.v, p.log_alpha, p.beta, p.state, (Tin *)p.out, p.H, p.slots,
                              p.dbg);
}

template <template <typename, int, int> class L, typename P>
cudaError_t dispatch(const P &p, cudaStream_t stream) {
    auto by_dv = [&](auto tin, auto dk) -> cudaError_t {
        using Tin = decltype(tin);
        constexpr int DK = decltype(dk)::value;
        switch (p.dv) {
            case 32: return L<Tin, DK, 32>::run(p, stream);
            case 64: return L<Tin, DK, 64>::run(p, stream);
            case 128: return L<Tin, DK, 128>::run(p, stream);
        }
        return cudaErrorInvalidValue;
    };
    auto by_dk = [&](auto tin) -> cudaError_t {
        switch (p.dk) {
            case 32: return by_dv(tin, std::integral_constant<int, 32>{});
            case 64: return by_dv(tin, std::integral_constant<int, 64>{});
            case 128: return by_dv(tin, std::integral_constant<int, 128>{});
        }
        return cudaErrorInvalidValue;
    };
    return p.dtype == KDA_BF16 ? by_dk(__nv_bfloat16{}) : by_dk(float{});
}

template <typename Tin, int DK, int DV> struct DecodeLaunch {
    static cudaError_t run(const DecodeProblem &p, cudaStream_t s) { return launch3<Tin, DK, DV>(p, s); }
};
template <typename Tin, int DK, int DV> struct VerifyLaunch {
    static cudaError_t run(const VerifyProblem &p, cudaStream_t s) {
        return launch_verify3<Tin, DK, DV>(p, s);
    }
};

}  // namespace

cudaError_t launch_decode(const DecodeProblem &p, cudaStream_t stream) {
    if (p.num_seqs == 0) return cudaSuccess;
    return dispatch<DecodeLaunch>(p, stream);
}

cudaError_t launch_verify(const VerifyProblem &p, cudaStream_t stream) {
    if (p.num_seqs == 0) return cudaSuccess;
    return dispatch<VerifyLaunch>(p, stream);
}

}  // namespace kda
