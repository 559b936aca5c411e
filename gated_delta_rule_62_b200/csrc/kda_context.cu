// Context parallelism inside one GPU: a long sequence with few heads is cut into segments whose
// state chains run side by side.
//
// The per-chunk state map is affine, S_{j+1} = F_j S_j + K^_j^T U~_j with F_j = diag(gamma) -
// K^_j^T W_j, so a segment's end state is F_seg S_start + S0_end, where S0 is the segment's chain
// from a zero state and F_seg the product of its chunks' F. The pages say the KDA update is
// computed blockwise and context-parallel ("Kimi Delta Attention: the load-bearing choice" in the
// shivam2003.com Kimi K3 article); this is that idea at the level of chunk segments:
//
//   1. plan kernel: the segment table (each segment is a chain of its own in the split kernel);
//   2. split kernel: the first segment of a sequence runs from its initial state as usual; a later
//      segment's consumer runs S0 and the transition product R from I, writes its zero-start
//      outputs O0 and per chunk E = P R (see consumer_seg in kda_chunk_split.cu);
//   3. scan kernel (fp32): S_start(g + 1) = F_g S_start(g) + S0_end(g) along each sequence's
//      segments, which also gives the sequence's final state; each S_start goes out as a bf16 tile;
//   4. fix-up kernel (tcgen05): O_j += E_j S_start(g) for every chunk of the later segments.
//
// Workspace after the split kernel's own: the segment table, the chains' end states and
// transition products (fp32), the start-state tiles and the E tiles (bf16, 16 KB per chunk-head).
#include <cuda.h>

#include "kda_chunk_common.cuh"

namespace kda {
namespace {

using namespace sm100;
using namespace chunk;

size_t round1k(size_t x) { return (x + 1023) / 1024 * 1024; }

// ---------------------------------------------------------------- 1. plan
// One thread: the same segmentation the host planned (seg_count / seg_chunk_begin), as device tables.
__global__ void seg_plan_kernel(const int32_t *__restrict__ cu, int32_t N, int32_t segments,
                                int32_t *__restrict__ vcu, int4 *__restrict__ vinfo,
                                int32_t *__restrict__ vfirst) {
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    int v = 0, e_off = 0;
    for (int n = 0; n < N; ++n) {
        const int32_t bos = cu[n], len = cu[n + 1] - cu[n];
        const int chunks = (len + C - 1) / C;
        const int G = seg_count(chunks, segments);
        vfirst[n] = v;
        for (int g = 0; g < G; ++g, ++v) {
            const int cb = seg_chunk_begin(chunks, G, g), ce = seg_chunk_begin(chunks, G, g + 1);
            const int32_t off = (int32_t)C * cb;
            vcu[v] = bos + (off < len ? off : len);
            vinfo[v] = make_int4(n, g, G, e_off);
            if (g >= 1) e_off += ce - cb;
        }
    }
    vcu[v] = cu[N];
}

// ---------------------------------------------------------------- 3. scan
// One block of 256 threads per (sequence with several segments, head). S (the running true state,
// [c][d]) and F (the next segment's transition, [c][a]) in shared memory; thread t computes rows
// [64 (t / 128), +64) of column d = t % 128 of S_new = F S + S0.
constexpr int SCAN_THREADS = 256;
constexpr uint32_t SCAN_SMEM = 2u * D * D * 4u;

__global__ void __launch_bounds__(SCAN_THREADS)
seg_scan_kernel(const int4 *__restrict__ vinfo, const int32_t *__restrict__ vfirst, int32_t N,
                int32_t H, const float *__restrict__ seg_state, const float *__restrict__ seg_trans,
                uint8_t *__restrict__ s_start, float *final_state, StateSlots ss, int32_t *status,
                DebugRanges dbg) {
    extern __shared__ float scan_sm[];
    float *S = scan_sm, *F = scan_sm + D * D;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    if (n >= N) return;
    const int v0 = vfirst[n];
    const int G = vinfo[v0].z;
    if (G < 2) return;  // a single chain wrote the final state itself
    const int tid = threadIdx.x, d = tid & (D - 1), r0 = 64 * (tid >> 7);
    const float4 *src = reinterpret_cast<const float4 *>(seg_state + ((size_t)v0 * H + h) * D * D);
    const bool src_ok = KDA_ACCESS_OK(status, dbg.ws, src, D * D * 4, 26);
    for (int i = tid; i < D * D / 4; i += SCAN_THREADS)
        reinterpret_cast<float4 *>(S)[i] = src_ok ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();
    for (int g = 1; g < G; ++g) {
        const size_t vh = (size_t)(v0 + g) * H + h;
        // the start state of segment g as the fix-up's A operand: S_start^T [d][a], K-major,
        // 128-byte swizzled, two 64-column blocks of 16 KB; thread: row d, columns [r0, r0 + 64)
        uint8_t *tile = s_start + vh * kSegStartTileBytes;
        const bool ok = KDA_ACCESS_OK(status, dbg.ws, tile, kSegStartTileBytes, 24) &&
                        KDA_ACCESS_OK(status, dbg.ws, seg_trans + vh * D * D, D * D * 4, 27) &&
                        KDA_ACCESS_OK(status, dbg.ws, seg_state + vh * D * D, D * D * 4, 28);
        if (!ok) break;
        for (int a8 = 0; a8 < 64; a8 += 8) {
            float x[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) x[e] = S[(r0 + a8 + e) * D + d];
            st_chunk(tile + tchunk(16384, d, r0 + a8), x);
        }
        const float4 *fsrc = reinterpret_cast<const float4 *>(seg_trans + vh * D * D);
        for (int i = tid; i < D * D / 4; i += SCAN_THREADS) reinterpret_cast<float4 *>(F)[i] = fsrc[i];
        __syncthreads();
        const float *s0 = seg_state + vh * D * D;
        float acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = s0[(size_t)(r0 + i) * D + d];
        for (int a = 0; a < D; a += 4) {
            const float sa0 = S[(a + 0) * D + d], sa1 = S[(a + 1) * D + d];
            const float sa2 = S[(a + 2) * D + d], sa3 = S[(a + 3) * D + d];
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float4 f = *reinterpret_cast<const float4 *>(F + (r0 + i) * D + a);
                acc[i] = fmaf(f.x, sa0, fmaf(f.y, sa1, fmaf(f.z, sa2, fmaf(f.w, sa3, acc[i]))));
            }
        }
        __syncthreads();  // every thread has read S and F
#pragma unroll
        for (int i = 0; i < 64; ++i) S[(r0 + i) * D + d] = acc[i];
        __syncthreads();
    }
    float *fs = final_state_block(final_state, n, H, h, (size_t)D * D, ss);
    if (fs && KDA_ACCESS_OK(status, dbg.fin, fs, D * D * 4, 25))
        for (int i = tid; i < D * D / 4; i += SCAN_THREADS)
            reinterpret_cast<float4 *>(fs)[i] = reinterpret_cast<const float4 *>(S)[i];
}

// ---------------------------------------------------------------- 4. fix-up
// One block of 128 threads per (later segment, head, range of FIX_CHUNKS chunks). The start state
// S_start^T is the A operand (K-major, [d][a]); per chunk the E^T tile (MN-major B, [a][i]) is
// brought in with a bulk copy (double-buffered) and D^T = S_start^T E^T (M = 128 value channels,
// N = 64 tokens, K = 128) lands in TMEM; thread d adds row d of D^T to its channel of the chunk's
// outputs.
constexpr int FIX_THREADS = 128;
constexpr int FIX_CHUNKS = 64;
constexpr uint32_t FIX_A = 0, FIX_E0 = 32768, FIX_E1 = 49152, FIX_MISC = 65536;
constexpr uint32_t FIX_SMEM = FIX_MISC + 128 + 1024;

struct FixParams {
    const int32_t *vcu;
    const int4 *vinfo;
    const uint8_t *s_start, *e_tiles;
    const int32_t *e_live;
    __nv_bfloat16 *out;
    int32_t *status;
    int32_t H, num_vseqs, ranges;  // ranges: chunk ranges per (segment, head) in the grid
    uint64_t timeout_ns;
    DebugRanges dbg;               // buffer ranges (checked by debug builds only)
};

__global__ void __launch_bounds__(FIX_THREADS)
seg_fixup_kernel(const FixParams p) {
    extern __shared__ uint8_t fix_raw[];
    uint8_t *sm = fix_raw + ((1024u - (smem_u32(fix_raw) & 1023u)) & 1023u);
    const int H = p.H;
    const int vh = blockIdx.x / p.ranges, r = blockIdx.x % p.ranges;
    const int v = vh / H, h = vh % H;
    if (v >= p.num_vseqs) return;
    const int4 vi = p.vinfo[v];
    const int64_t bos = p.vcu[v], eos = p.vcu[v + 1];
    if (vi.y < 1) return;  // a first segment: its outputs are final
    // chunks whose E tile is live (the segment's transition product had not decayed away)
    const int live = min((int)((eos - bos + C - 1) / C), p.e_live[(size_t)v * H + h]);
    const int c0 = r * FIX_CHUNKS, c1 = min(live, c0 + FIX_CHUNKS);
    if (c0 >= c1) return;  // the block's whole range is empty: nothing allocated yet

    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + FIX_MISC);  // a, e0, e1, mma
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + FIX_MISC + 64);
    const int tid = threadIdx.x, warp = tid >> 5;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    constexpr uint32_t I_F = idesc_bf16_f32(128, 64, false, 0, 1);
    const uint8_t *e_base = p.e_tiles + ((size_t)vi.w * H + h) * kSegETileBytes;  // chunk c: + c H tiles
    auto e_tile = [&](int c) { return e_base + (size_t)c * H * kSegETileBytes; };
    // debug builds: the block's whole range of E tiles and its start tile lie in the workspace
    if (!KDA_ACCESS_OK(p.status, p.dbg.ws, e_tile(c0), kSegETileBytes, 22) ||
        !KDA_ACCESS_OK(p.status, p.dbg.ws, e_tile(c1 - 1), kSegETileBytes, 22) ||
        !KDA_ACCESS_OK(p.status, p.dbg.ws, p.s_start + ((size_t)v * H + h) * kSegStartTileBytes,
                       kSegStartTileBytes, 23))
        return;

    if (tid == 0) {
        for (int k = 0; k < 4; ++k) mbar_init(&bars[k], 1);
        fence_mbarrier_init();
    }
    if (warp == 0) {
        tmem_alloc(s_tmem, 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    // thread 0 owns the copies: bit k of `pending` is set while copy k (0: A, 1 / 2: E stages) may
    // be in flight. E stage s serves chunks c with (c - c0) % 2 == s, use (c - c0) / 2.
    bool ok = true;
    uint32_t pending = 0;
    if (tid == 0) {
        mbar_arrive_expect_tx(&bars[0], kSegStartTileBytes);
        bulk_load(sm + FIX_A, p.s_start + ((size_t)v * H + h) * kSegStartTileBytes, kSegStartTileBytes, &bars[0]);
        pending = 1u;
        for (int k = 0; k < 2 && c0 + k < c1; ++k) {
            mbar_arrive_expect_tx(&bars[1 + k], kSegETileBytes);
            bulk_load(sm + (k ? FIX_E1 : FIX_E0), e_tile(c0 + k), kSegETileBytes, &bars[1 + k]);
            pending |= 2u << k;
        }
        ok = mbar_wait_bounded(&bars[0], 0, p.timeout_ns);
        if (ok) pending &= ~1u;
    }
    uint32_t ph_mma = 0;
    const uint32_t sb = smem_u32(sm);
    const int d = tid;
    int brk = -1;  // the chunk the loop broke off at (its copy and the next one may be in flight)
    for (int c = c0; c < c1; ++c) {
        const int s = (c - c0) & 1;
        if (tid == 0) {
            if (ok) {
                ok = mbar_wait_bounded(&bars[1 + s], (uint32_t)((c - c0) >> 1) & 1u, p.timeout_ns);
                if (ok) pending &= ~(2u << s);
            }
            if (ok) {
                tc_fence_after();
                const uint64_t dA = desc_k(sb + FIX_A, 16384, 0);
                const uint64_t dE = desc_mn(sb + (s ? FIX_E1 : FIX_E0), 8192, 0);
#pragma unroll
                for (uint32_t kk = 0; kk < 8; ++kk)
                    mma_bf16_ss(tmem, desc_k_at(dA, 16384, kk), desc_mn_at(dE, kk), I_F, kk > 0);
            }
            mma_commit(&bars[3]);  // arrives once the MMAs above (if any) have completed
        }
        const bool done = mbar_wait_bounded(&bars[3], ph_mma, p.timeout_ns);
        ph_mma ^= 1u;
        if (__syncthreads_or(!done || (tid == 0 && !ok))) {
            if (tid == 0) atomicOr(p.status, 1);
            brk = c;
            break;
        }
        tc_fence_after();
        if (tid == 0 && c + 2 < c1) {  // stage s is free: the MMA that read it has completed
            mbar_arrive_expect_tx(&bars[1 + s], kSegETileBytes);
            bulk_load(sm + (s ? FIX_E1 : FIX_E0), e_tile(c + 2), kSegETileBytes, &bars[1 + s]);
            pending |= 2u << s;
        }
        float x[2][32];
        tmem_ld32(tmem + lane_base, x[0]);
        tmem_ld32(tmem + lane_base + 32, x[1]);
        tmem_wait_ld();
        tc_fence_before();
        const int64_t tc = bos + (int64_t)c * C;
        const int vc = (int)(eos - tc < C ? eos - tc : C);
        __nv_bfloat16 *dst = p.out + ((size_t)tc * H + h) * D + d;
#pragma unroll
        for (int t = 0; t < C; ++t)
            if (t < vc && KDA_ACCESS_OK(p.status, p.dbg.out, dst + (size_t)t * H * D, 2, 21)) {
                __nv_bfloat16 *q = dst + (size_t)t * H * D;
                *q = __float2bfloat16_rn(__bfloat162float(*q) + x[t >> 5][t & 31]);
            }
        __syncthreads();  // the accumulator is read before the next chunk's MMA rewrites it
    }
    if (tid == 0 && pending) {  // copies still in flight (after a timeout) land before the block exits
        if (pending & 1u) mbar_wait_bounded(&bars[0], 0, p.timeout_ns);
        // only after a break: the copies of chunks brk and brk + 1 (one per stage) may be in
        // flight; chunk c's copy completes use (c - c0) / 2 of stage (c - c0) % 2's barrier
        for (int cc = brk; cc >= 0 && cc <= brk + 1 && cc < c1; ++cc) {
            const int k = (cc - c0) & 1;
            if (pending & (2u << k)) mbar_wait_bounded(&bars[1 + k], (uint32_t)((cc - c0) >> 1) & 1u, p.timeout_ns);
        }
    }
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

}  // namespace

size_t seg_workspace_bytes(int32_t num_seqs, int32_t num_vseqs, int64_t e_chunks, int32_t H) {
    size_t b = round1k((size_t)(num_vseqs + 1) * 4) + round1k((size_t)num_vseqs * 16) +
               round1k((size_t)num_seqs * 4);
    b += 2 * (size_t)num_vseqs * H * D * D * 4;              // end states, transition products
    b += (size_t)num_vseqs * H * kSegStartTileBytes;         // start-state tiles
    b += (size_t)e_chunks * H * kSegETileBytes;              // E tiles
    b += round1k((size_t)num_vseqs * H * 4);                 // live E chunks per segment-head
    return b;
}

void seg_carve(SegPlan &sp, void *base, int32_t num_seqs, int32_t num_vseqs, int64_t e_chunks, int32_t H) {
    uint8_t *p = static_cast<uint8_t *>(base);
    sp.vcu = reinterpret_cast<int32_t *>(p);
    p += round1k((size_t)(num_vseqs + 1) * 4);
    sp.vinfo = reinterpret_cast<int4 *>(p);
    p += round1k((size_t)num_vseqs * 16);
    sp.vfirst = reinterpret_cast<int32_t *>(p);
    p += round1k((size_t)num_seqs * 4);
    sp.seg_state = reinterpret_cast<float *>(p);
    p += (size_t)num_vseqs * H * D * D * 4;
    sp.seg_trans = reinterpret_cast<float *>(p);
    p += (size_t)num_vseqs * H * D * D * 4;
    sp.s_start = p;
    p += (size_t)num_vseqs * H * kSegStartTileBytes;
    sp.e_tiles = p;
    p += (size_t)e_chunks * H * kSegETileBytes;
    sp.e_live = reinterpret_cast<int32_t *>(p);
    sp.num_vseqs = num_vseqs;
    sp.e_chunks = (int32_t)e_chunks;
}

cudaError_t launch_seg_plan(const Problem &p, const SegPlan &sp, cudaStream_t stream) {
    seg_plan_kernel<<<1, 32, 0, stream>>>(p.cu_seqlens, p.num_seqs, sp.segments, sp.vcu, sp.vinfo, sp.vfirst);
    return cudaGetLastError();
}

cudaError_t launch_seg_scan_fixup(const Problem &p, const SegPlan &sp, int32_t *status, cudaStream_t stream,
                                  int32_t *launches) {
    static PerDeviceOnce<> once_scan, once_fix;
    cudaError_t e = set_smem_limit_once(once_scan, (const void *)seg_scan_kernel, (int)SCAN_SMEM);
    if (e != cudaSuccess) return e;
    e = set_smem_limit_once(once_fix, (const void *)seg_fixup_kernel, (int)FIX_SMEM);
    if (e != cudaSuccess) return e;
    seg_scan_kernel<<<(unsigned)(p.num_seqs * p.H), SCAN_THREADS, SCAN_SMEM, stream>>>(
        sp.vinfo, sp.vfirst, p.num_seqs, p.H, sp.seg_state, sp.seg_trans, sp.s_start, p.final_state, p.slots,
        status, p.dbg);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    *launches += 1;
    if (sp.e_chunks == 0) return cudaSuccess;
    FixParams fp;
    fp.vcu = sp.vcu;
    fp.vinfo = sp.vinfo;
    fp.s_start = sp.s_start;
    fp.e_tiles = sp.e_tiles;
    fp.e_live = sp.e_live;
    fp.out = static_cast<__nv_bfloat16 *>(p.out);
    fp.status = status;
    fp.H = p.H;
    fp.num_vseqs = sp.num_vseqs;
    fp.ranges = (sp.max_chunks + FIX_CHUNKS - 1) / FIX_CHUNKS;
    fp.timeout_ns = kWaitTimeoutNs;
    fp.dbg = p.dbg;
    const unsigned grid = (unsigned)((int64_t)sp.num_vseqs * p.H * fp.ranges);
    seg_fixup_kernel<<<grid, FIX_THREADS, FIX_SMEM, stream>>>(fp);
    e = cudaGetLastError();
    if (e == cudaSuccess) *launches += 1;
    return e;
}

}  // namespace kda
