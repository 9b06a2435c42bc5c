// Stable log-sum-exp merge of W partial attention outputs, one output row at a
// time; shared by the fused pack->a2a->combine kernel and the combine kernel,
// so that both produce the same bits for the same LSE values.
//
// Method (vLLM-Ascend pull request "Fuse local SFA LSE formation into DCP
// pack", section "What this PR does / why we need it?"): each rank's
// contribution carries LSE = softmax_max + log(softmax_sum), -inf when the
// statistics are invalid; the stable combine merges the W contributions of a
// row as LSE* = logsumexp_r LSE_r and O = sum_r exp(LSE_r - LSE*) O_r, with
// -inf contributions weighted zero and an all-invalid row giving O = 0,
// LSE* = -inf.
//
// Work split. A warp owns chunks of 32 consecutive output rows.
//   Phase A: lane i takes row i of the chunk. It loads the row's W statistics
//     (coalesced across the warp: consecutive rows are consecutive floats of
//     each rank's plane), forms each LSE, and computes M, the sum, LSE* and the
//     W weights sequentially in rank order, all in registers.
//   Phase B: G lanes cover one row's D elements with 16-byte vectors (VPL per
//     lane), 32/G rows per step. The row's weights reach the group through a
//     per-warp table in shared memory that phase A writes; its addresses and a
//     mask of the ranks with nonzero weight come by warp shuffles from the
//     lane that owns the row. (Shuffling all W weights to every lane held them
//     twice in registers: on the 16-rank stress workload the table measured
//     2 % faster.) Every rank's vector is loaded before any is used (U steps at
//     once), accumulated in fp32 in rank order, rounded to the payload type
//     and stored.
// An invalid contribution (weight 0) is neither loaded nor added: its payload
// is replaced by -0.0, which leaves the fp32 accumulator (started at -0.0)
// unchanged bit for bit.
#pragma once

#include <math.h>

#include "common.cuh"
#include "launch.h"

namespace cplse {

#ifndef CPLSE_COMBINE_THREADS
#define CPLSE_COMBINE_THREADS 128
#endif
#ifndef CPLSE_LOADS_IN_FLIGHT
#define CPLSE_LOADS_IN_FLIGHT 8
#endif
constexpr int kCombineThreads = CPLSE_COMBINE_THREADS;
// 16-byte loads each lane keeps in flight in phase B (sets U below)
constexpr int kLoadsInFlight = CPLSE_LOADS_IN_FLIGHT;
constexpr unsigned kFull = 0xffffffffu;
constexpr uint32_t kNegZero2 = 0x80008000u;   // two -0.0 payload elements

enum { kModeFused = 0, kModeCombine = 1 };

// How a grid's warps share the output rows of a merge. Full rounds first: in
// round k, warp w takes the 32-row chunk k*nwarps + w, so that warps working
// at the same time read neighbouring rows. The rows left after the last full
// round (fewer than 32 per warp) are then split evenly, ceil(rem / nwarps) per
// warp, rather than as whole chunks to some warps only: a whole chunk can be
// hundreds of KB of payload, and the warps that would take an extra one would
// keep the grid running long after the others had finished.
struct ChunkPlan {
    int64_t rows, warp, nwarps;
    int64_t full;             // full rounds of 32-row chunks
    int64_t last_base;        // first row of the last, partial round
    int64_t last_rows;        // rows per warp in the last round (<= 32)

    __host__ __device__ __forceinline__ ChunkPlan(int64_t rows_, int64_t warp_, int64_t nwarps_)
        : rows(rows_), warp(warp_), nwarps(nwarps_)
    {
        full = rows / (32 * nwarps);
        last_base = full * 32 * nwarps;
        last_rows = (rows - last_base + nwarps - 1) / nwarps;
    }

    // chunks of this warp
    __host__ __device__ __forceinline__ int64_t count() const
    {
        return full + (last_base + warp * last_rows < rows ? 1 : 0);
    }

    // chunk i of this warp: its first row and its row count (1..32)
    __host__ __device__ __forceinline__ void chunk(int64_t i, int64_t& start, int& n) const
    {
        if (i < full) {
            start = (warp + i * nwarps) * 32;
            n = 32;
        } else {
            start = last_base + warp * last_rows;
            const int64_t left = rows - start;
            n = (int)(left < last_rows ? left : last_rows);
        }
    }
};

// The merge weights of one row from its W contributions' LSE values (-inf for
// an invalid contribution or one beyond W), in rank order: M = max_r lse_r;
// if M = -inf the row is all invalid (returns false, every weight 0, L = -inf);
// else L = M + logf(sum over valid r of expf(lse_r - M)) and
// w_r = expf(lse_r - L) for valid r, 0 otherwise. Every merge kernel calls
// this, so they all produce the same bits for the same LSE values.
template <int WMAX, int NW>
__device__ __forceinline__ bool merge_weights(const float (&lse)[WMAX], float (&w)[NW], float& L)
{
    static_assert(NW >= WMAX, "weight array shorter than the ranks");
#pragma unroll
    for (int r = 0; r < NW; ++r) w[r] = 0.f;
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < WMAX; ++r) M = fmaxf(M, lse[r]);
    L = -INFINITY;
    if (!(M > -INFINITY)) return false;
    float S = 0.f;
#pragma unroll
    for (int r = 0; r < WMAX; ++r)
        if (lse[r] > -INFINITY) S += expf(lse[r] - M);
    L = M + logf(S);
#pragma unroll
    for (int r = 0; r < WMAX; ++r) w[r] = lse[r] > -INFINITY ? expf(lse[r] - L) : 0.f;
    return true;
}

// Phase A for one row: addresses and the W LSE values (-inf beyond W or q).
template <int MODE, int WMAX>
__device__ __forceinline__ void row_stats(const CombineArgs& a, int64_t q, bool qv,
                                          int64_t& src_row, int64_t& dst_row, float (&lse)[WMAX])
{
    if (MODE == kModeFused) {
        int64_t t = 0, h = 0;
        if (qv) {
            t = q / a.H;
            h = q - t * a.H;
        }
        const int64_t j = h / a.Hc;
        const int64_t hc = h - j * a.Hc;
        src_row = t * a.so_t + h * a.so_h;
        dst_row = a.token_scatter ? q : (j * a.T + t) * a.Hc + hc;
        const float* pm = a.smax + t * a.sm_t + h * a.sm_h;
        const float* ps = a.ssum + t * a.ss_t + h * a.ss_h;
        float m[WMAX], s[WMAX];
#pragma unroll
        for (int r = 0; r < WMAX; ++r) {
            if (qv && r < a.W) {
                m[r] = ld_ro(pm + r * a.sm_r);
                s[r] = ld_ro(ps + r * a.ss_r);
            } else {
                m[r] = -INFINITY;
                s[r] = 0.f;
            }
        }
#pragma unroll
        for (int r = 0; r < WMAX; ++r) {
            // invalid statistic: non-finite max, non-finite sum, or sum <= 0
            const bool ok = isfinite(m[r]) && isfinite(s[r]) && s[r] > 0.f;
            lse[r] = ok ? m[r] + logf(s[r]) : -INFINITY;
        }
    } else {
        int64_t j = 0, n = 0;
        if (qv) {
            j = q / a.N;
            n = q - j * a.N;
        }
        src_row = (j * a.W * a.N + n) * a.D;
        dst_row = q;
        const float* pl = a.lse + j * a.W * a.N + n;
#pragma unroll
        for (int r = 0; r < WMAX; ++r) {
            float x = (qv && r < a.W) ? ld_ro(pl + r * a.N) : -INFINITY;
            lse[r] = x > -INFINITY ? x : -INFINITY;   // NaN counts as invalid
        }
    }
}

// Rows of one 16-byte vector per lane (D <= 256) keep four blocks resident: a
// register budget of 128 per thread, which the 16-rank stress workload needs
// for its loads in flight and which the compiler would exceed unbidden in
// combine mode. Wider rows need more registers for their vectors.
template <int VPL>
constexpr int merge_min_blocks()
{
    return VPL == 1 ? 4 : 1;
}

template <typename P, int MODE, int WMAX, int G, int VPL, int U>
__global__ void __launch_bounds__(kCombineThreads, merge_min_blocks<VPL>())
rowcombine_kernel(const CombineArgs a)
{
    constexpr int RPI = 32 / G;          // rows per step
    constexpr int STEPS = 32 / RPI;      // steps per chunk
    // ranks loaded at once: 16 vectors in flight per lane per batch
    constexpr int RB = WMAX < 16 / VPL ? WMAX : 16 / VPL;
    constexpr int WS = (WMAX + 3) / 4 * 4;
    static_assert(STEPS % U == 0, "U must divide the steps of a chunk");
    // per-warp row table: the weights of the chunk's 32 rows
    __shared__ __align__(16) float wtab[kCombineThreads / 32][32][WS];

    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int sub = lane / G;
    const int gl = lane % G;
    const int64_t warp = ((int64_t)blockIdx.x * kCombineThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kCombineThreads) >> 5;
    const ChunkPlan plan(a.rows, warp, nwarps);
    const int V = a.D >> 3;
    const int64_t rank_stride = a.rank_stride;

    // Programmatic dependent launch, as in the shared-memory-staged kernel: the
    // next kernel in the stream may be scheduled now, and this one reads
    // nothing until the previous kernel has completed and its writes are
    // visible.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int64_t my_chunks = plan.count();
    for (int64_t ci = 0; ci < my_chunks; ++ci) {
        int64_t c0;
        int cn;
        plan.chunk(ci, c0, cn);
        // ---------------- phase A: lane owns row c0 + lane
        const int64_t q = c0 + lane;
        const bool qv = lane < cn;
        int64_t src_row, dst_row;
        uint32_t vmask = 0;               // bit r: contribution r has a nonzero weight
        bool row_dead;
        {
            float lse[WMAX];
            row_stats<MODE, WMAX>(a, q, qv, src_row, dst_row, lse);
            float w[WS];
            float L;
            row_dead = !merge_weights(lse, w, L);
            if (qv) st_stream(a.out_lse + dst_row, L);
#pragma unroll
            for (int r = 0; r < WMAX; ++r) vmask |= (w[r] != 0.f ? 1u : 0u) << r;
            __syncwarp();                 // the previous chunk's table is read
#pragma unroll
            for (int r = 0; r < WS; r += 4)
                *reinterpret_cast<float4*>(&wtab[wib][lane][r]) =
                    make_float4(w[r], w[r + 1], w[r + 2], w[r + 3]);
            __syncwarp();                 // the table is visible to the warp
        }

        // ---------------- phase B: G lanes per row; the row's weights come from
        // the table, its addresses and valid-rank mask from the owning lane
#pragma unroll 1
        for (int s0 = 0; s0 < STEPS; s0 += U) {
            int64_t sb[U], db[U];
            bool rv[U], dead[U];
            uint32_t msk[U];
            int kk[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = (s0 + u) * RPI + sub;
                kk[u] = k;
                sb[u] = __shfl_sync(kFull, src_row, k);
                db[u] = __shfl_sync(kFull, dst_row, k);
                dead[u] = __shfl_sync(kFull, (int)row_dead, k) != 0;
                msk[u] = __shfl_sync(kFull, vmask, k);
                rv[u] = k < cn;
            }
            float acc[U][VPL][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int e = 0; e < VPL; ++e)
#pragma unroll
                    for (int x = 0; x < 8; ++x) acc[u][e][x] = -0.f;

#pragma unroll 1
            for (int r0 = 0; r0 < WMAX; r0 += RB) {   // one batch of ranks at a time
                uint4 v[U][VPL][RB];
#pragma unroll
                for (int u = 0; u < U; ++u)
#pragma unroll
                    for (int e = 0; e < VPL; ++e) {
                        const int vec = gl + e * G;
                        const uint4* base = reinterpret_cast<const uint4*>(a.src + sb[u]) + vec;
#pragma unroll
                        for (int rr = 0; rr < RB; ++rr) {
                            const int r = r0 + rr;
                            if (rv[u] && vec < V && ((msk[u] >> r) & 1u))
                                v[u][e][rr] = ld_ro(base + (r * rank_stride >> 3));
                            else
                                v[u][e][rr] = make_uint4(kNegZero2, kNegZero2, kNegZero2, kNegZero2);
                        }
                    }
#pragma unroll
                for (int u = 0; u < U; ++u)
#pragma unroll
                    for (int e = 0; e < VPL; ++e)
#pragma unroll
                        for (int rr = 0; rr < RB; ++rr) {
                            const float wr = wtab[wib][kk[u]][r0 + rr];
                            const uint32_t wd[4] = {v[u][e][rr].x, v[u][e][rr].y, v[u][e][rr].z,
                                                    v[u][e][rr].w};
#pragma unroll
                            for (int x = 0; x < 4; ++x) {
                                const float2 f = unpack2<P>(wd[x]);
                                acc[u][e][2 * x] = fmaf(wr, f.x, acc[u][e][2 * x]);
                                acc[u][e][2 * x + 1] = fmaf(wr, f.y, acc[u][e][2 * x + 1]);
                            }
                        }
            }

#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int e = 0; e < VPL; ++e) {
                    const int vec = gl + e * G;
                    if (!(rv[u] && vec < V)) continue;
                    uint4 o;
                    if (dead[u]) {
                        o = make_uint4(0u, 0u, 0u, 0u);   // all-invalid row: +0
                    } else {
                        o.x = pack2<P>(acc[u][e][0], acc[u][e][1]);
                        o.y = pack2<P>(acc[u][e][2], acc[u][e][3]);
                        o.z = pack2<P>(acc[u][e][4], acc[u][e][5]);
                        o.w = pack2<P>(acc[u][e][6], acc[u][e][7]);
                    }
                    st_stream(reinterpret_cast<uint4*>(a.out + db[u] * a.D) + vec, o);
                }
        }
    }
}

// Blocks of a merge grid: enough warps that each gets at least `min_rows`
// output rows (one batch of loads in flight; ChunkPlan then splits the rows
// evenly), at most what is resident on the whole GPU at once. A problem with
// few rows thus still spreads over every SM instead of giving each of a few
// warps a whole 32-row chunk.
inline int64_t merge_grid(int64_t rows, int threads, int per_sm, int min_rows)
{
    const int64_t wpb = threads / 32;
    const int64_t warps = (rows + min_rows - 1) / min_rows;
    int64_t blocks = (warps + wpb - 1) / wpb;
    const int64_t cap = (int64_t)per_sm * sm_count();
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return blocks;
}

// Launch with programmatic stream serialization: back-to-back launches overlap
// the next grid's scheduling with this one's drain. Every merge kernel opens
// with griddepcontrol.wait, so none reads memory before the previous kernel in
// the stream has completed.
template <typename K, typename A>
cudaError_t launch_pdl(K kern, unsigned blocks, int threads, int smem, cudaStream_t s,
                       const A& a)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

// Lanes per row and vectors per lane for a head dim of D elements (D % 8 == 0).
struct RowShape {
    int G, VPL;
};

inline RowShape row_shape(int D)
{
    const int V = D / kVecElems;
    if (V <= 4) return {4, 1};
    if (V <= 8) return {8, 1};
    if (V <= 16) return {16, 1};
    if (V <= 32) return {32, 1};
    if (V <= 64) return {32, 2};
    return {32, 4};
}

template <typename P, int MODE, int WMAX, int G, int VPL>
cudaError_t launch_rowcombine_inst(const CombineArgs& a, cudaStream_t s)
{
    constexpr int U0 = (WMAX * VPL) >= kLoadsInFlight ? 1 : kLoadsInFlight / (WMAX * VPL);
    constexpr int U = U0 > G ? G : U0;
    constexpr auto kern = rowcombine_kernel<P, MODE, WMAX, G, VPL, U>;
    int per_sm = 0;
    {
        const cudaError_t e = resident_blocks<kern>(kCombineThreads, 0, per_sm);
        if (e != cudaSuccess) return e;
    }
    // one batch of loads: U steps of 32/G rows
    const int64_t blocks = merge_grid(a.rows, kCombineThreads, per_sm, U * (32 / G));
    return launch_pdl(kern, (unsigned)blocks, kCombineThreads, 0, s, a);
}

}  // namespace cplse
