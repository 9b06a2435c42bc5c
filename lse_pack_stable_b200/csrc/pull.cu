// Pull-based DCP exchange for one real destination rank: the fused
// pack -> all-to-all -> combine across GPUs, in which destination j reads the
// rows it combines straight out of every source rank's partial output and
// statistics (peer memory over NVLink, mapped into this process) instead of
// receiving a packet.
//
// Method: vLLM-Ascend pull request "Fuse local SFA LSE formation into DCP
// pack", section "What this PR does / why we need it?": each source rank's
// contribution to a row is LSE_r = softmax_max_r + log(softmax_sum_r), -inf
// for invalid statistics; destination j, which owns head chunk j (or token
// chunk j), merges the W contributions with the stable combine. The exchange
// there is an HCCL all-to-all of the packed head chunks; here the destination
// loads each source row once, with plain 16-byte global loads, so the packet
// never exists on either side.
//
// Work split: the register-staged scheme of rowcombine.cuh. A warp owns chunks
// of 32 output rows. Phase A: lane i forms the W LSE values of row i (one
// coalesced float from each rank's max and sum plane) and the merge weights
// (merge_weights, the arithmetic every merge kernel shares), which it writes
// to a per-warp table in shared memory. Phase B: G lanes cover a row with
// 16-byte vectors; every rank's vector of U steps is loaded before any is
// used, accumulated in fp32 in rank order, rounded and stored.
// A weight-0 contribution is neither loaded nor added (-0.0 stands in).
//
// No bulk copies, no TMA and no multicast: every remote byte arrives through
// an ordinary load instruction, so nothing here depends on how the peer
// memory was mapped beyond its being addressable from this device.
#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "rowcombine.cuh"

namespace cplse {
namespace {

constexpr int kPullThreads = 128;

template <typename P, int WMAX, int G, int VPL, int U>
__global__ void __launch_bounds__(kPullThreads, merge_min_blocks<VPL>())
pull_combine_kernel(const PullArgs a)
{
    constexpr int RPI = 32 / G;          // rows per step
    constexpr int STEPS = 32 / RPI;      // steps per chunk
    // ranks loaded at once: 16 vectors in flight per lane per batch
    constexpr int RB = WMAX < 16 / VPL ? WMAX : 16 / VPL;
    constexpr int WS = (WMAX + 3) / 4 * 4;
    static_assert(STEPS % U == 0, "U must divide the steps of a chunk");
    // per-warp row table: the weights of the chunk's 32 rows
    __shared__ __align__(16) float wtab[kPullThreads / 32][32][WS];

    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    const int sub = lane / G;
    const int gl = lane % G;
    const int64_t warp = ((int64_t)blockIdx.x * kPullThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kPullThreads) >> 5;
    const ChunkPlan plan(a.rows, warp, nwarps);
    const int V = a.D >> 3;

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int64_t my_chunks = plan.count();
    for (int64_t ci = 0; ci < my_chunks; ++ci) {
        int64_t c0;
        int cn;
        plan.chunk(ci, c0, cn);
        // ---------------- phase A: lane owns output row q = c0 + lane
        const int64_t q = c0 + lane;
        const bool qv = lane < cn;
        int64_t t = 0, h = 0;
        if (qv) {
            if (a.token_scatter) {          // token chunk dst: row (tc, h), t = dst*Tc + tc
                const int64_t tc = q / a.H;
                h = q - tc * a.H;
                t = (int64_t)a.dst * a.Tc + tc;
            } else {                        // head chunk dst: row (t, hc), h = dst*Hc + hc
                t = q / a.Hc;
                h = (int64_t)a.dst * a.Hc + (q - t * a.Hc);
            }
        }
        const int64_t src_row = t * a.so_t + h * a.so_h;
        const int64_t mo = t * a.sm_t + h * a.sm_h;
        const int64_t so = t * a.ss_t + h * a.ss_h;
        uint32_t vmask = 0;               // bit r: contribution r has a nonzero weight
        bool row_dead;
        {
            float lse[WMAX];
#pragma unroll
            for (int r = 0; r < WMAX; ++r) {
                float m = -INFINITY, sm = 0.f;
                if (qv && r < a.W) {
                    m = ld_ro(a.smax[r] + mo);
                    sm = ld_ro(a.ssum[r] + so);
                }
                // invalid statistic: non-finite max, non-finite sum, or sum <= 0
                const bool ok = isfinite(m) && isfinite(sm) && sm > 0.f;
                lse[r] = ok ? m + logf(sm) : -INFINITY;
            }
            float w[WS];
            float L;
            row_dead = !merge_weights(lse, w, L);
            if (qv) st_stream(a.out_lse + q, L);
#pragma unroll
            for (int r = 0; r < WMAX; ++r) vmask |= (w[r] != 0.f ? 1u : 0u) << r;
            __syncwarp();                 // the previous chunk's table is read
#pragma unroll
            for (int r = 0; r < WS; r += 4)
                *reinterpret_cast<float4*>(&wtab[wib][lane][r]) =
                    make_float4(w[r], w[r + 1], w[r + 2], w[r + 3]);
            __syncwarp();                 // the table is visible to the warp
        }

        // ---------------- phase B: G lanes per row (weights from the table)
#pragma unroll 1
        for (int s0 = 0; s0 < STEPS; s0 += U) {
            int64_t sb[U];
            bool rv[U], dead[U];
            uint32_t msk[U];
            int kk[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = (s0 + u) * RPI + sub;
                kk[u] = k;
                sb[u] = __shfl_sync(kFull, src_row, k);
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
#pragma unroll
                        for (int rr = 0; rr < RB; ++rr) {
                            const int r = r0 + rr;
                            if (rv[u] && vec < V && ((msk[u] >> r) & 1u))
                                v[u][e][rr] = ld_ro(
                                    reinterpret_cast<const uint4*>(a.o[r] + sb[u]) + vec);
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
                    const int k = (s0 + u) * RPI + sub;
                    st_stream(reinterpret_cast<uint4*>(a.out + (c0 + k) * a.D) + vec, o);
                }
        }
    }
}

template <typename P, int WMAX, int G, int VPL>
cudaError_t launch_pull_inst(const PullArgs& a, cudaStream_t s)
{
    constexpr int U0 = (WMAX * VPL) >= kLoadsInFlight ? 1 : kLoadsInFlight / (WMAX * VPL);
    constexpr int U = U0 > G ? G : U0;
    constexpr auto kern = pull_combine_kernel<P, WMAX, G, VPL, U>;
    int per_sm = 0;
    {
        const cudaError_t e = resident_blocks<kern>(kPullThreads, 0, per_sm);
        if (e != cudaSuccess) return e;
    }
    const int64_t blocks = merge_grid(a.rows, kPullThreads, per_sm, U * (32 / G));
    return launch_pdl(kern, (unsigned)blocks, kPullThreads, 0, s, a);
}

template <typename P, int WMAX>
cudaError_t launch_pull_w(const PullArgs& a, cudaStream_t s)
{
    const RowShape rs = row_shape(a.D);
    switch (rs.G * 10 + rs.VPL) {
    case 41: return launch_pull_inst<P, WMAX, 4, 1>(a, s);
    case 81: return launch_pull_inst<P, WMAX, 8, 1>(a, s);
    case 161: return launch_pull_inst<P, WMAX, 16, 1>(a, s);
    case 321: return launch_pull_inst<P, WMAX, 32, 1>(a, s);
    case 322: return launch_pull_inst<P, WMAX, 32, 2>(a, s);
    default: return launch_pull_inst<P, WMAX, 32, 4>(a, s);
    }
}

template <typename P>
cudaError_t launch_pull_p(const PullArgs& a, cudaStream_t s)
{
    if (a.W <= 2) return launch_pull_w<P, 2>(a, s);
    if (a.W <= 4) return launch_pull_w<P, 4>(a, s);
    if (a.W <= 8) return launch_pull_w<P, 8>(a, s);
    if (a.W <= 16) return launch_pull_w<P, 16>(a, s);
    return launch_pull_w<P, 32>(a, s);
}

}  // namespace

cudaError_t launch_pull_combine(const PullArgs& a, Dtype dt, cudaStream_t s)
{
    return dt == Dtype::kBf16 ? launch_pull_p<Bf16>(a, s) : launch_pull_p<Fp16>(a, s);
}

}  // namespace cplse
