// Stable log-sum-exp merge with shared-memory staging: each warp streams its
// rows through a private ring of shared-memory stages filled by 16-byte
// cp.async copies, several steps ahead of the arithmetic.
//
// Same method and the same per-row arithmetic, in the same order, as
// rowcombine.cuh (vLLM-Ascend pull request "Fuse local SFA LSE formation into
// DCP pack": LSE_r = max_r + log(sum_r), -inf for invalid statistics;
// LSE* = logsumexp_r LSE_r; O = sum_r exp(LSE_r - LSE*) O_r), hence the same
// bits. What differs is how the payload arrives: rowcombine.cuh holds loads in
// flight in registers, which caps how far ahead a warp can run; here the bytes
// in flight live in shared memory, so a warp keeps NST-1 steps of every rank's
// rows in flight continuously, across chunk boundaries, while it forms the
// weights of the next chunk (phase A) and merges the current one (phase B).
//
// Work: warp w owns chunks w, w + nwarps, ... of 32 output rows; a chunk has
// STEPS = G steps of RPI = 32/G rows. A "group" is one step of one chunk; group
// number n of the warp is chunk n / STEPS, step n % STEPS. Group n lands in
// ring slot n % NST. The first group of a chunk also brings the chunk's
// statistics (lane = row) into the warp's statistics slot (chunk parity).
// Every lane reads back only the 16-byte vectors it copied itself, so
// cp.async.wait_group alone orders the copies before their use: there are no
// barriers and no spin-waits.
#pragma once

#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "rowcombine.cuh"

namespace cplse {

constexpr int kAsyncThreads = 128;

__device__ __forceinline__ uint32_t sh_addr(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_f32(uint32_t dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 64-bit quotient and remainder, on the 32-bit path when both operands fit.
__device__ __forceinline__ void divmod_u(int64_t x, int64_t d, int64_t& q, int64_t& r)
{
    if (((uint64_t)x | (uint64_t)d) < (1ull << 32)) {
        const uint32_t q32 = (uint32_t)x / (uint32_t)d;
        q = q32;
        r = (uint32_t)x - q32 * (uint32_t)d;
    } else {
        q = x / d;
        r = x - q * d;
    }
}

// Output row q -> (payload element offset of rank 0, destination row).
template <int MODE>
__device__ __forceinline__ void row_addr(const CombineArgs& a, int64_t q, int64_t& src, int64_t& dst)
{
    if (MODE == kModeFused) {
        int64_t t, h, j, hc;
        divmod_u(q, a.H, t, h);
        divmod_u(h, a.Hc, j, hc);
        src = t * a.so_t + h * a.so_h;
        dst = (j * a.T + t) * a.Hc + hc;
    } else {
        int64_t j, n;
        divmod_u(q, a.N, j, n);
        src = (j * a.W * a.N + n) * a.D;
        dst = q;
    }
}

// Shared memory per warp: NST payload slots of [VPL][WMAX][32 lanes] 16-byte
// vectors, then two statistics slots of [2][WMAX][32] floats.
template <int WMAX, int VPL, int NST>
struct AsyncRing {
    static constexpr int kSlotVecs = VPL * WMAX * 32;
    static constexpr int kPayBytes = NST * kSlotVecs * 16;
    static constexpr int kStatBytes = 2 * 2 * WMAX * 32 * 4;
    static constexpr int kWarpBytes = kPayBytes + kStatBytes;
};

template <typename P, int MODE, int WMAX, int G, int VPL, int NST>
__global__ void __launch_bounds__(kAsyncThreads)
rowcombine_async_kernel(const CombineArgs a)
{
    using Ring = AsyncRing<WMAX, VPL, NST>;
    constexpr int RPI = 32 / G;
    constexpr int STEPS = G;
    extern __shared__ __align__(16) uint8_t smem[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    uint4* ring = reinterpret_cast<uint4*>(smem + wib * Ring::kWarpBytes);
    float* sring = reinterpret_cast<float*>(smem + wib * Ring::kWarpBytes + Ring::kPayBytes);
    const int sub = lane / G;
    const int gl = lane % G;
    const int V = a.D >> 3;
    const int W = a.W;
    const int64_t warp = ((int64_t)blockIdx.x * kAsyncThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kAsyncThreads) >> 5;
    const int64_t nchunks = (a.rows + 31) >> 5;
    const int64_t my_chunks = warp < nchunks ? (nchunks - warp + nwarps - 1) / nwarps : 0;
    const int64_t ngroups = my_chunks * STEPS;

    // enqueue the copies of group n (an empty group past the end)
    auto issue = [&](int64_t n) {
        if (n < ngroups) {
            const int64_t ci = n / STEPS;
            const int step = (int)(n - ci * STEPS);
            const int64_t c = warp + ci * nwarps;
            const int slot = (int)(n % NST);
            if (step == 0) {   // this chunk's statistics, lane = row
                const int64_t q = c * 32 + lane;
                if (q < a.rows) {
                    float* sl = sring + (int)(ci & 1) * (2 * WMAX * 32);
                    if (MODE == kModeFused) {
                        int64_t t, h;
                        divmod_u(q, a.H, t, h);
#pragma unroll
                        for (int r = 0; r < WMAX; ++r)
                            if (r < W) {
                                cp_async_f32(sh_addr(sl + r * 32 + lane),
                                             a.smax + r * a.sm_r + t * a.sm_t + h * a.sm_h);
                                cp_async_f32(sh_addr(sl + (WMAX + r) * 32 + lane),
                                             a.ssum + r * a.ss_r + t * a.ss_t + h * a.ss_h);
                            }
                    } else {
                        int64_t j, nn;
                        divmod_u(q, a.N, j, nn);
#pragma unroll
                        for (int r = 0; r < WMAX; ++r)
                            if (r < W)
                                cp_async_f32(sh_addr(sl + r * 32 + lane),
                                             a.lse + (j * W + r) * a.N + nn);
                    }
                }
            }
            const int64_t q = c * 32 + step * RPI + sub;
            if (q < a.rows) {
                int64_t src, dst;
                row_addr<MODE>(a, q, src, dst);
                const uint4* base = reinterpret_cast<const uint4*>(a.src + src);
                uint4* sl = ring + slot * Ring::kSlotVecs;
#pragma unroll
                for (int e = 0; e < VPL; ++e) {
                    const int vec = gl + e * G;
                    if (vec < V) {
#pragma unroll
                        for (int r = 0; r < WMAX; ++r)
                            if (r < W)
                                cp_async16(sh_addr(sl + (e * WMAX + r) * 32 + lane),
                                           base + vec + ((r * a.rank_stride) >> 3));
                    }
                }
            }
        }
        cp_async_commit();
    };

    // prologue: NST-1 groups in flight
#pragma unroll
    for (int d = 0; d < NST - 1; ++d) issue(d);

    float w[WMAX];
    int64_t dst_own = 0;
    bool dead_own = true;
    for (int64_t n = 0; n < ngroups; ++n) {
        cp_async_wait<NST - 2>();       // group n has landed (this lane's copies)
        issue(n + NST - 1);             // refill the slot that group n-1 used
        const int64_t ci = n / STEPS;
        const int step = (int)(n - ci * STEPS);
        const int64_t c = warp + ci * nwarps;
        if (step == 0) {
            // ---------------- phase A: lane owns row c*32 + lane
            const int64_t q = c * 32 + lane;
            const bool qv = q < a.rows;
            int64_t src_unused = 0;
            if (qv) row_addr<MODE>(a, q, src_unused, dst_own);
            const float* sl = sring + (int)(ci & 1) * (2 * WMAX * 32);
            float lse[WMAX];
#pragma unroll
            for (int r = 0; r < WMAX; ++r) {
                if (MODE == kModeFused) {
                    float m = -INFINITY, sm = 0.f;
                    if (qv && r < W) {
                        m = sl[r * 32 + lane];
                        sm = sl[(WMAX + r) * 32 + lane];
                    }
                    const bool ok = isfinite(m) && isfinite(sm) && sm > 0.f;
                    lse[r] = ok ? m + logf(sm) : -INFINITY;
                } else {
                    const float x = (qv && r < W) ? sl[r * 32 + lane] : -INFINITY;
                    lse[r] = x > -INFINITY ? x : -INFINITY;
                }
            }
            float M = -INFINITY;
#pragma unroll
            for (int r = 0; r < WMAX; ++r) M = fmaxf(M, lse[r]);
            float L = -INFINITY;
            if (M > -INFINITY) {
                float S = 0.f;
#pragma unroll
                for (int r = 0; r < WMAX; ++r)
                    if (lse[r] > -INFINITY) S += expf(lse[r] - M);
                L = M + logf(S);
#pragma unroll
                for (int r = 0; r < WMAX; ++r) w[r] = lse[r] > -INFINITY ? expf(lse[r] - L) : 0.f;
            } else {
#pragma unroll
                for (int r = 0; r < WMAX; ++r) w[r] = 0.f;
            }
            if (qv) st_stream(a.out_lse + dst_own, L);
            dead_own = !(M > -INFINITY);
        }
        // ---------------- phase B: this step's RPI rows, G lanes per row
        const int k = step * RPI + sub;                       // row of the chunk
        const int64_t q = c * 32 + k;
        const int64_t db = __shfl_sync(kFull, dst_own, k);
        const bool dead = __shfl_sync(kFull, (int)dead_own, k) != 0;
        float ws[WMAX];
#pragma unroll
        for (int r = 0; r < WMAX; ++r) ws[r] = __shfl_sync(kFull, w[r], k);
        if (q < a.rows) {
            const uint4* sl = ring + (int)(n % NST) * Ring::kSlotVecs;
#pragma unroll
            for (int e = 0; e < VPL; ++e) {
                const int vec = gl + e * G;
                if (vec >= V) continue;
                float acc[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) acc[x] = -0.f;
#pragma unroll
                for (int r = 0; r < WMAX; ++r) {
                    if (r >= W) break;
                    uint4 v = sl[(e * WMAX + r) * 32 + lane];
                    if (!(ws[r] != 0.f)) v = make_uint4(kNegZero2, kNegZero2, kNegZero2, kNegZero2);
                    const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const float2 f = unpack2<P>(wd[x]);
                        acc[2 * x] = fmaf(ws[r], f.x, acc[2 * x]);
                        acc[2 * x + 1] = fmaf(ws[r], f.y, acc[2 * x + 1]);
                    }
                }
                uint4 o;
                if (dead) {
                    o = make_uint4(0u, 0u, 0u, 0u);
                } else {
                    o.x = pack2<P>(acc[0], acc[1]);
                    o.y = pack2<P>(acc[2], acc[3]);
                    o.z = pack2<P>(acc[4], acc[5]);
                    o.w = pack2<P>(acc[6], acc[7]);
                }
                st_stream(reinterpret_cast<uint4*>(a.out + db * a.D) + vec, o);
            }
        }
    }
    cp_async_wait<0>();
}

}  // namespace cplse
