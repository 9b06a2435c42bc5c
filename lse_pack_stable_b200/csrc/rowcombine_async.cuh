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
// STEPS = G steps of RPI = 32/G rows. A "group" is one step of one chunk;
// group number n of the warp is chunk n / STEPS, step n % STEPS (compile-time
// divisors), and that step covers rows ((n + w) mod STEPS) * RPI .. of the
// chunk: every warp starts its chunks at a different step, so that warps in
// lockstep do not all touch the same offset of their chunks at once (measured:
// 2-3 % on a 4-rank decode merge, 1-1.5 % on an 8-rank one; the register-staged
// kernel of rowcombine.cuh gained nothing from it and keeps step order).
// Group n lands in ring slot n % NST. The first group of a chunk
// also brings the chunk's statistics (lane = row) into statistics slot
// chunk % NSTAT, where NSTAT = (NST-1)/STEPS + 1 guarantees the slot was read
// (phase A of an older chunk) before it is refilled NST-1 groups ahead.
// Every lane reads back only the 16-byte vectors it copied itself, so
// cp.async.wait_group alone orders the copies before their use: there are no
// barriers and no spin-waits.
#pragma once

#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "rowcombine.cuh"

namespace cplse {

#ifndef CPLSE_ASYNC_THREADS
#define CPLSE_ASYNC_THREADS 128
#endif
#ifndef CPLSE_ASYNC_INFLIGHT
#define CPLSE_ASYNC_INFLIGHT 4096
#endif

constexpr int kAsyncThreads = CPLSE_ASYNC_THREADS;
// payload bytes each warp keeps in flight (sets the ring depth NST)
constexpr int kAsyncInflight = CPLSE_ASYNC_INFLIGHT;

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

// Shared memory per warp: NST payload slots of [VPL][WMAX][32 lanes] 16-byte
// vectors; NSTAT statistics slots of [2][WMAX][32] floats; and the chunk's row
// table: weights [32][WS] (WS = WMAX rounded up to 4, for 16-byte reads) and
// destination rows [32] (bitwise-complemented for an all-invalid row).
template <int WMAX, int G, int VPL, int NST>
struct AsyncRing {
    static constexpr int kSlotVecs = VPL * WMAX * 32;
    static constexpr int kPayBytes = NST * kSlotVecs * 16;
    static constexpr int kStatSlotFloats = 2 * WMAX * 32;
    static constexpr int kStat = (NST - 1) / G + 1;
    static constexpr int kStatBytes = kStat * kStatSlotFloats * 4;
    static constexpr int WS = (WMAX + 3) / 4 * 4;
    static constexpr int kTabBytes = 32 * WS * 4 + 32 * 8;
    static constexpr int kWarpBytes = kPayBytes + kStatBytes + kTabBytes;
};

template <typename P, int MODE, int WMAX, int G, int VPL, int NST>
__global__ void __launch_bounds__(kAsyncThreads)
rowcombine_async_kernel(const CombineArgs a)
{
    using Ring = AsyncRing<WMAX, G, VPL, NST>;
    constexpr int RPI = 32 / G;
    constexpr int STEPS = G;
    constexpr int WS = Ring::WS;
    extern __shared__ __align__(16) uint8_t smem[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    uint8_t* wbase = smem + wib * Ring::kWarpBytes;
    uint4* ring = reinterpret_cast<uint4*>(wbase);
    float* sring = reinterpret_cast<float*>(wbase + Ring::kPayBytes);
    float* wtab = reinterpret_cast<float*>(wbase + Ring::kPayBytes + Ring::kStatBytes);
    int64_t* dtab = reinterpret_cast<int64_t*>(wbase + Ring::kPayBytes + Ring::kStatBytes + 32 * WS * 4);
    const int sub = lane / G;
    const int gl = lane % G;
    const int V = a.D >> 3;
    const int W = a.W;
    const int64_t rs16 = a.rank_stride >> 3;              // rank stride in 16-byte vectors
    const uint4* src16 = reinterpret_cast<const uint4*>(a.src);
    const int64_t warp = ((int64_t)blockIdx.x * kAsyncThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kAsyncThreads) >> 5;
    const ChunkPlan plan(a.rows, warp, nwarps);
    const int64_t ngroups = plan.count() * STEPS;
    // Each warp walks the steps of its chunks starting at step warp mod STEPS.
    // Warps run nearly in lockstep, and chunks start on 32-row boundaries, so
    // without this every warp would be reading (and writing) the same offset
    // within its chunk at the same moment; rotated, the accesses in flight
    // spread over STEPS offsets. Each row's arithmetic is unchanged.
    static_assert((STEPS & (STEPS - 1)) == 0, "steps per chunk must be a power of two");
    const int rot = (int)(warp & (STEPS - 1));

    // Programmatic dependent launch: the next kernel in the stream may be
    // scheduled now, and this one reads nothing until the previous kernel in
    // the stream has completed and its writes are visible.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // payload vector offset (rank 0) of output row q
    auto row_src = [&](int64_t q) -> int64_t {
        if (MODE == kModeFused) {
            if (a.dense_rows) return q * (a.D >> 3);
            int64_t t, h;
            divmod_u(q, a.H, t, h);
            return (t * a.so_t + h * a.so_h) >> 3;
        } else {
            int64_t j, n;
            divmod_u(q, a.N, j, n);
            return ((j * W * a.N + n) * a.D) >> 3;
        }
    };

    // A chunk's rows are consecutive rows of one source block -- so that their
    // payload offsets are those of its first row plus k*D -- when rows are
    // dense (fused), or when the chunk stays inside one (dst) block (combine).
    auto chunk_is_linear = [&](int64_t c0, int cn) -> bool {
        if (MODE == kModeFused) return a.dense_rows != 0;
        return c0 / a.N == (c0 + cn - 1) / a.N;
    };

    // issue cursor: group ni = chunk ci_i, step st_i, ring slot sl_i
    int64_t ni = 0, ci_i = 0, chunk_src = 0, c0_i = 0;
    int st_i = 0, sl_i = 0, cn_i = 0;
    bool lin_i = false;
    auto issue_next = [&]() {
        if (ni < ngroups) {
            if (st_i == 0) {
                plan.chunk(ci_i, c0_i, cn_i);
                lin_i = chunk_is_linear(c0_i, cn_i);
                chunk_src = row_src(c0_i);                 // rank-0 offset of the chunk's row 0
            }
            if (st_i == 0) {   // this chunk's statistics, lane = row
                const int64_t q = c0_i + lane;
                if (lane < cn_i) {
                    float* sl = sring + (int)(ci_i % Ring::kStat) * Ring::kStatSlotFloats;
                    if (MODE == kModeFused) {
                        int64_t t, h;
                        divmod_u(q, a.H, t, h);
                        const float* pm = a.smax + t * a.sm_t + h * a.sm_h;
                        const float* ps = a.ssum + t * a.ss_t + h * a.ss_h;
#pragma unroll
                        for (int r = 0; r < WMAX; ++r)
                            if (r < W) {
                                cp_async_f32(sh_addr(sl + r * 32 + lane), pm + r * a.sm_r);
                                cp_async_f32(sh_addr(sl + (WMAX + r) * 32 + lane), ps + r * a.ss_r);
                            }
                    } else {
                        int64_t j, nn;
                        divmod_u(q, a.N, j, nn);
                        const float* pl = a.lse + j * W * a.N + nn;
#pragma unroll
                        for (int r = 0; r < WMAX; ++r)
                            if (r < W) cp_async_f32(sh_addr(sl + r * 32 + lane), pl + r * a.N);
                    }
                }
            }
            const int kq = ((st_i + rot) & (STEPS - 1)) * RPI + sub;   // row of the chunk
            if (kq < cn_i) {
                const int64_t off = lin_i ? chunk_src + kq * V : row_src(c0_i + kq);
                const uint4* base = src16 + off + gl;
                uint4* sl = ring + sl_i * Ring::kSlotVecs + lane;
#pragma unroll
                for (int e = 0; e < VPL; ++e) {
                    if (gl + e * G < V) {
#pragma unroll
                        for (int r = 0; r < WMAX; ++r)
                            if (r < W) cp_async16(sh_addr(sl + (e * WMAX + r) * 32), base + e * G + r * rs16);
                    }
                }
            }
            ++ni;
            if (++st_i == STEPS) {
                st_i = 0;
                ++ci_i;
            }
            if (++sl_i == NST) sl_i = 0;
        }
        cp_async_commit();
    };

    // prologue: NST-1 groups in flight
#pragma unroll 1
    for (int d = 0; d < NST - 1; ++d) issue_next();

    int64_t ci = 0, c0 = 0;
    int step = 0, slot = 0, cn = 0;
    for (int64_t n = 0; n < ngroups; ++n) {
        cp_async_wait<NST - 2>();       // group n has landed (this lane's copies)
        issue_next();                   // refill the slot that group n-1 used
        if (step == 0) plan.chunk(ci, c0, cn);
        if (step == 0) {
            // ---------------- phase A: lane owns row c0 + lane
            const int64_t q = c0 + lane;
            const bool qv = lane < cn;
            int64_t dst = 0;
            if (qv) {
                if (MODE == kModeFused && !a.token_scatter) {
                    int64_t t, h, j, hc;
                    divmod_u(q, a.H, t, h);
                    divmod_u(h, a.Hc, j, hc);
                    dst = (j * a.T + t) * a.Hc + hc;
                } else {
                    dst = q;                                // token chunks keep source order
                }
            }
            const float* sl = sring + (int)(ci % Ring::kStat) * Ring::kStatSlotFloats;
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
            float L;
            float w[WS];
            const bool alive = merge_weights(lse, w, L);
            if (qv) st_stream(a.out_lse + dst, L);
            __syncwarp();                                   // the previous chunk's table is read
#pragma unroll
            for (int r = 0; r < WS; r += 4)
                *reinterpret_cast<float4*>(wtab + lane * WS + r) =
                    make_float4(w[r], w[r + 1], w[r + 2], w[r + 3]);
            dtab[lane] = alive ? dst : ~dst;
            __syncwarp();                                   // the table is visible to the warp
        }
        // ---------------- phase B: this step's RPI rows, G lanes per row
        const int k = ((step + rot) & (STEPS - 1)) * RPI + sub;     // row of the chunk
        if (k < cn) {
            int64_t db = dtab[k];
            const bool dead = db < 0;
            if (dead) db = ~db;
            float ws[WS];
#pragma unroll
            for (int r = 0; r < WS; r += 4) {
                const float4 f = *reinterpret_cast<const float4*>(wtab + k * WS + r);
                ws[r] = f.x;
                ws[r + 1] = f.y;
                ws[r + 2] = f.z;
                ws[r + 3] = f.w;
            }
            const uint4* sl = ring + slot * Ring::kSlotVecs + lane;
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
                    uint4 v = sl[(e * WMAX + r) * 32];
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
        if (++step == STEPS) {
            step = 0;
            ++ci;
        }
        if (++slot == NST) slot = 0;
    }
    cp_async_wait<0>();
}

}  // namespace cplse
