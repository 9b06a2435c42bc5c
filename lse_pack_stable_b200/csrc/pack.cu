// Max/sum-aware DCP pack: forms LSE = softmax_max + log(softmax_sum) (-inf for
// invalid statistics) while writing the destination-major send packet.
//
// Source: vLLM-Ascend pull request "[Performance][Attention] Fuse local SFA LSE
// formation into DCP pack", section "What this PR does / why we need it?"
// (After pipeline: the LSE comes out of the pack itself, with no separate LSE
// tensor; the rule for invalid statistics) and "How was this patch tested?"
// (scatter_dim 0 and 1, non-contiguous output/max/sum strides).
//
// Two kernels. Back-to-back rows (so_h == D), head or token chunks, take the
// 2-D block copy further down. Everything else takes the row kernel: a warp
// owns chunks of 32 consecutive source rows (r, t, h) in input order. Phase A:
// lane i forms the LSE of row i (coalesced max/sum loads) and writes it to the
// LSE region. Phase B: G lanes copy one row's D elements with 16-byte vectors;
// U steps of loads are in flight before the first store.
#include <math.h>

#include "common.cuh"
#include "launch.h"
#include "rowcombine.cuh"

namespace cplse {
namespace {

constexpr int kPackThreads = 128;

// 64-bit quotient and remainder, on the 32-bit path when both operands fit.
__device__ __forceinline__ void divmod_pack(int64_t x, int64_t d, int64_t& q, int64_t& r)
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

template <int G, int VPL, int U, bool FROM_LSE>
__global__ void __launch_bounds__(kPackThreads) pack_kernel(const PackArgs a)
{
    constexpr int RPI = 32 / G;
    constexpr int STEPS = 32 / RPI;
    static_assert(STEPS % U == 0, "U must divide the steps of a chunk");
    const int lane = threadIdx.x & 31;
    const int sub = lane / G;
    const int gl = lane % G;
    const int64_t warp = ((int64_t)blockIdx.x * kPackThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kPackThreads) >> 5;
    const int64_t nchunks = (a.rows + 31) >> 5;
    const int V = a.D >> 3;
    const int64_t TH = a.T * a.H;
    const int64_t block_rows = a.T * a.Hc;   // rows of one [src][dst] packet block

    for (int64_t c = warp; c < nchunks; c += nwarps) {
        // ---------------- phase A: lane owns source row q = (r, t, h)
        const int64_t q = c * 32 + lane;
        const bool qv = q < a.rows;
        int64_t src_row = 0, dst_row = 0;
        if (qv) {
            int64_t r, rem, t, h;
            divmod_pack(q, TH, r, rem);
            divmod_pack(rem, (int64_t)a.H, t, h);
            int64_t j, slot;
            if (a.scatter_dim == 1) {
                divmod_pack(h, (int64_t)a.Hc, j, slot);
                slot += t * a.Hc;
            } else {
                int64_t tc;
                divmod_pack(t, a.Tc, j, tc);
                slot = tc * a.H + h;
            }
            dst_row = (r * a.W + j) * block_rows + slot;
            src_row = r * a.so_r + t * a.so_t + h * a.so_h;
            if (FROM_LSE) {
                // legacy: the materialized LSE moves into the packet layout
                st_stream(a.pkt_lse + dst_row, ld_ro(a.lse + r * a.sm_r + t * a.sm_t + h * a.sm_h));
            } else {
                const float m = ld_ro(a.smax + r * a.sm_r + t * a.sm_t + h * a.sm_h);
                const float s = ld_ro(a.ssum + r * a.ss_r + t * a.ss_t + h * a.ss_h);
                const bool ok = isfinite(m) && isfinite(s) && s > 0.f;
                st_stream(a.pkt_lse + dst_row, ok ? m + logf(s) : -INFINITY);
            }
        }

        // ---------------- phase B: copy the payload rows
#pragma unroll 1
        for (int s0 = 0; s0 < STEPS; s0 += U) {
            int64_t sb[U], db[U];
            bool rv[U];
            uint4 v[U][VPL];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = (s0 + u) * RPI + sub;
                sb[u] = __shfl_sync(kFull, src_row, k);
                db[u] = __shfl_sync(kFull, dst_row, k);
                rv[u] = c * 32 + k < a.rows;
#pragma unroll
                for (int e = 0; e < VPL; ++e) {
                    const int vec = gl + e * G;
                    if (rv[u] && vec < V)
                        v[u][e] = ld_ro(reinterpret_cast<const uint4*>(a.o + sb[u]) + vec);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int e = 0; e < VPL; ++e) {
                    const int vec = gl + e * G;
                    if (rv[u] && vec < V)
                        st_stream(reinterpret_cast<uint4*>(a.pkt_o + db[u] * a.D) + vec, v[u][e]);
                }
        }

    }
}

template <int G, int VPL, bool FROM_LSE>
cudaError_t launch_pack_inst(const PackArgs& a, cudaStream_t s)
{
    constexpr int U0 = VPL >= 8 ? 1 : 8 / VPL;
    constexpr int U = U0 > G ? G : U0;
    constexpr auto kern = pack_kernel<G, VPL, U, FROM_LSE>;
    int per_sm = 0;
    {
        const cudaError_t e = resident_blocks<kern>(kPackThreads, 0, per_sm);
        if (e != cudaSuccess) return e;
    }
    const int64_t nchunks = (a.rows + 31) / 32;
    int64_t blocks = (nchunks + kPackThreads / 32 - 1) / (kPackThreads / 32);
    const int64_t cap = (int64_t)per_sm * sm_count();
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    kern<<<(unsigned)blocks, kPackThreads, 0, s>>>(a);
    return cudaGetLastError();
}

// Block-copy pack of rank rows that are back to back (so_h == D). Packet block
// (r, j) is NB rows of RE contiguous elements:
//   head chunks  (scatter_dim 1): NB = T rows of Hc*D, row t read from source
//                (r, t) at head j*Hc;
//   token chunks (scatter_dim 0): NB = T/W rows of H*D, row tc read from source
//                (r, j*T/W + tc), i.e. the whole block is one run of token rows.
// Each thread moves U 16-byte vectors (all loads in flight before the first
// store) and the grid covers every block once, so blocks retire and start
// continuously; grid.y is the source rank, grid.x enumerates (column,
// destination) with the destination fastest. Columns below lse_cols form (or,
// legacy, move) the block's LSE values, the rest copy the payload.
#ifndef CPLSE_PACK_U
#define CPLSE_PACK_U 8
#endif
constexpr int kBlockThreads = 256;
constexpr int kBlockU = CPLSE_PACK_U;

// rows per packet block and 16-byte vectors per packet row
__host__ __device__ __forceinline__ void pack_block_shape(const PackArgs& a, int64_t& nb, int64_t& rv)
{
    const bool tok = a.scatter_dim == 0;
    nb = tok ? a.Tc : a.T;
    rv = ((int64_t)(tok ? a.H : a.Hc) * a.D) >> 3;
}

template <bool FROM_LSE>
__global__ void __launch_bounds__(kBlockThreads)
pack_block_kernel(const PackArgs a, int64_t pay_cols, int64_t lse_cols)
{
    // Grid order: the destination j varies fastest, so that the blocks running
    // at the same time copy every head chunk of the same source rows, i.e. read
    // whole token rows between them instead of one Hc*D piece of each row
    // (stress 5712 -> 5386 us, mla 2632 -> 2526 us). The LSE columns come
    // first, so that their latency overlaps the payload copy.
    const int j = (int)(blockIdx.x % (unsigned)a.W);
    const int r = blockIdx.y;                               // source rank
    const int rj = r * a.W + j;                             // packet block (r, j)
    int64_t bx = blockIdx.x / (unsigned)a.W;
    bx = bx < lse_cols ? pay_cols + bx : bx - lse_cols;     // payload columns: bx < pay_cols
    const bool tok = a.scatter_dim == 0;
    int64_t nb, rv;
    pack_block_shape(a, nb, rv);
    if (bx < pay_cols) {
        const int64_t nvec = nb * rv;
        const int64_t first = tok ? (int64_t)j * a.Tc * a.so_t : (int64_t)j * a.Hc * a.D;
        const uint4* src = reinterpret_cast<const uint4*>(a.o + r * a.so_r + first);
        uint4* dst = reinterpret_cast<uint4*>(a.pkt_o) + (int64_t)rj * nvec;
        const int64_t st8 = a.so_t >> 3;
        const int64_t base = bx * kBlockThreads * kBlockU + threadIdx.x;
        uint4 v[kBlockU];
#pragma unroll
        for (int u = 0; u < kBlockU; ++u) {
            const int64_t k = base + (int64_t)u * kBlockThreads;
            if (k < nvec) {
                int64_t t, off;
                divmod_pack(k, rv, t, off);
                v[u] = ld_ro(src + t * st8 + off);
            }
        }
#pragma unroll
        for (int u = 0; u < kBlockU; ++u) {
            const int64_t k = base + (int64_t)u * kBlockThreads;
            if (k < nvec) st_stream(dst + k, v[u]);
        }
    } else {
        // packet LSE k of block (r, j): row k / L, column k % L, L = H (tokens) or Hc (heads)
        const int64_t L = tok ? a.H : a.Hc;
        const int64_t block_rows = nb * L;
        const int64_t base = (bx - pay_cols) * kBlockThreads * 4 + threadIdx.x;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t k = base + (int64_t)u * kBlockThreads;
            if (k >= block_rows) break;
            int64_t row, col;
            divmod_pack(k, L, row, col);
            const int64_t t = tok ? (int64_t)j * a.Tc + row : row;
            const int64_t h = tok ? col : (int64_t)j * a.Hc + col;
            float lv;
            if (FROM_LSE) {
                lv = ld_ro(a.lse + r * a.sm_r + t * a.sm_t + h * a.sm_h);
            } else {
                const float m = ld_ro(a.smax + r * a.sm_r + t * a.sm_t + h * a.sm_h);
                const float sv = ld_ro(a.ssum + r * a.ss_r + t * a.ss_t + h * a.ss_h);
                const bool ok = isfinite(m) && isfinite(sv) && sv > 0.f;
                lv = ok ? m + logf(sv) : -INFINITY;
            }
            st_stream(a.pkt_lse + (int64_t)rj * block_rows + k, lv);
        }
    }
}

template <bool FROM_LSE>
cudaError_t launch_pack_blocks(const PackArgs& a, cudaStream_t s)
{
    int64_t nb, rv;
    pack_block_shape(a, nb, rv);
    const int64_t L = a.scatter_dim == 0 ? a.H : a.Hc;
    const int64_t pay_cols = (nb * rv + kBlockThreads * kBlockU - 1) / (kBlockThreads * kBlockU);
    const int64_t lse_cols = (nb * L + kBlockThreads * 4 - 1) / (kBlockThreads * 4);
    if ((pay_cols + lse_cols) * a.W > 0x7fffffff) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)((pay_cols + lse_cols) * a.W), (unsigned)a.nsrc);
    pack_block_kernel<FROM_LSE><<<grid, kBlockThreads, 0, s>>>(a, pay_cols, lse_cols);
    return cudaGetLastError();
}

template <bool FROM_LSE>
cudaError_t launch_pack_l(const PackArgs& a, cudaStream_t s)
{
    // back-to-back rows: block copies (head or token chunks); anything else: row by row
    if (a.so_h == a.D) return launch_pack_blocks<FROM_LSE>(a, s);
    const RowShape rs = row_shape(a.D);
    switch (rs.G * 10 + rs.VPL) {
    case 41: return launch_pack_inst<4, 1, FROM_LSE>(a, s);
    case 81: return launch_pack_inst<8, 1, FROM_LSE>(a, s);
    case 161: return launch_pack_inst<16, 1, FROM_LSE>(a, s);
    case 321: return launch_pack_inst<32, 1, FROM_LSE>(a, s);
    case 322: return launch_pack_inst<32, 2, FROM_LSE>(a, s);
    default: return launch_pack_inst<32, 4, FROM_LSE>(a, s);
    }
}

// Legacy first step: lse[q] for q = (r, t, h) in row-major order, four rows per
// thread, one pass over the grid.
constexpr int kMatThreads = 256;

__global__ void __launch_bounds__(kMatThreads) lse_materialize_kernel(const PackArgs a, float* lse)
{
    const int64_t TH = a.T * a.H;
    const int64_t q0 = ((int64_t)blockIdx.x * kMatThreads + threadIdx.x) * 4;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int64_t q = q0 + k;
        if (q >= a.rows) break;
        int64_t r, rem, t, h;
        divmod_pack(q, TH, r, rem);
        divmod_pack(rem, (int64_t)a.H, t, h);
        const float m = ld_ro(a.smax + r * a.sm_r + t * a.sm_t + h * a.sm_h);
        const float sv = ld_ro(a.ssum + r * a.ss_r + t * a.ss_t + h * a.ss_h);
        const bool ok = isfinite(m) && isfinite(sv) && sv > 0.f;
        st_stream(lse + q, ok ? m + logf(sv) : -INFINITY);
    }
}

}  // namespace

cudaError_t launch_pack(const PackArgs& a, cudaStream_t s)
{
    return a.lse != nullptr ? launch_pack_l<true>(a, s) : launch_pack_l<false>(a, s);
}

cudaError_t launch_lse_materialize(const PackArgs& a, float* lse, cudaStream_t s)
{
    const int64_t blocks = (a.rows + 4 * kMatThreads - 1) / (4 * kMatThreads);
    if (blocks > 0x7fffffff) return cudaErrorInvalidConfiguration;
    lse_materialize_kernel<<<(unsigned)blocks, kMatThreads, 0, s>>>(a, lse);
    return cudaGetLastError();
}

}  // namespace cplse
