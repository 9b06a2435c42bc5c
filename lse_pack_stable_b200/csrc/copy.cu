// Layout kernels that move bytes without arithmetic:
//  - the all-to-all's block permutation between W simulated ranks
//    (vLLM-Ascend "Fuse local SFA LSE formation into DCP pack", Before/After
//    pipelines: the HCCL All2All of the packed layout);
//  - the Ulysses sequence-scatter/head-gather transform and its inverse
//    (FastVideo "[perf] Probe H3 chunked all-to-all with direct output
//    slices": all_to_all_4D(x, 2, 1) and all_to_all_4D(x, 1, 2)).
// Every access is the widest vector (16, 8, 4, 2 or 1 bytes) that the block
// size and both base addresses allow; several loads are in flight per thread
// before the first store.
#include "common.cuh"
#include "launch.h"

namespace cplse {
namespace {

constexpr int kCopyThreads = 256;

// Loads: the block permutation reads through the read-only path (1 % faster
// than evict-first on a 16-rank packet); the Ulysses copies keep the
// evict-first hint, which measured faster there (seq->head 361 against 383 us).
template <typename V>
__device__ __forceinline__ V ld_cs(const V* p) { return __ldcs(p); }
template <typename V>
__device__ __forceinline__ V ld_nc(const V* p) { return __ldg(p); }
template <typename V>
__device__ __forceinline__ void st_cs(V* p, V v) { __stcs(p, v); }

// recv[j][r] = send[r][j]; grid.y enumerates destination blocks d = j*W + r.
// Each thread moves U vectors, U loads in flight before the first store; the
// grid covers every vector once (no grid-stride loop), so blocks retire and
// new ones start continuously instead of marching in lockstep.
template <typename V, int U>
__global__ void __launch_bounds__(kCopyThreads)
permute_kernel(const V* __restrict__ send, V* __restrict__ recv, int W, int64_t nvec)
{
    const int d = blockIdx.y;
    const int j = d / W, r = d - j * W;
    const V* src = send + (int64_t)(r * W + j) * nvec;
    V* dst = recv + (int64_t)d * nvec;
    const int64_t base = (int64_t)blockIdx.x * kCopyThreads * U + threadIdx.x;
    V v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t i = base + (int64_t)u * kCopyThreads;
        if (i < nvec) v[u] = ld_nc(src + i);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t i = base + (int64_t)u * kCopyThreads;
        if (i < nvec) st_cs(dst + i, v[u]);
    }
}

#ifndef CPLSE_PERMUTE_U
#define CPLSE_PERMUTE_U 8
#endif

template <typename V>
cudaError_t launch_permute_v(const void* send, void* recv, int W, int64_t block_bytes,
                             cudaStream_t s)
{
    constexpr int U = CPLSE_PERMUTE_U;
    const int64_t nvec = block_bytes / (int64_t)sizeof(V);
    const int64_t gx = (nvec + kCopyThreads * U - 1) / (kCopyThreads * U);
    if (gx > 0x7fffffff) return cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)gx, (unsigned)(W * W));
    permute_kernel<V, U><<<grid, kCopyThreads, 0, s>>>(static_cast<const V*>(send),
                                                      static_cast<V*>(recv), W, nvec);
    return cudaGetLastError();
}

// One warp per contiguous chunk of Hc*D elements, K chunks per iteration (all
// their loads in flight before the first store).
//   mode 0 (seq->head): chunk c = ((r*B + b)*S_l + s)*W + j of the input
//       lands at chunk (j*B + b)*S + r*S_l + s of the output;
//   mode 1 (head->seq): chunk c = (r*B + b)*S + (j*S_l + s) of the input
//       lands at chunk ((j*B + b)*S_l + s)*W + r of the output.
// x / d and x % d, on the 32-bit path when both operands fit.
__device__ __forceinline__ int64_t div_u(int64_t x, int64_t d, int64_t& rem)
{
    if (((uint64_t)x | (uint64_t)d) < (1ull << 32)) {
        const uint32_t q = (uint32_t)x / (uint32_t)d;
        rem = (uint32_t)x - q * (uint32_t)d;
        return q;
    }
    const int64_t q = x / d;
    rem = x - q * d;
    return q;
}

template <int MODE>
__device__ __forceinline__ int64_t ulysses_dst_chunk(const UlyssesArgs& a, int64_t c)
{
    int64_t j, s, b, sg;
    if (MODE == 0) {
        int64_t rest = div_u(c, a.W, j);
        rest = div_u(rest, a.S_l, s);
        const int64_t r = div_u(rest, a.B, b);
        return (j * a.B + b) * a.S + r * a.S_l + s;
    }
    const int64_t rest = div_u(c, a.S, sg);
    const int64_t r = div_u(rest, a.B, b);
    j = div_u(sg, a.S_l, s);
    return ((j * a.B + b) * a.S_l + s) * a.W + r;
}

template <typename V, int MODE, int K, int UNR>
__global__ void __launch_bounds__(kCopyThreads)
ulysses_kernel(const V* __restrict__ in, V* __restrict__ out, const UlyssesArgs a, int64_t cv)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * kCopyThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kCopyThreads) >> 5;
    for (int64_t c0 = warp; c0 < a.nchunks; c0 += nwarps * K) {
        int64_t dcs[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const int64_t c = c0 + k * nwarps;
            dcs[k] = c < a.nchunks ? ulysses_dst_chunk<MODE>(a, c) : 0;
        }
        for (int64_t v0 = lane; v0 < cv; v0 += 32 * UNR) {
            V x[K][UNR];
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const int64_t c = c0 + k * nwarps;
#pragma unroll
                for (int u = 0; u < UNR; ++u) {
                    const int64_t i = v0 + 32 * u;
                    if (c < a.nchunks && i < cv) x[k][u] = ld_cs(in + c * cv + i);
                }
            }
#pragma unroll
            for (int k = 0; k < K; ++k) {
                const int64_t c = c0 + k * nwarps;
#pragma unroll
                for (int u = 0; u < UNR; ++u) {
                    const int64_t i = v0 + 32 * u;
                    if (c < a.nchunks && i < cv) st_cs(out + dcs[k] * cv + i, x[k][u]);
                }
            }
        }
    }
}

// The transforms as 2-D block copies, one grid row per (dst rank j, src rank r)
// and one grid layer per batch plane b: S_l rows of Hc*D elements each. In the
// pull form (one real destination) the grid rows are the source ranks alone,
// each read through its own base address, and j is the destination.
//   mode 0: source rows s of in[r][b] at heads j*Hc (row stride H*D) land as
//           the contiguous rows r*S_l + s of out[j][b];
//   mode 1: the contiguous source rows j*S_l + s of in[r][b] land as rows s of
//           out[j][b] at heads r*Hc (row stride H*D).
// Each thread moves U vectors, all loads in flight before the first store;
// the grid covers every block once.
// vectors per thread: 4 measured best on B200 (Ulysses workload: 376 / 129 us
// at 4, 431 / 149 us at 8, 599 / 196 us at 16)
#ifndef CPLSE_ULY_U
#define CPLSE_ULY_U 4
#endif
constexpr int kUlyU = CPLSE_ULY_U;

template <typename V, int MODE>
__global__ void __launch_bounds__(kCopyThreads)
ulysses_block_kernel(const V* __restrict__ in, V* __restrict__ out, const UlyssesArgs a, int64_t cv)
{
    constexpr int U = kUlyU;
    const int jr = blockIdx.y;
    const int j = a.pull ? a.dst : jr / a.W;
    const int r = a.pull ? jr : jr - j * a.W;
    const int64_t b = blockIdx.z;
    const int64_t rowv = (int64_t)a.W * cv;          // a full H*D row, in vectors
    const int64_t plane = (int64_t)a.B * a.S_l * rowv;   // one rank's tensor, in vectors
    // rank r's input and destination j's output
    const V* in_r = a.pull ? static_cast<const V*>(a.ins[r]) : in + (int64_t)r * plane;
    V* out_j = a.pull ? out : out + (int64_t)j * plane;
    const V* src;
    V* dst;
    int64_t src_stride, dst_stride;
    if (MODE == 0) {
        src = in_r + (b * a.S_l) * rowv + (int64_t)j * cv;
        dst = out_j + (b * a.S + (int64_t)r * a.S_l) * cv;
        src_stride = rowv;
        dst_stride = cv;
    } else {
        src = in_r + (b * a.S + (int64_t)j * a.S_l) * cv;
        dst = out_j + (b * a.S_l) * rowv + (int64_t)r * cv;
        src_stride = cv;
        dst_stride = rowv;
    }
    const int64_t nvec = a.S_l * cv;
    const int64_t base = (int64_t)blockIdx.x * kCopyThreads * U + threadIdx.x;
    V v[U];
    int64_t row[U], col[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t k = base + (int64_t)u * kCopyThreads;
        row[u] = div_u(k, cv, col[u]);
        if (k < nvec) v[u] = ld_cs(src + row[u] * src_stride + col[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t k = base + (int64_t)u * kCopyThreads;
        if (k < nvec) st_cs(dst + row[u] * dst_stride + col[u], v[u]);
    }
}

template <typename V, int MODE>
cudaError_t launch_ulysses_v(const UlyssesArgs& a, cudaStream_t s)
{
    const int64_t cv = a.chunk_bytes / (int64_t)sizeof(V);
    constexpr int U = kUlyU;
    if (a.B <= 65535) {
        const int64_t gx = (a.S_l * cv + kCopyThreads * U - 1) / (kCopyThreads * U);
        if (gx <= 0x7fffffff) {
            dim3 grid((unsigned)gx, (unsigned)(a.pull ? a.W : a.W * a.W), (unsigned)a.B);
            ulysses_block_kernel<V, MODE><<<grid, kCopyThreads, 0, s>>>(
                static_cast<const V*>(a.in), static_cast<V*>(a.out), a, cv);
            return cudaGetLastError();
        }
    }
    // more batch planes than a grid layer count allows: one warp per chunk
    if (a.pull) return cudaErrorInvalidConfiguration;   // the pull form takes B <= 65535
    constexpr int UNR = 4;
    constexpr int K = 2;
    constexpr auto kern = ulysses_kernel<V, MODE, K, UNR>;
    int per_sm = 0;
    {
        const cudaError_t e = resident_blocks<kern>(kCopyThreads, 0, per_sm);
        if (e != cudaSuccess) return e;
    }
    const int64_t warps_per_block = kCopyThreads / 32;
    int64_t blocks = (a.nchunks + warps_per_block - 1) / warps_per_block;
    const int64_t cap = (int64_t)per_sm * sm_count();
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    kern<<<(unsigned)blocks, kCopyThreads, 0, s>>>(static_cast<const V*>(a.in),
                                                  static_cast<V*>(a.out), a, cv);
    return cudaGetLastError();
}

// Widest power-of-two access (<= 16 bytes) dividing n and both addresses.
int vector_bytes(int64_t n, const void* p, const void* q)
{
    const uint64_t m = (uint64_t)n | (uint64_t)(uintptr_t)p | (uint64_t)(uintptr_t)q;
    for (int w = 16; w > 1; w >>= 1)
        if ((m & (uint64_t)(w - 1)) == 0) return w;
    return 1;
}

template <int MODE>
cudaError_t launch_ulysses_m(const UlyssesArgs& a, cudaStream_t s)
{
    int vb = vector_bytes(a.chunk_bytes, a.in, a.out);
    if (a.pull)
        for (int r = 0; r < a.W; ++r) {
            const int w = vector_bytes(a.chunk_bytes, a.ins[r], a.out);
            if (w < vb) vb = w;
        }
    switch (vb) {
    case 16: return launch_ulysses_v<uint4, MODE>(a, s);
    case 8: return launch_ulysses_v<uint2, MODE>(a, s);
    case 4: return launch_ulysses_v<unsigned int, MODE>(a, s);
    case 2: return launch_ulysses_v<unsigned short, MODE>(a, s);
    default: return launch_ulysses_v<unsigned char, MODE>(a, s);
    }
}

}  // namespace

cudaError_t launch_permute(const void* send, void* recv, int W, int64_t block_bytes,
                           cudaStream_t s)
{
    switch (vector_bytes(block_bytes, send, recv)) {
    case 16: return launch_permute_v<uint4>(send, recv, W, block_bytes, s);
    case 8: return launch_permute_v<uint2>(send, recv, W, block_bytes, s);
    case 4: return launch_permute_v<unsigned int>(send, recv, W, block_bytes, s);
    case 2: return launch_permute_v<unsigned short>(send, recv, W, block_bytes, s);
    default: return launch_permute_v<unsigned char>(send, recv, W, block_bytes, s);
    }
}

cudaError_t launch_ulysses(const UlyssesArgs& a, cudaStream_t s)
{
    return a.mode == 0 ? launch_ulysses_m<0>(a, s) : launch_ulysses_m<1>(a, s);
}

}  // namespace cplse
