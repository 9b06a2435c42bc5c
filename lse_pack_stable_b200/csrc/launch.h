// Internal launcher interface between the C-ABI layer (api.cu) and the kernels.
// Arguments arrive here already validated; launchers only pick a kernel
// instantiation and a grid, enqueue, and report cudaGetLastError().
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace cplse {

enum class Dtype : int { kBf16 = 0, kFp16 = 1 };

// Stable log-sum-exp merge of W contributions per output row. FUSED mode forms
// each contribution's LSE from (max, sum) and reads the partial outputs in
// place; COMBINE mode reads a received packet.
struct CombineArgs {
    const uint16_t* src;      // payload base
    int64_t rank_stride;      // elements between ranks' rows
    // fused: o[r][t][h] at src + r*rank_stride + t*so_t + h*so_h
    int64_t so_t, so_h;
    const float* smax;
    const float* ssum;
    int64_t sm_r, sm_t, sm_h, ss_r, ss_t, ss_h;
    // combine: recv_lse[j][r][n]
    const float* lse;
    uint16_t* out;
    float* out_lse;
    int W, H, Hc, D;
    int64_t T;                // fused: tokens
    int64_t N;                // combine: rows per block
    int64_t rows;             // output rows
    int dense_rows;           // fused: rank rows back to back (so_h == D, so_t == H*D)
    int token_scatter;        // fused: token-chunk exchange, output row (t, h) = source row (t, h);
                              // otherwise head chunks, output row (j, t, hc) for h = j*Hc + hc
};

struct PackArgs {
    const uint16_t* o;
    int64_t so_r, so_t, so_h;
    const float* smax;        // max/sum-aware pack: statistics ...
    const float* ssum;
    int64_t sm_r, sm_t, sm_h, ss_r, ss_t, ss_h;
    const float* lse;         // ... or (legacy) a materialized LSE tensor, strides in sm_*
    uint16_t* pkt_o;
    float* pkt_lse;
    int W, H, Hc, D, scatter_dim;
    int64_t T, Tc;
    int64_t rows;             // nsrc*T*H
    int nsrc;                 // source ranks in this call: W (all simulated ranks) or 1 (one real rank)
};

// The pull-based exchange for one real destination rank: each source rank's
// o/max/sum rows are read where they live (this GPU's memory or a peer's,
// mapped into this process), through a table of per-rank base addresses.
struct PullArgs {
    const uint16_t* o[32];
    const float* smax[32];
    const float* ssum[32];
    int64_t so_t, so_h, sm_t, sm_h, ss_t, ss_h;   // the same layout on every rank
    uint16_t* out;
    float* out_lse;
    int W, H, Hc, D;
    int dst;                  // this destination rank
    int token_scatter;        // 0: head chunk dst (out [T][Hc][D]); 1: token chunk dst (out [T/W][H][D])
    int64_t T, Tc;
    int64_t rows;             // output rows
};

struct UlyssesArgs {
    const void* in;
    void* out;
    int W, B, H, Hc;
    int64_t S_l, S;
    int64_t chunk_bytes;      // Hc*D*elem_bytes
    int64_t nchunks;
    int mode;                 // 0: seq->head, 1: head->seq
    // pull form (one real destination rank): rank r's plane at ins[r] (this
    // GPU's memory or a peer's mapped into this process); out is destination
    // dst's plane alone
    int pull;
    int dst;
    const void* ins[32];
};

// the stable merge, fused (from max/sum, in place) or on a received packet:
// shared-memory-staged (rowcombine_async.cuh) up to 8 ranks, register-staged
// (rowcombine.cuh) from 16; same arithmetic, same bits
cudaError_t launch_fused_async(const CombineArgs& a, Dtype dt, cudaStream_t s);
cudaError_t launch_combine_async(const CombineArgs& a, Dtype dt, cudaStream_t s);
cudaError_t launch_pack(const PackArgs& a, cudaStream_t s);
cudaError_t launch_pull_combine(const PullArgs& a, Dtype dt, cudaStream_t s);
cudaError_t launch_lse_materialize(const PackArgs& a, float* lse, cudaStream_t s);
cudaError_t launch_permute(const void* send, void* recv, int W, int64_t block_bytes,
                           cudaStream_t s);
cudaError_t launch_ulysses(const UlyssesArgs& a, cudaStream_t s);

// Streaming multiprocessors of the current device (cached per device).
int sm_count();

// Resident blocks per SM of kernel K at this block size and dynamic shared
// memory, on the current device. The first call on each device opts K in to
// that much dynamic shared memory there (a per-device function attribute).
// Cached per device and kernel; devices beyond the cache are queried each time.
template <auto K>
cudaError_t resident_blocks(int threads, int smem, int& blocks)
{
    constexpr int kCachedDevices = 64;
    static std::atomic<int> cache[kCachedDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cached = dev >= 0 && dev < kCachedDevices;
    if (cached) {
        blocks = cache[dev].load(std::memory_order_relaxed);
        if (blocks > 0) return cudaSuccess;
    }
    if (smem > 0) {
        e = cudaFuncSetAttribute(K, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
    }
    int n = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, K, threads, (size_t)smem);
    if (e != cudaSuccess) return e;
    blocks = n > 0 ? n : 1;
    if (cached) cache[dev].store(blocks, std::memory_order_relaxed);
    return cudaSuccess;
}

}  // namespace cplse
