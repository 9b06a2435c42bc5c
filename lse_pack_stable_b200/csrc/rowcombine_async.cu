// Shared-memory-staged stable log-sum-exp merge: launch planning for the
// fused pack->a2a->combine and for the combine of a received packet.
#include <type_traits>

#include "rowcombine_async.cuh"

namespace cplse {
namespace {

// Stages per warp: enough that kAsyncInflight bytes of every warp's payload
// are in flight (NST-1 slots), between 3 and 8. Measured on B200: shallow
// rings with more resident warps beat deep ones (4 KB per warp, i.e. NST = 3
// on every workload here: decode 35.0 us against 39.4 us at 16 KB).
template <int WMAX, int VPL>
constexpr int stages_for()
{
    constexpr int slot = VPL * WMAX * 32 * 16;
    constexpr int n = kAsyncInflight / slot + 1;
    return n < 3 ? 3 : (n > 8 ? 8 : n);
}

template <typename P, int MODE, int WMAX, int G, int VPL>
cudaError_t launch_async_inst(const CombineArgs& a, cudaStream_t s)
{
    constexpr int NST = stages_for<WMAX, VPL>();
    using Ring = AsyncRing<WMAX, G, VPL, NST>;
    constexpr int smem = (kAsyncThreads / 32) * Ring::kWarpBytes;
    constexpr auto kern = rowcombine_async_kernel<P, MODE, WMAX, G, VPL, NST>;
    int per_sm = 0;
    {
        const cudaError_t e = resident_blocks<kern>(kAsyncThreads, smem, per_sm);
        if (e != cudaSuccess) return e;
    }
    // the ring's groups in flight: NST-1 steps of 32/G rows
    const int64_t blocks = merge_grid(a.rows, kAsyncThreads, per_sm, (NST - 1) * (32 / G));
    return launch_pdl(kern, (unsigned)blocks, kAsyncThreads, smem, s, a);
}

// Shared-memory staging for up to 8 ranks with rows of one 16-byte vector per
// lane (D <= 256); register staging otherwise. From 16 ranks on, one step of
// every rank is 8 KB or more per warp and the ring leaves too few warps
// resident (stress, W=16 D=128: 2.95 ms against 3.3-4.4 ms). For wider rows the
// register path with its per-warp weight table keeps 16 vectors per lane in
// flight and measured faster (mla, W=8 D=512: 1405 against 1516 us); for
// D = 128 at 4 and 8 ranks the ring stays ahead (ulysses: 572 against 580 us).
template <typename P, int MODE, int WMAX, int G, int VPL>
cudaError_t launch_staged(const CombineArgs& a, cudaStream_t s)
{
    if constexpr (WMAX >= 16 || VPL >= 2)
        return launch_rowcombine_inst<P, MODE, WMAX, G, VPL>(a, s);
    else
        return launch_async_inst<P, MODE, WMAX, G, VPL>(a, s);
}

template <typename P, int MODE, int WMAX>
cudaError_t launch_async_w(const CombineArgs& a, cudaStream_t s)
{
    const RowShape rs = row_shape(a.D);
    switch (rs.G * 10 + rs.VPL) {
    case 41: return launch_staged<P, MODE, WMAX, 4, 1>(a, s);
    case 81: return launch_staged<P, MODE, WMAX, 8, 1>(a, s);
    case 161: return launch_staged<P, MODE, WMAX, 16, 1>(a, s);
    case 321: return launch_staged<P, MODE, WMAX, 32, 1>(a, s);
    case 322: return launch_staged<P, MODE, WMAX, 32, 2>(a, s);
    default: return launch_staged<P, MODE, WMAX, 32, 4>(a, s);
    }
}

template <typename P, int MODE>
cudaError_t launch_async_p(const CombineArgs& a, cudaStream_t s)
{
    if (a.W <= 2) return launch_async_w<P, MODE, 2>(a, s);
    if (a.W <= 4) return launch_async_w<P, MODE, 4>(a, s);
    if (a.W <= 8) return launch_async_w<P, MODE, 8>(a, s);
    if (a.W <= 16) return launch_async_w<P, MODE, 16>(a, s);
    return launch_async_w<P, MODE, 32>(a, s);
}

}  // namespace

cudaError_t launch_fused_async(const CombineArgs& a, Dtype dt, cudaStream_t s)
{
    return dt == Dtype::kBf16 ? launch_async_p<Bf16, kModeFused>(a, s)
                              : launch_async_p<Fp16, kModeFused>(a, s);
}

cudaError_t launch_combine_async(const CombineArgs& a, Dtype dt, cudaStream_t s)
{
    return dt == Dtype::kBf16 ? launch_async_p<Bf16, kModeCombine>(a, s)
                              : launch_async_p<Fp16, kModeCombine>(a, s);
}

}  // namespace cplse
